"""The oracle's FP8 (e4m3) -> int4 requantiser ("GLM-5.2-colibri-int4架构解析…",
"GLM-5.2-colibri-int4的量化流程": FP8 e4m3 source, dequantised to F32, then
int4 per row; weight_block_size [128, 128]), pinned to things other than
itself: the e4m3 decode of all 256 codes against torch's float8_e4m3fn
conversion, and the requantiser against the separately pinned int4 row
quantiser applied to a dequantisation computed with numpy."""
import numpy as np
import pytest


def _torch_e4m3(codes):
    import torch
    t = torch.from_numpy(np.asarray(codes, np.uint8).copy()).view(torch.float8_e4m3fn)
    return t.float().numpy()


def test_e4m3_all_codes_match_library(ora):
    codes = np.arange(256, dtype=np.uint8)
    mine = ora.e4m3_to_f32(codes)
    ref = _torch_e4m3(codes)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(mine), nan)
    assert set(np.nonzero(nan)[0].tolist()) == {0x7F, 0xFF}
    assert np.array_equal(mine[~nan].view(np.uint32), ref[~nan].view(np.uint32))  # signed zeros included


def test_e4m3_landmarks(ora):
    v = ora.e4m3_to_f32(np.array([0x00, 0x80, 0x01, 0x08, 0x38, 0x7E, 0xFE], np.uint8))
    assert v[0] == 0.0 and np.signbit(v[1])
    assert v[2] == 2.0 ** -9                  # smallest subnormal
    assert v[3] == 2.0 ** -6                  # smallest normal
    assert v[4] == 1.0
    assert v[5] == 448.0 and v[6] == -448.0   # largest finite


def _dequant_numpy(codes, scales, block):
    rows, cols = codes.shape
    vals = _torch_e4m3(codes)
    f = np.repeat(np.repeat(scales, block, axis=0), block, axis=1)[:rows, :cols]
    w = (vals.astype(np.float32) * f.astype(np.float32)).astype(np.float32)  # one F32 rounding
    w[~np.isfinite(w)] = 0.0
    return w


@pytest.mark.parametrize("rows,cols,block", [(3, 64, 128), (130, 256, 128), (128, 384, 128), (40, 96, 32),
                                             (257, 160, 64)])
def test_requantize_equals_int4_of_dequantised(ora, syn, rows, cols, block):
    codes, scales = syn.fp8_blocks(rows, cols, block, seed=rows + cols)
    q, s = ora.requantize_fp8_int4(codes, scales, block)
    q_ref, s_ref = ora.quantize_rows_int4(_dequant_numpy(codes, scales, block))
    assert np.array_equal(q, q_ref)
    assert np.array_equal(s.view(np.uint32), s_ref.view(np.uint32))


def test_requantize_special_rows(ora):
    block, cols = 128, 128
    codes = np.zeros((4, cols), np.uint8)      # row 0: all zero -> scale 0, q 0
    codes[1, :] = 0x7F                         # row 1: all NaN codes -> treated as 0
    codes[2, 0] = 0x7E                         # row 2: one 448, rest 0: that element -> 7
    codes[3, :] = 0x38                         # row 3: all 1.0 -> scale f/7, q = 7
    scales = np.array([[0.5]], np.float32)
    q, s = ora.requantize_fp8_int4(codes, scales, block)
    assert s[0] == 0.0 and not q[0].any()
    assert s[1] == 0.0 and not q[1].any()
    assert s[2] == np.float32(224.0) / np.float32(7.0) and q[2, 0] == 0x07 and not q[2, 1:].any()
    assert s[3] == np.float32(0.5) / np.float32(7.0) and (q[3] == 0x77).all()


def test_requantize_overflowing_products_count_as_zero(ora):
    """A tile factor so large that e4m3 * factor overflows F32: those
    elements count as 0 (the same rule as NaN codes); finite ones keep
    their values."""
    codes = np.zeros((1, 64), np.uint8)
    codes[0, 0] = 0x7E          # 448 * 1e37 = inf in F32 -> 0
    codes[0, 1] = 0x01          # 2^-9 * 1e37, finite
    factors = np.array([[1e37]], np.float32)
    q, s = ora.requantize_fp8_int4(codes, factors, 128)
    v = np.float32(2.0 ** -9) * np.float32(1e37)
    assert s[0] == v / np.float32(7.0)
    assert q[0, 0] == 0x70      # element 0 -> 0 (low nibble), element 1 -> 7 (high nibble)
    assert not q[0, 1:].any()
