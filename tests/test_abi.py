"""The C ABI without a GPU: libcoli.so loads, exports every function that
include/coli.h declares, and rejects bad arguments on the host (these paths
return before any CUDA call)."""
import ctypes as C
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "coli.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(coli_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    import int4_weight_only_sigmoid_b200 as m
    from int4_weight_only_sigmoid_b200 import build
    build.build()
    return m.load()


def test_every_declared_symbol_is_exported(lib):
    import int4_weight_only_sigmoid_b200 as m
    names = _declared()
    assert len(names) >= 11
    assert sorted(m.EXPORTS) == names
    for n in names:
        assert hasattr(lib, n), n


def test_workspace_bytes_host_only(lib):
    import int4_weight_only_sigmoid_b200 as m
    cfg = m.make_config(6144, 2048, 256, 8, 1)
    b1 = m.workspace_bytes(cfg, 1)
    b2048 = m.workspace_bytes(cfg, 2048)
    assert 0 < b1 < b2048
    # y buffer dominates at 2048 tokens: (8 + 1) * 2048 rows of 6144 floats
    assert b2048 >= 9 * 2048 * 6144 * 4
    bad = m.make_config(100, 2048, 256, 8, 1)
    assert m.workspace_bytes(bad, 1) == 0
    bad = m.make_config(6144, 2048, 256, 17, 1)
    assert m.workspace_bytes(bad, 1) == 0


def test_workspace_holds_prefill_buffers_only_for_that_path(lib):
    """Calls of <= 16 tokens take the decode path and need no int8 operand
    rows of x; above that the tensor-core path keeps one int8 row of x per
    (slot, token) and the accumulator starting values.  The documented
    no-allocation limit (8 MiB of scratch) is 22 GLM tokens."""
    import int4_weight_only_sigmoid_b200 as m
    cfg = m.make_config(6144, 2048, 256, 8, 1)
    b16, b17 = (m.workspace_bytes(cfg, t) for t in (16, 17))
    rows17 = 17 * (8 + 1)
    assert b17 - b16 >= rows17 * 6144
    assert m.workspace_bytes(cfg, 22) <= 8 << 20 < m.workspace_bytes(cfg, 23)


def test_bad_arguments_rejected_before_any_cuda_call(lib):
    import int4_weight_only_sigmoid_b200 as m
    assert lib.coli_quantize_act_q8(None, 1, 64, None, None, None) == m.COLI_EINVAL
    assert b"null pointer" in lib.coli_last_error()
    assert lib.coli_quantize_act_q8(C.c_void_p(16), 1, 40, C.c_void_p(16), C.c_void_p(16), None) == m.COLI_EINVAL
    assert b"multiple of 32" in lib.coli_last_error()
    assert lib.coli_quantize_rows_int4(C.c_void_p(8), 2, 64, C.c_void_p(16), C.c_void_p(16), None) == m.COLI_EINVAL
    assert b"aligned" in lib.coli_last_error()
    assert lib.coli_quantize_rows_int4(None, 0, 64, None, None, None) == m.COLI_OK  # nothing to do
    cfg = m.make_config(6144, 2048, 256, 8, 1)
    e = m.Expert()
    assert lib.coli_moe_expert_ffn(C.byref(cfg), C.byref(e), None, None, 1, None, None, 0, None) == m.COLI_EINVAL
    L = m.MoeLayerC(cfg, None, None, None, None)
    assert lib.coli_moe_layer_forward(C.byref(L), None, 1, None, None, 0, None) == m.COLI_EINVAL
    assert lib.coli_moe_route(None, None, 1, None, None, None, None) == m.COLI_EINVAL
    assert lib.coli_moe_bucket(None, 1, 8, 1000, None, None, None, None) == m.COLI_EINVAL
    assert lib.coli_rmsnorm(None, 1, 100, 1e-5, None, None) == m.COLI_EINVAL
    assert lib.coli_debug_block_partials(None, 0, None, 1, 64, 1, None, None) == m.COLI_EINVAL
    assert lib.coli_moe_stack_forward(None, 0, None, 1, 1e-5, None, None, 0, None) == m.COLI_EINVAL
    assert lib.coli_requantize_fp8_int4(None, None, 4, 40, 128, None, None, None) == m.COLI_EINVAL
    assert b"multiple of 32" in lib.coli_last_error()
    assert lib.coli_requantize_fp8_int4(None, None, 4, 64, 12, None, None, None) == m.COLI_EINVAL
    assert b"block" in lib.coli_last_error()
    assert lib.coli_requantize_fp8_int4(None, None, 0, 64, 128, None, None, None) == m.COLI_OK
    assert lib.coli_debug_capture_partials(None, 100) == m.COLI_EINVAL
    assert lib.coli_debug_capture_partials(C.c_void_p(8), 100) == m.COLI_EINVAL
    assert lib.coli_debug_wait_probe(None, 1000, None) == m.COLI_EINVAL
    assert lib.coli_debug_wait_probe(C.c_void_p(256), -1, None) == m.COLI_EINVAL
    assert lib.coli_sync_status(C.c_void_p(8), None) == m.COLI_EINVAL  # misaligned workspace


def test_noalloc_rejects_token_counts_outside_range_before_sizing(lib):
    """n_tok < 0 or > 2^24 is refused before the scratch need is computed
    (whose size arithmetic would otherwise run on absurd counts)."""
    import int4_weight_only_sigmoid_b200 as m
    cfg = m.make_config(6144, 2048, 256, 8, 1)
    L = m.MoeLayerC(cfg, None, None, None, None)
    for n in (-1, (1 << 24) + 1, 1 << 40, (1 << 62)):
        assert lib.coli_moe_layer_forward_noalloc(C.byref(L), None, n, None, None) == m.COLI_EINVAL
        assert b"n_tok" in lib.coli_last_error()


def test_prepared_bytes_and_prepare_arguments(lib):
    """The streaming copy is as large as the row-major weights (plus the
    scales, each expert padded to 256 bytes); shapes without a streaming
    layout report 0; bad buffers are refused before any CUDA call."""
    import int4_weight_only_sigmoid_b200 as m
    cfg = m.make_config(6144, 2048, 256, 8, 1)
    per_expert = 3 * 2048 * 6144 // 2 + (2 * 2048 + 6144) * 4
    per_expert = (per_expert + 255) // 256 * 256
    assert m.prepared_bytes(cfg) == 257 * per_expert
    tiny = m.make_config(256, 128, 16, 4, 1)
    assert m.prepared_bytes(tiny) == 17 * ((3 * 128 * 256 // 2 + (2 * 128 + 256) * 4 + 255) // 256 * 256)
    assert m.prepared_bytes(m.make_config(384, 128, 16, 4, 1)) == 0  # hidden/32 = 12
    assert m.prepared_bytes(m.make_config(256, 96, 16, 4, 1)) == 0   # inter not a multiple of 128
    ex = (m.Expert * 17)(*[m.Expert(256, 256, 256, 256, 256, 256) for _ in range(17)])
    L = m.MoeLayerC(tiny, 256, 256, C.cast(ex, C.POINTER(m.Expert)), C.cast(ex, C.POINTER(m.Expert)), None)
    n = m.prepared_bytes(tiny)
    assert lib.coli_moe_prepare(C.byref(L), None, n, None) == m.COLI_EINVAL
    assert lib.coli_moe_prepare(C.byref(L), C.c_void_p(4096 + 16), n, None) == m.COLI_EINVAL
    assert b"aligned" in lib.coli_last_error()
    assert lib.coli_moe_prepare(C.byref(L), C.c_void_p(4096), n - 1, None) == m.COLI_ENOMEM
    L.prepared = 4096 + 128  # a forward refuses a misaligned copy too
    assert lib.coli_moe_layer_forward(C.byref(L), C.c_void_p(256), 1, C.c_void_p(512), C.c_void_p(768), 1 << 20,
                                      None) == m.COLI_EINVAL


def test_int8_weight_config_checks(lib):
    """weight_bits 8: the streaming copy holds one byte per weight; other
    widths are refused; the reference-shape expert call is int4 only."""
    import int4_weight_only_sigmoid_b200 as m
    c8 = m.make_config(6144, 2048, 256, 8, 1, weight_bits=8)
    per_expert = (3 * 2048 * 6144 + (2 * 2048 + 6144) * 4 + 255) // 256 * 256
    assert m.prepared_bytes(c8) == 257 * per_expert
    assert m.workspace_bytes(m.make_config(6144, 2048, 256, 8, 1, weight_bits=5), 1) == 0
    assert m.workspace_bytes(m.make_config(256, 96, 16, 4, 1, weight_bits=8), 1) == 0  # inter % 128
    e = m.Expert(256, 256, 256, 256, 256, 256)
    rc = lib.coli_moe_expert_ffn(C.byref(c8), C.byref(e), C.c_void_p(256), C.c_void_p(256), 1, C.c_void_p(256),
                                 C.c_void_p(256), 1 << 30, None)
    assert rc == m.COLI_EINVAL and b"int4" in lib.coli_last_error()
    assert lib.coli_quantize_rows_int8(C.c_void_p(16), 2, 40, C.c_void_p(16), C.c_void_p(16), None) == m.COLI_EINVAL


def test_zero_tokens_is_ok_without_touching_pointers(lib):
    import int4_weight_only_sigmoid_b200 as m
    assert lib.coli_quantize_act_q8(None, 0, 64, None, None, None) == m.COLI_OK


def test_missing_library_fails_loudly(tmp_path):
    import int4_weight_only_sigmoid_b200 as m
    saved = m._lib
    try:
        m._lib = None
        with pytest.raises(ImportError):
            m.load(str(tmp_path / "nope.so"))
    finally:
        m._lib = saved
