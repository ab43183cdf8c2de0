"""The int8 expert-weight variant on the GPU ("Colibri：在笔记本上跑744B参数
的AI模型", section "关键特性": int8 / packed int4 / packed int2 kernels):
the int8 row quantiser bit for bit, and the layer forward with int8 experts
against the oracle, bit for bit, on the streaming kernel (prepared layer,
<= 4 tokens) and on the tensor-core kernels (any other call)."""
import numpy as np
import pytest

from tests.helpers import assert_layer_close, bits_equal, oracle_layer_forward

pytestmark = pytest.mark.gpu

_cache = {}


def _np(t):
    return t.detach().cpu().numpy()


def _layer(cfg, prepare):
    from synth.layers import device_layer
    key = (tuple(sorted((k, v) for k, v in cfg.items() if not isinstance(v, (list, dict)))), prepare)
    if key not in _cache:
        if len(_cache) > 2:
            _cache.clear()
        _cache[key] = device_layer(cfg, 0, prepare=prepare)
    return _cache[key]


@pytest.mark.parametrize("rows,cols", [(1, 32), (37, 96), (128, 256), (64, 6144), (96, 2048)])
def test_quantize_rows_int8_bit_exact(coli, ora, syn, rows, cols):
    import torch
    w = syn.normal(rows * cols, 0, 0, 700 + rows, 0.01).reshape(rows, cols)
    w[0, :] = 0.0
    if rows > 2:
        w[1, :6] = np.array([127, 2.5, -3.5, 0.5, -0.5, 126.5], np.float32) * np.float32(2 ** -4)
        w[1, 6:] = 0.0
    q, s = coli.quantize_rows_int8(torch.from_numpy(w).cuda())
    qo, so = ora.quantize_rows_int8(w)
    assert bits_equal(_np(q), qo)
    assert bits_equal(_np(s), so)


def _check(coli, syn, cfg, n_tok, prepare, sample=None):
    import torch
    L = _layer(cfg, prepare)
    x = syn.tokens(cfg, n_tok)
    out = _np(coli.moe_layer_forward(L, torch.from_numpy(x).cuda()))
    sub = np.arange(n_tok) if sample is None else np.sort(np.random.default_rng(3).choice(n_tok, sample, replace=False))
    want, _, _, _ = oracle_layer_forward(cfg, x[sub])
    assert_layer_close(out[sub], want)
    assert bits_equal(out[sub], want)
    return out


@pytest.mark.parametrize("n_tok", [1, 2, 3, 4, 6])
def test_int8_tiny_streaming(coli, syn, n_tok):
    _check(coli, syn, syn.config("tiny", weight_bits=8), n_tok, prepare=True)


@pytest.mark.parametrize("n_tok", [1, 4, 8, 17, 200])
def test_int8_tiny_tensor_cores(coli, syn, n_tok):
    _check(coli, syn, syn.config("tiny", weight_bits=8), n_tok, prepare=False)


@pytest.mark.parametrize("over", [dict(n_shared=0), dict(n_shared=2), dict(top_k=1), dict(norm_topk_prob=False)])
def test_int8_tiny_variants(coli, syn, over):
    cfg = syn.config("tiny", weight_bits=8, **over)
    _check(coli, syn, cfg, 4, prepare=True)
    _check(coli, syn, cfg, 40, prepare=False)


def test_int8_glm_decode1_streaming(coli, syn):
    _check(coli, syn, syn.config("decode1_int8"), 1, prepare=True)


def test_int8_glm_prefill_sampled(coli, syn):
    _check(coli, syn, syn.config("decode1_int8", bias_boost_n=32, bias_boost=0.2), 300, prepare=False, sample=6)


def test_int8_streaming_equals_tensor_cores(coli, syn):
    """The same prepared int8 layer at 4 tokens through both kernel paths."""
    import torch
    cfg = syn.config("tiny", weight_bits=8)
    L = _layer(cfg, True)
    x = torch.from_numpy(syn.tokens(cfg, 4)).cuda()
    a = _np(coli.moe_layer_forward(L, x))
    b = _np(coli.moe_layer_forward(L, x, cstruct=L.cstruct(use_prepared=False)))
    assert bits_equal(a, b)
