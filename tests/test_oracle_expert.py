"""Pins for the oracle's integer dots, row fold, SwiGLU expert and layer.

Sources: "Colibri：在笔记本上跑744B参数的AI模型", "关键特性" (integer dot
kernels with Q8_0-style int8 activations); "GLM-5.2-colibri-int4架构解析…",
sections "GLM-5.2的MoE实现" / "MoE的工作原理" (routed + shared experts,
weighted combine); HN summary (hn.213312.xyz), "已实现的功能" (batched MoE).
Pins: brute-force integer dots, dequantise-then-matmul in double with a
rounding-error bound, the single-expert reduction, a one-hot router, token
independence and permutation equivariance."""
import os

import numpy as np
import pytest

U = 2.0 ** -24
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _qexpert(ora, syn, cfg, layer, e, shared=False):
    mats = []
    for m in (syn.GATE, syn.UP, syn.DOWN):
        w = syn.expert_matrix(cfg, layer, e, m, shared)
        mats.extend(ora.quantize_rows_int4(w))
    return ora.QExpert(*mats)


def _deq(ora, q, s):
    rows = q.shape[0]
    return ora.unpack_int4(q.ravel()).reshape(rows, -1).astype(np.float64) * s[:, None].astype(np.float64)


def test_block_isums_brute_force(ora, syn):
    w = syn.normal(8 * 256, 0, 0, 900, 0.02).reshape(8, 256)
    q, s = ora.quantize_rows_int4(w)
    x = syn.normal(3 * 256, 0, 0, 901, 1.0).reshape(3, 256)
    xq, xd = ora.quantize_act_q8(x)
    qi = ora.unpack_int4(q.ravel()).reshape(8, 256).astype(np.int64)
    for r in range(8):
        for t in range(3):
            got = ora.block_isums(q[r], xq[t])
            want = (qi[r].reshape(8, 32) * xq[t].astype(np.int64).reshape(8, 32)).sum(axis=1)
            assert np.array_equal(got, want)
            assert np.all(np.abs(got) <= 32 * 8 * 127)


def test_block_isums_extremes(ora):
    # -8 * -127 on every element: the largest magnitude a block can reach
    q = ora.pack_int4(np.full(64, -8, np.int8))
    xq = np.full(64, -127, np.int8)
    assert list(ora.block_isums(q, xq)) == [32 * 8 * 127] * 2


@pytest.mark.parametrize("dim", [256, 6144, 2048])
def test_row_dot_against_double_dequant(ora, syn, dim):
    w = syn.normal(6 * dim, 0, 0, 902, 0.01).reshape(6, dim)
    q, s = ora.quantize_rows_int4(w)
    x = syn.normal(2 * dim, 0, 0, 903, 1.0).reshape(2, dim)
    xq, xd = ora.quantize_act_q8(x)
    Wd = _deq(ora, q, s)
    nb = dim // 32
    for t in range(2):
        xdq = xq[t].astype(np.float64) * np.repeat(xd[t].astype(np.float64), 32)
        for r in range(6):
            got = ora.row_dot(q[r], s[r], xq[t], xd[t])
            exact = float(Wd[r] @ xdq)
            isum = ora.block_isums(q[r], xq[t]).astype(np.float64)
            mag = float(np.abs(xd[t].astype(np.float64) * isum).sum()) * float(s[r])
            assert abs(got - exact) <= (nb + 2) * U * mag * 1.01


def test_expert_token_against_double(ora, syn):
    cfg = syn.config("tiny")
    ex = _qexpert(ora, syn, cfg, 0, 3)
    x = syn.tokens(cfg)
    xq, xd = ora.quantize_act_q8(x)
    Wg, Wu, Wd = _deq(ora, ex.gate_q, ex.gate_s), _deq(ora, ex.up_q, ex.up_s), _deq(ora, ex.down_q, ex.down_s)
    for t in range(x.shape[0]):
        y, hq, hd = ora.expert_ffn_token(ex, xq[t], xd[t])
        xdq = xq[t].astype(np.float64) * np.repeat(xd[t].astype(np.float64), 32)
        g = Wg @ xdq
        u = Wu @ xdq
        h = g / (1.0 + np.exp(-g)) * u
        # the oracle's Q8 of h sits within half a step (plus float error) of h
        hdq = hq.astype(np.float64) * np.repeat(hd.astype(np.float64), 32)
        step = np.repeat(hd.astype(np.float64), 32)
        assert np.all(np.abs(hdq - h) <= 0.5 * step + 1e-4 * np.abs(h).max())
        assert np.all(np.abs(hq.reshape(-1, 32)).max(axis=1) == 127)
        # down projection of the oracle's own Q8 h, recomputed in double
        y_ref = Wd @ hdq
        mag = np.abs(Wd) @ np.abs(hdq)
        assert np.all(np.abs(y - y_ref) <= (cfg["inter"] // 32 + 2) * U * mag * 1.01 + 1e-30)


def test_expert_batch_equals_per_token(ora, syn):
    cfg = syn.config("tiny")
    ex = _qexpert(ora, syn, cfg, 0, 5)
    x = syn.tokens(cfg)
    xq, xd = ora.quantize_act_q8(x)
    yb = ora.expert_ffn(ex, xq, xd)
    for t in range(x.shape[0]):
        y, _, _ = ora.expert_ffn_token(ex, xq[t], xd[t])
        assert np.array_equal(y, yb[t])


def _tiny_layer(ora, syn, cfg, layer=0):
    experts = {e: _qexpert(ora, syn, cfg, layer, e) for e in range(cfg["n_experts"])}
    shared = [_qexpert(ora, syn, cfg, layer, 0, shared=True)]
    return syn.router_w(cfg, layer), syn.bias(cfg, layer), experts, shared


def _zero_expert(ora, H, I):
    z = lambda r, c: ora.quantize_rows_int4(np.zeros((r, c), np.float32))
    return ora.QExpert(*z(I, H), *z(I, H), *z(H, I))


def test_single_expert_layer_is_one_swiglu_mlp(ora, syn):
    cfg = syn.config("tiny", n_experts=1, top_k=1, routed_scaling_factor=1.0)
    W, b = syn.router_w(cfg), syn.bias(cfg)
    ex = _qexpert(ora, syn, cfg, 0, 0)
    zero = _zero_expert(ora, cfg["hidden"], cfg["inter"])
    x = syn.tokens(cfg)
    out, idx, w = ora.moe_layer(cfg, W, b, {0: ex}, [zero], x)
    xq, xd = ora.quantize_act_q8(x)
    assert np.all(idx == 0) and np.all(w == 1.0)
    assert np.array_equal(out, ora.expert_ffn(ex, xq, xd))


def test_one_hot_router_reduces_to_scaled_expert(ora, syn):
    cfg = syn.config("tiny", top_k=1)
    W, b, experts, _ = _tiny_layer(ora, syn, cfg)
    x = syn.tokens(cfg)
    W1 = np.zeros_like(W)
    W1[7] = 1.0  # expert 7's logit is sum(x); make it win for every token
    x1 = x.copy()
    x1[:, 0] += 1000.0
    zero = _zero_expert(ora, cfg["hidden"], cfg["inter"])
    out, idx, w = ora.moe_layer(cfg, W1, np.zeros_like(b), experts, [zero], x1)
    assert np.all(idx == 7) and np.all(w == np.float32(2.5))
    xq, xd = ora.quantize_act_q8(x1)
    y = ora.expert_ffn(experts[7], xq, xd)
    assert np.array_equal(out, (np.float32(2.5) * y).astype(np.float32))


def test_layer_token_independence_and_equivariance(ora, syn):
    cfg = syn.config("tiny")
    W, b, experts, shared = _tiny_layer(ora, syn, cfg)
    x = syn.tokens(cfg)
    out, idx, w = ora.moe_layer(cfg, W, b, experts, shared, x)
    sub = [5, 1, 6]
    o2, i2, w2 = ora.moe_layer(cfg, W, b, experts, shared, x[sub])
    assert np.array_equal(o2, out[sub]) and np.array_equal(i2, idx[sub]) and np.array_equal(w2, w[sub])
    perm = np.random.default_rng(0).permutation(x.shape[0])
    o3, _, _ = ora.moe_layer(cfg, W, b, experts, shared, x[perm])
    assert np.array_equal(o3, out[perm])


def test_layer_against_double_combine(ora, syn):
    cfg = syn.config("tiny")
    W, b, experts, shared = _tiny_layer(ora, syn, cfg)
    x = syn.tokens(cfg)
    out, idx, w = ora.moe_layer(cfg, W, b, experts, shared, x)
    xq, xd = ora.quantize_act_q8(x)
    for t in range(x.shape[0]):
        ys = [ora.expert_ffn_token(experts[e], xq[t], xd[t])[0].astype(np.float64) for e in idx[t]]
        ysh = ora.expert_ffn_token(shared[0], xq[t], xd[t])[0].astype(np.float64)
        ref = sum(float(w[t, k]) * ys[k] for k in range(len(ys))) + ysh
        mag = sum(abs(float(w[t, k])) * np.abs(ys[k]) for k in range(len(ys))) + np.abs(ysh)
        assert np.all(np.abs(out[t] - ref) <= 6 * U * mag + 1e-30)


def test_layer_missing_expert_is_an_error(ora, syn):
    cfg = syn.config("tiny")
    W, b, experts, shared = _tiny_layer(ora, syn, cfg)
    x = syn.tokens(cfg)
    _, idx, _ = ora.moe_layer(cfg, W, b, experts, shared, x)
    e0 = int(idx[0, 0])
    del experts[e0]
    with pytest.raises(KeyError):
        ora.moe_layer(cfg, W, b, experts, shared, x)


def test_layer_golden_regression(ora, syn):
    """The tiny layer's output, idx and w as written by tests/golden/make_golden.py
    (oracle + generator only).  Guards the oracle against silent change."""
    cfg = syn.config("tiny")
    W, b, experts, shared = _tiny_layer(ora, syn, cfg)
    x = syn.tokens(cfg)
    out, idx, w = ora.moe_layer(cfg, W, b, experts, shared, x)
    g = {}
    with open(os.path.join(GOLDEN, "tiny_layer.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                k, v = line.split("=", 1)
                g[k.strip()] = v.split()
    assert [int(v) for v in g["idx"]] == idx.ravel().tolist()
    assert [int(v, 16) for v in g["w_bits"]] == w.view(np.uint32).ravel().tolist()
    assert [int(v, 16) for v in g["out_bits"]] == out.view(np.uint32).ravel().tolist()


def test_rmsnorm_against_double(ora, syn):
    x = syn.normal(4 * 6144, 0, 0, 904, 3.0).reshape(4, 6144)
    y = ora.rmsnorm(x, 1e-5)
    xd = x.astype(np.float64)
    ref = xd / np.sqrt((xd ** 2).mean(axis=1, keepdims=True) + 1e-5)
    assert np.abs(y - ref).max() <= 1e-5 * np.abs(ref).max()
    z = ora.rmsnorm(np.zeros((1, 64), np.float32), 1e-5)
    assert np.all(z == 0)
