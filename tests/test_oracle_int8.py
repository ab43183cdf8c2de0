"""Pins for the oracle's int8 expert-weight variant ("Colibri：在笔记本上跑
744B参数的AI模型", section "关键特性": quantisation kernels int8 / packed
int4 / packed int2).  Reading: the int4 row recipe with the int8 range --
scale = absmax/127 per row (F32), q = rint(w/scale) clamped to [-127,127],
one signed byte per element -- and the same Q8_0 integer dot and contract F.

Checked against exact rationals (closed forms, half-way ties), brute-force
integer sums, a double-precision dequantise-then-matmul, and an identity:
an int8 expert whose bytes hold int4-range values equals the packed int4
expert with the same scales, bit for bit, at expert and at layer level."""
from fractions import Fraction

import numpy as np

U = 2.0 ** -24


def _qexpert8(ora, syn, cfg, layer, e, shared=False):
    mats = []
    for m in (syn.GATE, syn.UP, syn.DOWN):
        mats.extend(ora.quantize_rows_int8(syn.expert_matrix(cfg, layer, e, m, shared)))
    return ora.QExpert(*mats, bits=8)


def test_int8_rows_closed_form(ora):
    rng = np.random.default_rng(0)
    for c in (2.0 ** -7, 2.0 ** -3, 1.0, 4.0):
        k = rng.integers(-127, 128, size=(5, 96)).astype(np.float32)
        k[:, 7] = 127 * np.sign(rng.standard_normal(5)).astype(np.float32)  # max |k| = 127 in every row
        q, s = ora.quantize_rows_int8(k * np.float32(c))
        assert np.all(s == np.float32(c))
        assert np.array_equal(q.astype(np.int32), k.astype(np.int32))


def test_int8_rows_ties_round_to_even(ora):
    c = 2.0 ** -4
    row = np.zeros((1, 32), np.float32)
    vals = [127, 2.5, 3.5, -0.5, -1.5, 0.5, 126.5, -126.5]
    row[0, :len(vals)] = np.array(vals, np.float32) * np.float32(c)
    q, s = ora.quantize_rows_int8(row)
    assert s[0] == np.float32(c)
    for got, v in zip(q[0], vals):
        f = Fraction(v)
        n, r = divmod(f, 1)
        want = int(n) + (1 if r > Fraction(1, 2) or (r == Fraction(1, 2) and int(n) % 2 == 1) else 0)
        assert got == max(-127, min(127, want)), (v, got, want)


def test_int8_rows_zero_row_and_error_bound(ora, syn):
    w = syn.normal(64 * 256, 0, 0, 901, 0.01).reshape(64, 256)
    w[3] = 0.0
    q, s = ora.quantize_rows_int8(w)
    assert s[3] == 0.0 and not q[3].any()
    deq = q.astype(np.float64) * s[:, None].astype(np.float64)
    err = np.abs(deq - w.astype(np.float64))
    assert np.all(err <= 0.5 * s[:, None].astype(np.float64) * (1 + 2 ** -20))
    big = np.abs(w).argmax(axis=1)
    nz = s != 0
    assert np.all(np.abs(q[np.arange(64), big])[nz] == 127)


def test_int8_block_isums_brute_force(ora, syn):
    rng = np.random.default_rng(5)
    for _ in range(4):
        w = rng.integers(-127, 128, 256).astype(np.int8)
        x = rng.integers(-127, 128, 256).astype(np.int8)
        got = ora.block_isums_int8(w, x)
        want = (w.astype(np.int64) * x.astype(np.int64)).reshape(-1, 32).sum(axis=1)
        assert np.array_equal(got.astype(np.int64), want)
    w = np.full(32, -127, np.int8)
    assert ora.block_isums_int8(w, w)[0] == 32 * 127 * 127


def test_int8_expert_against_double(ora, syn):
    cfg = syn.config("tiny")
    ex = _qexpert8(ora, syn, cfg, 0, 3)
    x = syn.tokens(cfg)
    xq, xd = ora.quantize_act_q8(x)
    deq = lambda q, s: q.astype(np.float64) * s[:, None].astype(np.float64)
    Wg, Wu, Wd = deq(ex.gate_q, ex.gate_s), deq(ex.up_q, ex.up_s), deq(ex.down_q, ex.down_s)
    for t in range(x.shape[0]):
        y, hq, hd = ora.expert_ffn_token(ex, xq[t], xd[t])
        xdq = xq[t].astype(np.float64) * np.repeat(xd[t].astype(np.float64), 32)
        g, u = Wg @ xdq, Wu @ xdq
        h = g / (1.0 + np.exp(-g)) * u
        hdq = hq.astype(np.float64) * np.repeat(hd.astype(np.float64), 32)
        assert np.all(np.abs(hdq - h) <= 0.5 * np.repeat(hd.astype(np.float64), 32) + 1e-4 * np.abs(h).max())
        y_ref = Wd @ hdq
        mag = np.abs(Wd) @ np.abs(hdq)
        assert np.all(np.abs(y - y_ref) <= (cfg["inter"] // 32 + 2) * U * mag * 1.01 + 1e-30)


def _int4_as_int8(ora, ex4):
    """The int8 expert holding exactly the int4 expert's values and scales."""
    un = lambda q: ora.unpack_int4(q.ravel()).reshape(q.shape[0], q.shape[1] * 2)
    return ora.QExpert(un(ex4.gate_q), ex4.gate_s, un(ex4.up_q), ex4.up_s, un(ex4.down_q), ex4.down_s, bits=8)


def test_int8_expert_with_int4_values_equals_int4_expert(ora, syn):
    from tests.helpers import oracle_expert
    cfg = syn.config("tiny")
    ex4 = oracle_expert(cfg, 0, 2)
    ex8 = _int4_as_int8(ora, ex4)
    xq, xd = ora.quantize_act_q8(syn.tokens(cfg))
    assert np.array_equal(ora.expert_ffn(ex4, xq, xd).view(np.uint32), ora.expert_ffn(ex8, xq, xd).view(np.uint32))


def test_int8_layer_with_int4_values_equals_int4_layer(ora, syn):
    from tests.helpers import oracle_expert
    cfg = syn.config("tiny")
    W, b = syn.router_w(cfg), syn.bias(cfg)
    e4 = {e: oracle_expert(cfg, 0, e) for e in range(cfg["n_experts"])}
    s4 = [oracle_expert(cfg, 0, 0, shared=True)]
    e8 = {e: _int4_as_int8(ora, v) for e, v in e4.items()}
    s8 = [_int4_as_int8(ora, v) for v in s4]
    x = syn.tokens(cfg)
    o4, i4, w4 = ora.moe_layer(cfg, W, b, e4, s4, x)
    o8, i8, w8 = ora.moe_layer(cfg, W, b, e8, s8, x)
    assert np.array_equal(i4, i8) and np.array_equal(w4, w8)
    assert np.array_equal(o4.view(np.uint32), o8.view(np.uint32))
