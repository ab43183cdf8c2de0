"""GPU parity of the individual steps against the oracle, through the C ABI.

Bit-exact: the device generator vs the host generator, int4 packed bytes and
scales, Q8_0 bytes and scales, per-block int32 partial sums, router scores,
selected expert indices and weights, bucketing.  The expert FFN output is
checked bit-exact too (the kernels follow the oracle's fold contract) and,
separately, against the layer tolerance."""
import numpy as np
import pytest

from tests.helpers import assert_layer_close, bits_equal, oracle_expert

pytestmark = pytest.mark.gpu


def _np(t):
    return t.detach().cpu().numpy()


# --------------------------------------------------------------------------
# generator

def test_device_generator_matches_host(coli, syn):
    import torch
    syn.build()
    for n, i0, sigma in [(1000, 0, 1.0), (4097, 123456789, 0.01), (33, 7, 0.006)]:
        d = torch.empty(n, dtype=torch.float32, device="cuda")
        syn.dev_normal(d, 0, 3, 17, sigma, i0=i0)
        assert bits_equal(_np(d), syn.normal(n, 0, 3, 17, sigma, i0=i0))
        syn.dev_uniform(d, 5, 1, 2, -0.05, 0.05, i0=i0)
        assert bits_equal(_np(d), syn.uniform(n, 5, 1, 2, -0.05, 0.05, i0=i0))
    for name in ["tiny", "decode4", "prefill2048"]:
        cfg = syn.config(name)
        assert bits_equal(_np(syn.dev_bias(cfg)), syn.bias(cfg))
        assert bits_equal(_np(syn.dev_tokens(cfg, 4)), syn.tokens(cfg, 4))
        assert bits_equal(_np(syn.dev_router_w(cfg)), syn.router_w(cfg))


# --------------------------------------------------------------------------
# quantisers

@pytest.mark.parametrize("rows,cols", [(1, 32), (37, 96), (128, 256), (256, 128), (64, 6144), (96, 2048)])
def test_quantize_rows_int4_bit_exact(coli, ora, syn, rows, cols):
    import torch
    w = syn.normal(rows * cols, 0, 0, 500 + rows, 0.01).reshape(rows, cols)
    w[0, :] = 0.0  # an all-zero row
    if rows > 2:
        w[1, :5] = np.array([7, 3.5, -2.5, 0.5, -0.5], np.float32) * np.float32(2 ** -4)  # half-way cases
        w[1, 5:] = 0.0
    q, s = coli.quantize_rows_int4(torch.from_numpy(w).cuda())
    qo, so = ora.quantize_rows_int4(w)
    assert bits_equal(_np(q), qo)
    assert bits_equal(_np(s), so)


def test_quantize_rows_int4_glm_expert_sampled_rows(coli, ora, syn):
    import torch
    cfg = syn.config("decode1")
    w = torch.empty(2048, 6144, dtype=torch.float32, device="cuda")
    syn.dev_expert_matrix(w, cfg, 0, 11, syn.GATE)
    q, s = coli.quantize_rows_int4(w)
    rows = np.array([0, 1, 777, 2047])
    wr = syn.expert_rows(cfg, 0, 11, syn.GATE, rows)
    qo, so = ora.quantize_rows_int4(wr)
    assert bits_equal(_np(q)[rows], qo)
    assert bits_equal(_np(s)[rows], so)


@pytest.mark.parametrize("n,dim", [(1, 6144), (4, 6144), (3, 256), (7, 2048), (2048, 6144)])
def test_quantize_act_q8_bit_exact(coli, ora, syn, n, dim):
    import torch
    x = syn.normal(n * dim, 0, 0, 600 + n, 1.0).reshape(n, dim)
    x[0, :32] = 0.0  # a zero block
    x[0, 32:64] = 0.37  # a constant block
    q, d = coli.quantize_act_q8(torch.from_numpy(x).cuda())
    qo, do = ora.quantize_act_q8(x)
    assert bits_equal(_np(q), qo)
    assert bits_equal(_np(d), do)


def test_quantize_act_q8_quotients_near_half_integers(coli, ora):
    """Blocks whose elements sit a few ulps either side of (k + 1/2) d, so
    that the integer codes hang on the last bit of each quotient v / d; the
    scales span 2^-90 .. 2^90 (the quotient from one reciprocal per block is
    exact there) plus subnormal-range blocks (plain division)."""
    import torch
    rng = np.random.default_rng(0x51)
    blocks = []
    for b in range(4096):
        e = int(rng.integers(-90, 91)) if b % 8 else int(rng.integers(-140, -120))
        amax = np.float32(np.ldexp(1.0 + rng.random(), e))
        d = np.float32(amax / np.float32(127.0))
        k = rng.integers(-127, 127, size=31).astype(np.float32) + np.float32(0.5)
        v = (k * d).astype(np.float32)
        v = (v.view(np.int32) + rng.integers(-3, 4, size=31).astype(np.int32)).view(np.float32)
        v = np.clip(v, -amax, amax).astype(np.float32)
        blocks.append(np.concatenate([[amax], v]).astype(np.float32))
    x = np.stack(blocks).reshape(64, -1).astype(np.float32)
    q, d = coli.quantize_act_q8(torch.from_numpy(x).cuda())
    qo, do = ora.quantize_act_q8(x)
    assert bits_equal(_np(d), do)
    assert bits_equal(_np(q), qo)


# --------------------------------------------------------------------------
# integer partial sums

@pytest.mark.parametrize("name", ["tiny", "decode1"])
def test_block_partials_bit_exact(coli, ora, syn, name):
    import torch
    from synth.layers import device_layer
    cfg = syn.config(name, n_experts=2)
    L = device_layer(cfg, 0)
    ex_o = oracle_expert(cfg, 0, 1)
    H, I = cfg["hidden"], cfg["inter"]
    x = syn.normal(3 * H, 0, 0, 700, 1.0).reshape(3, H)
    xq, _ = ora.quantize_act_q8(x)
    h = syn.normal(3 * I, 0, 0, 701, 1.0).reshape(3, I)
    hq, _ = ora.quantize_act_q8(h)
    for which, act, rows, qmat in [(0, xq, I, ex_o.gate_q), (1, xq, I, ex_o.up_q), (2, hq, H, ex_o.down_q)]:
        got = _np(coli.debug_block_partials(L.experts[1], which, torch.from_numpy(act).cuda(), rows))
        for t in range(3):
            for r in ([0, 1, rows // 2, rows - 1] if rows > 64 else range(rows)):
                assert np.array_equal(got[t, r], ora.block_isums(qmat[r], act[t])), (which, t, r)


# --------------------------------------------------------------------------
# router

@pytest.mark.parametrize("name,n_tok", [("tiny", 8), ("tiny", 1), ("tiny", 5), ("decode1", 1), ("decode4", 4),
                                        ("decode16", 16), ("prefill2048", 2048)])
def test_route_bit_exact(coli, ora, syn, name, n_tok):
    import torch
    cfg = syn.config(name)
    ccfg = coli.make_config(cfg["hidden"], cfg["inter"], cfg["n_experts"], cfg["top_k"], cfg["n_shared"],
                            cfg["shared_inter"], cfg["norm_topk_prob"], cfg["routed_scaling_factor"])
    L = coli.MoeLayer(ccfg, syn.dev_router_w(cfg), syn.dev_bias(cfg), [], [])
    x = syn.tokens(cfg, n_tok)
    scores, idx, w = coli.moe_route(L, torch.from_numpy(x).cuda())
    sub = np.arange(n_tok) if n_tok <= 16 else np.random.default_rng(0).choice(n_tok, 48, replace=False)
    so, io, wo = ora.route(x[sub], syn.router_w(cfg), syn.bias(cfg), cfg["top_k"], cfg["norm_topk_prob"],
                           cfg["routed_scaling_factor"])
    assert bits_equal(_np(scores)[sub], so)
    assert np.array_equal(_np(idx)[sub], io)
    assert bits_equal(_np(w)[sub], wo)


@pytest.mark.parametrize("name,n_tok", [("tiny", 8), ("decode16", 16), ("prefill2048", 300)])
def test_route_without_scores_buffer(coli, ora, syn, name, n_tok):
    """coli_moe_route with scores = NULL (scores kept on chip): the same
    expert indices and weights, bit for bit, as the oracle."""
    import torch
    cfg = syn.config(name)
    ccfg = coli.make_config(cfg["hidden"], cfg["inter"], cfg["n_experts"], cfg["top_k"], cfg["n_shared"],
                            cfg["shared_inter"], cfg["norm_topk_prob"], cfg["routed_scaling_factor"])
    L = coli.MoeLayer(ccfg, syn.dev_router_w(cfg), syn.dev_bias(cfg), [], [])
    x = syn.tokens(cfg, n_tok)
    scores, idx, w = coli.moe_route(L, torch.from_numpy(x).cuda(), with_scores=False)
    assert scores is None
    sub = np.arange(n_tok) if n_tok <= 16 else np.random.default_rng(2).choice(n_tok, 24, replace=False)
    _, io, wo = ora.route(x[sub], syn.router_w(cfg), syn.bias(cfg), cfg["top_k"], cfg["norm_topk_prob"],
                          cfg["routed_scaling_factor"])
    assert np.array_equal(_np(idx)[sub], io)
    assert bits_equal(_np(w)[sub], wo)


def test_route_ties_and_k_equals_e(coli, ora):
    import torch
    E, H = 16, 128
    for K in (4, 16):
        ccfg = coli.make_config(H, 32, E, K, 0, 32, True, 2.5)
        W = np.zeros((E, H), np.float32)
        bias = np.zeros(E, np.float32)
        bias[[3, 9, 12]] = 0.25
        bias[[5, 14]] = 0.125
        x = np.ones((3, H), np.float32)
        L = coli.MoeLayer(ccfg, torch.from_numpy(W).cuda(), torch.from_numpy(bias).cuda(), [], [])
        s, idx, w = coli.moe_route(L, torch.from_numpy(x).cuda())
        so, io, wo = ora.route(x, W, bias, K, True, 2.5)
        assert np.array_equal(_np(idx), io) and bits_equal(_np(w), wo)
        _, idx2, w2 = coli.moe_route(L, torch.from_numpy(x).cuda(), with_scores=False)
        assert np.array_equal(_np(idx2), io) and bits_equal(_np(w2), wo)


# --------------------------------------------------------------------------
# bucketing

@pytest.mark.parametrize("T,K,E", [(1, 8, 256), (4, 8, 256), (16, 8, 256), (8, 4, 16), (2048, 8, 256),
                                   (2500, 8, 256), (3, 16, 512), (0, 8, 256)])
def test_bucket_bit_exact(coli, ora, T, K, E):
    import torch
    rng = np.random.default_rng(T + K + E)
    idx = np.array([rng.permutation(E)[:K] for _ in range(T)], dtype=np.int32).reshape(T, K)
    if T > 100:  # skew like the prefill workload
        idx[: T // 2, :4] = np.stack([rng.permutation(32)[:4] for _ in range(T // 2)])
        for t in range(T // 2):
            rest = [e for e in rng.permutation(E) if e not in idx[t, :4]][:K - 4]
            idx[t, 4:] = rest
    counts, offsets, perm = coli.moe_bucket(torch.from_numpy(idx).cuda(), E)
    co, oo, po = ora.bucket(idx, E)
    assert np.array_equal(_np(counts), co)
    assert np.array_equal(_np(offsets), oo)
    assert np.array_equal(_np(perm), po)


# --------------------------------------------------------------------------
# one expert

@pytest.mark.parametrize("name,n_tok", [("tiny", 1), ("tiny", 3), ("tiny", 8), ("decode1", 1), ("decode1", 2),
                                        ("decode1", 5)])
def test_expert_ffn(coli, ora, syn, name, n_tok):
    import torch
    from synth.layers import device_layer
    cfg = syn.config(name, n_experts=1, top_k=1)
    L = device_layer(cfg, 0)
    x = syn.tokens(cfg, n_tok)
    xq, xd = ora.quantize_act_q8(x)
    y = _np(coli.moe_expert_ffn(L.cfg, L.experts[0], torch.from_numpy(xq).cuda(), torch.from_numpy(xd).cuda()))
    yo = ora.expert_ffn(oracle_expert(cfg, 0, 0), xq, xd)
    assert_layer_close(y, yo)
    assert bits_equal(y, yo)


@pytest.mark.parametrize("rows,cols,block", [(1, 32, 128), (130, 256, 128), (6144, 2048, 128), (257, 160, 64),
                                             (40, 96, 8)])
def test_requantize_fp8_int4_bit_exact(coli, ora, syn, rows, cols, block):
    """The FP8 -> int4 converter step: packed bytes and row scales equal the
    oracle's bit for bit (ragged tiles, NaN codes and a GLM down-matrix
    shape included)."""
    import torch
    codes, factors = syn.fp8_blocks(rows, cols, block, seed=7 * rows + cols)
    q, s = coli.requantize_fp8_int4(torch.from_numpy(codes).cuda(), torch.from_numpy(factors).cuda(), block)
    q_ref, s_ref = ora.requantize_fp8_int4(codes, factors, block)
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
