"""The streaming decode path (prepared layers, batches of 1..4 tokens):
the layout that coli_moe_prepare writes, and the layer output of the
streaming kernel against the oracle, bit for bit, through the C ABI."""
import numpy as np
import pytest

from tests.helpers import assert_layer_close, bits_equal, oracle_layer_forward

pytestmark = pytest.mark.gpu

_cache = {}


def _np(t):
    return t.detach().cpu().numpy()


def _layer(cfg):
    from synth.layers import device_layer
    key = tuple(sorted((k, v) for k, v in cfg.items() if not isinstance(v, (list, dict))))
    if key not in _cache:
        if len(_cache) > 2:
            _cache.clear()
        _cache[key] = device_layer(cfg, 0, prepare=True)
    return _cache[key]


def _geom(H, I, bits):
    bpb = 16 if bits == 4 else 32
    gmax = 256 // bpb
    nbh, nbi = H // 32, I // 32
    g_gu, g_dn = min(gmax, nbh), min(gmax, nbi)
    lpr = 2 if nbh % gmax == 0 and nbi % (2 * gmax) == 0 else 1  # lanes per down row
    st_gu, st_dn = nbh // g_gu, nbi // (lpr * g_dn)
    stage_gu, stage_dn = 32 * g_gu * bpb, 32 * g_dn * bpb
    gu_bytes = (I // 32) * 2 * st_gu * stage_gu
    dn_bytes = (H // (32 // lpr)) * st_dn * stage_dn
    return bpb, g_gu, g_dn, st_gu, st_dn, stage_gu, stage_dn, gu_bytes, dn_bytes, lpr


def _layout_offset(H, I, m, r, b, bits=4, h=0):
    """Byte offset of 16-byte chunk h of block b of row r of matrix m (0 gate,
    1 up, 2 down) in one expert's streaming copy, as include/coli.h and the
    layout header document it."""
    bpb, g_gu, g_dn, st_gu, st_dn, stage_gu, stage_dn, gu_bytes, _, lpr = _geom(H, I, bits)
    cpb = bpb // 16
    if m < 2:
        swz = min(g_gu * cpb, 8) - 1
        u, half = r // 32, (r // 16) % 2
        sr = (0 if m == 0 else 16) + r % 16
        s, j = divmod(b, g_gu)
        c = j * cpb + h
        return ((u * 2 + half) * st_gu + s) * stage_gu + sr * g_gu * bpb + ((c ^ (sr & swz)) * 16)
    swz = min(g_dn * cpb, 8) - 1
    rpu = 32 // lpr
    v, rr = divmod(r, rpu)
    s, jj = divmod(b, lpr * g_dn)
    piece, j = divmod(jj, g_dn)
    sr = piece * rpu + rr
    c = j * cpb + h
    return gu_bytes + (v * st_dn + s) * stage_dn + sr * g_dn * bpb + ((c ^ (sr & swz)) * 16)


@pytest.mark.parametrize("name", ["tiny", "mid"])
@pytest.mark.parametrize("bits", [4, 8])
def test_prepare_writes_the_documented_layout(coli, syn, name, bits):
    cfg = syn.config(name, weight_bits=bits)
    H, I, E, S = cfg["hidden"], cfg["inter"], cfg["n_experts"], cfg["n_shared"]
    L = _layer(cfg)
    prep = _np(L.prepared)
    eb = len(prep) // (E + S)
    assert eb * (E + S) == len(prep) and eb % 256 == 0
    _, _, _, _, _, _, _, gu_bytes, dn_bytes, lpr = _geom(H, I, bits)
    assert lpr == (2 if name == "mid" else 1)
    bpb = 16 if bits == 4 else 32
    for j, ex in enumerate(L.experts + L.shared):
        base = j * eb
        mats = [_np(ex.gate_q).view(np.uint8), _np(ex.up_q).view(np.uint8), _np(ex.down_q).view(np.uint8)]
        for m, q in enumerate(mats):
            rows, nb = q.shape[0], q.shape[1] // bpb
            r, b = np.meshgrid(np.arange(rows), np.arange(nb), indexing="ij")
            blk = q.reshape(rows, nb, bpb)
            # int4: the block; int8: even elements, then odd elements
            chunks = [blk] if bits == 4 else [blk[:, :, 0::2], blk[:, :, 1::2]]
            for h, want in enumerate(chunks):
                o = base + _layout_offset(H, I, m, r, b, bits, h)
                got = prep[o[:, :, None] + np.arange(16)]
                assert np.array_equal(got, want), (j, m, h)
        sc = prep[base + gu_bytes + dn_bytes:base + gu_bytes + dn_bytes + (2 * I + H) * 4].view(np.float32)
        assert bits_equal(sc[:I], _np(ex.gate_s)) and bits_equal(sc[I:2 * I], _np(ex.up_s))
        assert bits_equal(sc[2 * I:], _np(ex.down_s))


def _check(coli, syn, cfg, n_tok, tokens=None):
    import torch
    L = _layer(cfg)
    x = syn.tokens(cfg, n_tok) if tokens is None else tokens
    xt = torch.from_numpy(x).cuda()
    out = _np(coli.moe_layer_forward(L, xt))
    plain = _np(coli.moe_layer_forward(L, xt, cstruct=L.cstruct(use_prepared=False)))
    want, idx, _, _ = oracle_layer_forward(cfg, x)
    assert_layer_close(out, want)
    assert bits_equal(out, want)
    assert bits_equal(out, plain)
    return out


@pytest.mark.parametrize("n_tok", [1, 2, 3, 4, 5, 6, 7, 8, 12, 16])
def test_stream_tiny(coli, syn, n_tok):
    _check(coli, syn, syn.config("tiny"), n_tok)


@pytest.mark.parametrize("n_tok", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("bits", [4, 8])
def test_stream_mid_lane_pairs(coli, syn, n_tok, bits):
    """Down rows split over lane pairs (rows of whole stages)."""
    _check(coli, syn, syn.config("mid", weight_bits=bits), n_tok)


@pytest.mark.parametrize("over", [dict(norm_topk_prob=False), dict(top_k=1), dict(top_k=16), dict(n_shared=0),
                                  dict(n_shared=2), dict(routed_scaling_factor=1.0)])
def test_stream_tiny_variants(coli, syn, over):
    _check(coli, syn, syn.config("tiny", **over), 4)


def test_stream_all_tokens_on_one_expert(coli, syn):
    """Four identical tokens: every routed slot holds all 4 tokens."""
    cfg = syn.config("tiny")
    x = np.repeat(syn.tokens(cfg, 1), 4, axis=0)
    _check(coli, syn, cfg, 4, tokens=x)


@pytest.mark.parametrize("name,n_tok", [("decode1", 1), ("decode4", 4), ("decode4", 2), ("decode4", 3),
                                        ("decode16", 5), ("decode16", 8), ("decode16", 16)])
def test_stream_glm(coli, syn, name, n_tok):
    _check(coli, syn, syn.config(name), n_tok)


@pytest.mark.parametrize("name,n_tok", [("decode1", 1), ("decode4", 4), ("tiny", 3)])
def test_stream_workspace_contents_do_not_matter(coli, syn, name, n_tok):
    """Workspaces filled with 0x00 / 0x5A / 0xFF (stale counters, stale h)
    before each call give the same bits: the router kernel clears the
    counters and every scratch word is written before it is read."""
    import torch
    cfg = syn.config(name)
    L = _layer(cfg)
    x = torch.from_numpy(syn.tokens(cfg, n_tok)).cuda()
    ref = _np(coli.moe_layer_forward(L, x))
    for it in range(12):
        ws = coli.make_workspace(L.cfg, n_tok)
        ws.fill_((0x00, 0x5A, 0xFF)[it % 3])
        got = _np(coli.moe_layer_forward(L, x, workspace=ws))
        assert bits_equal(got, ref), f"iteration {it}"
        assert coli.sync_status(ws) == coli.COLI_OK


def test_stream_repeated_calls_one_workspace(coli, syn):
    """Back-to-back forwards on one stream and one workspace (the counters
    of one call must not leak into the next)."""
    import torch
    cfg = syn.config("decode4")
    L = _layer(cfg)
    xs = [torch.from_numpy(syn.tokens(cfg, 4)[::-1].copy()).cuda(), torch.from_numpy(syn.tokens(cfg, 4)).cuda()]
    ws = coli.make_workspace(L.cfg, 4)
    refs = [_np(coli.moe_layer_forward(L, x, cstruct=L.cstruct(use_prepared=False))) for x in xs]
    outs = [torch.empty_like(xs[0]) for _ in range(20)]
    for i in range(20):
        coli.moe_layer_forward(L, xs[i % 2], out=outs[i], workspace=ws)
    for i in range(20):
        assert bits_equal(_np(outs[i]), refs[i % 2]), i
