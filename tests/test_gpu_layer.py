"""GPU parity of the whole MoE layer (coli_moe_layer_forward) and of the
pre-norm stack against the oracle.

The bar: selected experts identical, and max |out - oracle| <= 2e-3 *
RMS(oracle out).  The kernels follow the oracle's evaluation contracts, so
the output is also checked bit for bit (a separate assertion, so that a
tolerance-only regression is reported as such).  Large batches are checked
on a seeded sample of tokens: tokens are independent in a MoE layer, so the
oracle's rows for the sample are exactly the full batch's rows."""
import numpy as np
import pytest

from tests.helpers import assert_layer_close, bits_equal, oracle_layer_forward

pytestmark = pytest.mark.gpu

_layers = {}


def _np(t):
    return t.detach().cpu().numpy()


def _dev_layer(cfg, layer=0):
    from synth.layers import device_layer
    key = (cfg["hidden"], cfg["inter"], cfg["n_experts"], cfg["top_k"], cfg["n_shared"], layer, cfg["seed"],
           cfg["norm_topk_prob"], cfg["routed_scaling_factor"], cfg.get("bias_boost_n", 0),
           cfg["sigma_expert"], cfg["sigma_router"], cfg["bias_lo"], cfg["bias_hi"], cfg.get("weight_bits", 4))
    if key not in _layers:
        if len(_layers) > 3:
            _layers.clear()
        _layers[key] = device_layer(cfg, layer)
    return _layers[key]


def _check_layer(coli, syn, cfg, n_tok, sample=None, exact=True, tokens=None):
    """sample: a seeded random subset of that many tokens; tokens: these."""
    import torch
    L = _dev_layer(cfg)
    x = syn.tokens(cfg, n_tok)
    out = _np(coli.moe_layer_forward(L, torch.from_numpy(x).cuda()))
    if tokens is not None:
        sub = np.asarray(sorted(set(int(t) for t in tokens)))
    elif sample is None:
        sub = np.arange(n_tok)
    else:
        sub = np.sort(np.random.default_rng(1).choice(n_tok, sample, replace=False))
    want, idx, w, _ = oracle_layer_forward(cfg, x[sub])
    _, gidx, gw = coli.moe_route(L, torch.from_numpy(x[sub]).cuda())
    assert np.array_equal(_np(gidx), idx)
    assert_layer_close(out[sub], want)
    if exact:
        assert bits_equal(out[sub], want)
    return out


@pytest.mark.parametrize("n_tok", [8, 1, 2, 3, 5, 13, 16])
def test_layer_tiny(coli, syn, n_tok):
    """Decode path (<= 16 tokens)."""
    _check_layer(coli, syn, syn.config("tiny"), n_tok)


@pytest.mark.parametrize("n_tok", [17, 64, 65, 130, 300, 1000])
def test_layer_tiny_prefill_path(coli, syn, n_tok):
    """Tensor-core path (> 16 tokens): ragged tiles of <= 128 tokens, several
    tiles per expert (1000 tokens: ~250 per routed expert, 8 tiles of the
    shared expert), tiles with a single valid token and with partly filled
    lane quadrants."""
    _check_layer(coli, syn, syn.config("tiny"), n_tok)


@pytest.mark.parametrize("over", [dict(top_k=1), dict(n_shared=0), dict(n_shared=2), dict(norm_topk_prob=False)])
def test_layer_tiny_prefill_variants(coli, syn, over):
    _check_layer(coli, syn, syn.config("tiny", **over), 200)


@pytest.mark.parametrize("n_tok", [1, 5, 16, 40])
def test_layer_inter_not_multiple_of_128(coli, syn, n_tok):
    """Expert inter 96 (not a multiple of 128): neither the decode streaming
    kernels nor the tensor-core kernels take it, so the general expert
    kernels run at layer level, for decode and for prefill batch sizes."""
    _check_layer(coli, syn, syn.config("tiny", inter=96, shared_inter=96), n_tok)


@pytest.mark.parametrize("over", [dict(norm_topk_prob=False), dict(routed_scaling_factor=1.0),
                                  dict(top_k=1), dict(top_k=16), dict(n_shared=0), dict(n_shared=2)])
def test_layer_tiny_variants(coli, syn, over):
    _check_layer(coli, syn, syn.config("tiny", **over), 8)


def test_layer_decode1(coli, syn):
    _check_layer(coli, syn, syn.config("decode1"), 1)


def test_layer_decode4(coli, syn):
    _check_layer(coli, syn, syn.config("decode4"), 4)


def test_layer_decode16(coli, syn):
    """All 16 tokens of the verify batch."""
    _check_layer(coli, syn, syn.config("decode16"), 16)


def _tile_edge_tokens(coli, syn, cfg, n_tok, tile=128):
    """Tokens chosen where tiled kernels go wrong first, from the routing of
    the whole batch: the last token of every tile (and the last token) of
    the two most loaded experts, the first and last token of the shared
    expert's last tile, every token of up to four one-token experts, and the
    first token of the batch."""
    import torch
    L = _dev_layer(cfg)
    x = syn.tokens(cfg, n_tok)
    _, idx, _ = coli.moe_route(L, torch.from_numpy(x).cuda(), with_scores=False)
    idx = _np(idx)
    counts = np.bincount(idx.ravel(), minlength=cfg["n_experts"])
    chosen = {0, n_tok - 1, (n_tok - 1) // tile * tile}
    for e in np.argsort(-counts, kind="stable")[:2]:
        toks = np.flatnonzero((idx == e).any(axis=1))  # the expert's tokens in slot order (ascending)
        chosen.update(int(toks[i]) for i in range(tile - 1, len(toks), tile))
        chosen.add(int(toks[-1]))
    ones = np.flatnonzero(counts == 1)[:4]
    for e in ones:
        chosen.add(int(np.flatnonzero((idx == e).any(axis=1))[0]))
    return sorted(chosen), int(counts.max()), len(ones)


def test_layer_prefill2048_tile_edges(coli, syn):
    """GLM shape, 2048 tokens with the skewed bias: >= 16 tokens picked at
    tile edges of the heaviest experts (each ~700 tokens = 6 tiles), in the
    shared expert's last tile and in one-token experts, plus a random
    sample, all compared with the oracle bit for bit."""
    cfg = syn.config("prefill2048")
    edge, cmax, n_ones = _tile_edge_tokens(coli, syn, cfg, 2048)
    assert cmax > 2 * 128 and n_ones >= 1
    chosen = set(edge)
    for t in np.random.default_rng(7).permutation(2048):  # plus random tokens, up to 36 in all
        if len(chosen) >= 36:
            break
        chosen.add(int(t))
    chosen = sorted(chosen)
    assert len(chosen) >= 32 and len(edge) >= 12
    _check_layer(coli, syn, cfg, 2048, tokens=chosen)


def test_layer_prefill_glm_ragged(coli, syn):
    """GLM shape, 100 tokens: every expert gets a partial tile."""
    _check_layer(coli, syn, syn.config("prefill2048"), 100, sample=3)


def test_layer_zero_tokens_is_noop(coli, syn):
    import torch
    L = _dev_layer(syn.config("tiny"))
    x = torch.empty(0, 256, device="cuda")
    out = coli.moe_layer_forward(L, x)
    assert out.shape == (0, 256)


def test_layer_token_subset_consistency(coli, syn):
    """Rows of a batch equal the same tokens run alone (batched MoE only
    changes how often weights are read, never the result)."""
    import torch
    cfg = syn.config("tiny")
    L = _dev_layer(cfg)
    x = torch.from_numpy(syn.tokens(cfg, 13)).cuda()
    full = _np(coli.moe_layer_forward(L, x))
    for t in (0, 6, 12):
        one = _np(coli.moe_layer_forward(L, x[t:t + 1].contiguous()))
        assert bits_equal(one[0], full[t])


@pytest.mark.parametrize("name,n_tok", [("decode1", 1), ("decode4", 4), ("tiny", 16), ("tiny", 40)])
def test_workspace_contents_do_not_matter(coli, syn, name, n_tok):
    """Repeated forwards on workspaces first memset to 0x00, 0x5A or 0xFF give
    the same bits: no kernel reads scratch before the forward writes it, and
    no kernel launched early (programmatic dependent launch) reads a
    predecessor's output before that output is complete."""
    import torch
    cfg = syn.config(name)
    L = _dev_layer(cfg)
    x = torch.from_numpy(syn.tokens(cfg, n_tok)).cuda()
    ref = _np(coli.moe_layer_forward(L, x))
    for it in range(24):
        ws = coli.make_workspace(L.cfg, n_tok)
        ws.fill_((0x00, 0x5A, 0xFF)[it % 3])
        got = _np(coli.moe_layer_forward(L, x, workspace=ws))
        assert bits_equal(got, ref), f"iteration {it}"


def test_layer_guard_bytes_untouched(coli, syn):
    """Canary words after the output and around the workspace stay intact."""
    import torch
    cfg = syn.config("tiny")
    L = _dev_layer(cfg)
    T, H = 5, cfg["hidden"]
    x = torch.from_numpy(syn.tokens(cfg, T)).cuda()
    buf = torch.full((T * H + 64,), 12345.0, device="cuda")
    out = buf[:T * H].view(T, H)
    nws = coli.workspace_bytes(L.cfg, T)
    wbuf = torch.full((nws + 4096,), 0x5A, dtype=torch.uint8, device="cuda")
    coli.moe_layer_forward(L, x, out=out, workspace=wbuf[:nws])
    torch.cuda.synchronize()
    assert torch.all(buf[T * H:] == 12345.0)
    assert torch.all(wbuf[nws:] == 0x5A)


def test_stack8_teacher_forced_and_free(coli, ora, syn):
    """Each layer of the 8-layer stack (GPU) on the oracle's input for that
    layer: bit-exact indices and output.  Then the free-running stack."""
    import torch
    from synth.layers import device_layer
    cfg = syn.config("stack8")
    layers = [device_layer(cfg, l) for l in range(8)]
    x = syn.tokens(cfg, 1)
    xo = x.copy()
    for l in range(8):
        xn = ora.rmsnorm(xo, cfg["rms_eps"])
        gxn = _np(coli.rmsnorm(torch.from_numpy(xo).cuda(), cfg["rms_eps"]))
        assert bits_equal(gxn, xn)
        m, idx, _, _ = oracle_layer_forward(cfg, xn, l)
        gm = _np(coli.moe_layer_forward(layers[l], torch.from_numpy(xn).cuda()))
        assert_layer_close(gm, m)
        assert bits_equal(gm, m)
        xo = ora.residual_add(xo, m)
    free = _np(coli.moe_stack_forward(layers, torch.from_numpy(x).cuda(), cfg["rms_eps"]))
    assert_layer_close(free, xo)
    assert bits_equal(free, xo)
    del layers
    torch.cuda.empty_cache()


def test_stack8_prefill512_sampled_tokens(coli, syn):
    """The 8-layer stack on 512 tokens (the tensor-core path in every
    layer), free-running on the GPU; the oracle runs 6 of the tokens through
    the same 8 layers on its own.  Tokens are independent through the whole
    stack, so those rows must match bit for bit."""
    import torch
    from synth.layers import device_layer
    from tests.helpers import oracle_stack_forward
    cfg = syn.config("stack8_512")
    layers = [device_layer(cfg, l) for l in range(8)]
    x = syn.tokens(cfg, 512)
    out = _np(coli.moe_stack_forward(layers, torch.from_numpy(x).cuda(), cfg["rms_eps"]))
    del layers
    torch.cuda.empty_cache()
    sub = np.array([0, 137, 255, 256, 400, 511])
    want = oracle_stack_forward(cfg, x[sub], 8)
    assert_layer_close(out[sub], want)
    assert bits_equal(out[sub], want)


def test_invalid_arguments_return_einval(coli, syn):
    import torch
    cfg = syn.config("tiny")
    L = _dev_layer(cfg)
    x = torch.from_numpy(syn.tokens(cfg, 2)).cuda()
    ws = coli.make_workspace(L.cfg, 2)
    with pytest.raises(coli.ColiError) as ei:
        coli.moe_layer_forward(L, x, workspace=ws[:100])
    assert ei.value.status == coli.COLI_ENOMEM
    with pytest.raises(coli.ColiError) as ei:
        coli.moe_layer_forward(L, x, out=x)
    assert ei.value.status == coli.COLI_EINVAL
    with pytest.raises(coli.ColiError) as ei:
        coli.quantize_act_q8(x[:, :40].contiguous())
    assert ei.value.status == coli.COLI_EINVAL
