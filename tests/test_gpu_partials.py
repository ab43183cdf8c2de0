"""The per-32-block int32 partial sums of the kernels that run, against the
oracle's (coli_debug_capture_partials: the streaming kernel of a prepared
layer and the tensor-core kernels, the same kernels with every block sum
also stored).  Bit-exact: each captured isum[o][b] equals the oracle's
ora_block_isums of that weight row against the token's Q8 x (gate, up) or
its Q8 h (down), for every routed rank and every shared expert of every
token."""
import numpy as np
import pytest

from tests.helpers import oracle_expert

pytestmark = pytest.mark.gpu


def _np(t):
    return t.detach().cpu().numpy()


def _check_partials(ora, syn, cfg, x, isum, idx, rows_per_matrix=None, seed=0):
    H, I, K, S = cfg["hidden"], cfg["inter"], cfg["top_k"], cfg["n_shared"]
    nbh, nbi = H // 32, I // 32
    xq, xd = ora.quantize_act_q8(x)
    rng = np.random.default_rng(seed)
    bits = cfg.get("weight_bits", 4)
    isums = ora.block_isums if bits == 4 else ora.block_isums_int8
    for t in range(x.shape[0]):
        for j in range(K + S):
            ex = oracle_expert(cfg, 0, int(idx[t, j])) if j < K else oracle_expert(cfg, 0, j - K, shared=True)
            _, hq, _ = ora.expert_ffn_token(ex, xq[t], xd[t])
            got = isum[t, j]
            gate = got[:I * nbh].reshape(I, nbh)
            up = got[I * nbh:2 * I * nbh].reshape(I, nbh)
            down = got[2 * I * nbh:].reshape(H, nbi)
            o_gu = np.arange(I) if rows_per_matrix is None else rng.choice(I, rows_per_matrix, replace=False)
            o_dn = np.arange(H) if rows_per_matrix is None else rng.choice(H, rows_per_matrix, replace=False)
            for o in o_gu:
                assert np.array_equal(gate[o], isums(ex.gate_q[o], xq[t])), (t, j, "gate", o)
                assert np.array_equal(up[o], isums(ex.up_q[o], xq[t])), (t, j, "up", o)
            for o in o_dn:
                assert np.array_equal(down[o], isums(ex.down_q[o], hq)), (t, j, "down", o)


def _run(coli, ora, syn, cfg, n_tok, prepare, rows_per_matrix=None):
    import torch
    from synth.layers import device_layer
    L = device_layer(cfg, 0, prepare=prepare)
    x = syn.tokens(cfg, n_tok)
    xt = torch.from_numpy(x).cuda()
    out, isum = coli.capture_partials(L, xt)
    plain = coli.moe_layer_forward(L, xt)
    assert np.array_equal(_np(out).view(np.uint32), _np(plain).view(np.uint32))  # the capture changes nothing
    _, idx, _ = coli.moe_route(L, xt, with_scores=False)
    _check_partials(ora, syn, cfg, x, _np(isum), _np(idx), rows_per_matrix)


@pytest.mark.parametrize("n_tok", [1, 3, 4, 8, 11])
def test_partials_streaming_kernel_tiny(coli, ora, syn, n_tok):
    _run(coli, ora, syn, syn.config("tiny"), n_tok, prepare=True)


@pytest.mark.parametrize("n_tok", [17, 40])
def test_partials_tensor_cores_tiny(coli, ora, syn, n_tok):
    _run(coli, ora, syn, syn.config("tiny"), n_tok, prepare=False)


@pytest.mark.parametrize("prepare,n_tok", [(True, 4), (False, 20)])
def test_partials_int8_weights_tiny(coli, ora, syn, prepare, n_tok):
    _run(coli, ora, syn, syn.config("tiny", weight_bits=8), n_tok, prepare=prepare)


def test_partials_streaming_kernel_glm_decode1(coli, ora, syn):
    _run(coli, ora, syn, syn.config("decode1"), 1, prepare=True, rows_per_matrix=96)


def test_partials_tensor_cores_glm(coli, ora, syn):
    _run(coli, ora, syn, syn.config("prefill2048"), 24, prepare=False, rows_per_matrix=24)


def test_capture_rejects_other_paths_and_short_buffers(coli, syn):
    import ctypes as C
    import torch
    from synth.layers import device_layer
    cfg = syn.config("tiny")
    L = device_layer(cfg, 0)
    x = torch.from_numpy(syn.tokens(cfg, 2)).cuda()
    buf = torch.zeros(1 << 20, dtype=torch.int32, device="cuda")
    assert coli.lib().coli_debug_capture_partials(C.c_void_p(buf.data_ptr()), buf.numel()) == coli.COLI_OK
    with pytest.raises(coli.ColiError):  # unprepared, 2 tokens: the 16-token decode kernels
        coli.moe_layer_forward(L, x)
    coli.moe_layer_forward(L, x)  # the arming was consumed
    Lp = device_layer(cfg, 0, prepare=True)
    assert coli.lib().coli_debug_capture_partials(C.c_void_p(buf.data_ptr()), 16) == coli.COLI_OK
    with pytest.raises(coli.ColiError) as ei:
        coli.moe_layer_forward(Lp, x)
    assert "words" in str(ei.value)
