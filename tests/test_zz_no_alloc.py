"""coli_moe_layer_forward_noalloc: the layer forward for callers that cannot
allocate device memory (a host that owns every device allocation and gives a
plugin no allocator, or a serving loop that must not call cudaMalloc after
start-up because it can synchronise the device).  Its scratch is a fixed
8 MiB array inside the library.

Checked through the C ABI against coli_moe_layer_forward (the same layer,
same tokens) within the layer tolerance, on two calls in a row -- the second
call starts from the scratch contents the first one left behind.  The file
name sorts last so that a stop-at-first-failure run has already run every
other test before this one."""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu


def _close(got, want, rel=2e-3):
    want = want.astype(np.float64)
    err = np.abs(got.astype(np.float64) - want).max()
    assert err <= rel * np.sqrt((want ** 2).mean()), err


@pytest.mark.parametrize("name,n_tok,prep", [("tiny", 8, False), ("tiny", 3, False), ("tiny", 40, False),
                                             ("decode1", 1, False), ("decode16", 16, False),
                                             ("decode16", 22, False),  # the tensor-core path, the documented limit
                                             ("decode4", 4, True)])     # the streaming path of a prepared layer
def test_noalloc_matches_workspace_forward_twice(coli, syn, name, n_tok, prep):
    import torch
    from synth.layers import device_layer
    cfg = syn.config(name)
    L = device_layer(cfg, 0, prepare=prep)
    x = torch.from_numpy(syn.tokens(cfg, n_tok)).cuda()
    want = coli.moe_layer_forward(L, x).cpu().numpy()
    for _ in range(2):
        got = coli.moe_layer_forward_noalloc(L, x).cpu().numpy()
        _close(got, want)
        assert np.array_equal(got, want)  # same kernels, same contracts
    # a different token batch right after: no stale state leaks in
    x2 = torch.from_numpy(syn.tokens(cfg, n_tok)[::-1].copy()).cuda()
    _close(coli.moe_layer_forward_noalloc(L, x2).cpu().numpy(), coli.moe_layer_forward(L, x2).cpu().numpy())
    del L
    torch.cuda.empty_cache()


def test_noalloc_rejects_more_than_its_scratch(coli, syn):
    import torch
    from synth.layers import device_layer
    cfg = syn.config("tiny")
    L = device_layer(cfg, 0)
    x = torch.from_numpy(syn.tokens(cfg, 2048)).cuda()
    with pytest.raises(coli.ColiError) as ei:
        coli.moe_layer_forward_noalloc(L, x)
    assert ei.value.status == coli.COLI_EINVAL
    assert "scratch" in str(ei.value)
    # a token count beyond the forward's range is refused before any sizing
    Lc = L.cstruct()
    import ctypes as C
    rc = coli.lib().coli_moe_layer_forward_noalloc(C.byref(Lc), C.c_void_p(x.data_ptr()), (1 << 40),
                                                  C.c_void_p(x.data_ptr()), None)
    assert rc == coli.COLI_EINVAL
