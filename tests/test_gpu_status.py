"""The device status word and coli_sync_status, on the GPU, without any
fault: a forward clears the word, a bounded wait that nothing completes
(the test probe) records a timeout code that coli_sync_status reports as
COLI_ETIMEOUT, and the next forward clears it again."""
import pytest

pytestmark = pytest.mark.gpu


def _layer(syn):
    from synth.layers import device_layer
    return device_layer(syn.config("tiny"), 0)


@pytest.mark.parametrize("n_tok", [1, 8, 40])  # decode path (router kernel clears) and prefill path (memset)
def test_forward_clears_status(coli, syn, n_tok):
    import torch
    L = _layer(syn)
    ws = coli.make_workspace(L.cfg, n_tok)
    ws.random_(0, 255)  # stale bytes, status word included
    x = torch.from_numpy(syn.tokens(syn.config("tiny"), n_tok)).cuda()
    coli.moe_layer_forward(L, x, workspace=ws)
    assert coli.sync_status(ws) == coli.COLI_OK


def test_wait_probe_reports_timeout_then_forward_clears(coli, syn):
    import torch
    L = _layer(syn)
    ws = coli.make_workspace(L.cfg, 8)
    x = torch.from_numpy(syn.tokens(syn.config("tiny"), 8)).cuda()
    coli.moe_layer_forward(L, x, workspace=ws)
    assert coli.sync_status(ws) == coli.COLI_OK
    coli.debug_wait_probe(ws, 2_000_000)  # ~1 ms of waiting on a barrier nobody arrives at
    assert coli.sync_status(ws) == coli.COLI_ETIMEOUT
    msg = coli.lib().coli_last_error().decode()
    assert "status 30" in msg and "gave up" in msg
    # the GPU context is still usable and the next forward starts the word afresh
    out = coli.moe_layer_forward(L, x, workspace=ws)
    assert coli.sync_status(ws) == coli.COLI_OK
    assert torch.isfinite(out).all()


def test_stack_forward_clears_status(coli, syn):
    import torch
    from synth.layers import device_layer
    cfg = syn.config("tiny")
    layers = [device_layer(cfg, l) for l in range(2)]
    ws = coli.make_workspace(layers[0].cfg, 8)
    coli.debug_wait_probe(ws, 1000)
    assert coli.sync_status(ws) == coli.COLI_ETIMEOUT
    x = torch.from_numpy(syn.tokens(cfg, 8)).cuda()
    coli.moe_stack_forward(layers, x, workspace=ws)
    assert coli.sync_status(ws) == coli.COLI_OK


def test_noalloc_scratch_status(coli, syn):
    import torch
    L = _layer(syn)
    x = torch.from_numpy(syn.tokens(syn.config("tiny"), 4)).cuda()
    coli.moe_layer_forward_noalloc(L, x)
    assert coli.sync_status(None) == coli.COLI_OK
