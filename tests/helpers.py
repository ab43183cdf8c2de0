"""Shared test helpers: oracle-side layers built lazily from the host
generator (only the experts a routing needs), and comparison utilities."""
from __future__ import annotations

import numpy as np

import oracle
import synth

_qcache: dict = {}


def oracle_expert(cfg: dict, layer: int, e: int, shared: bool = False) -> oracle.QExpert:
    bits = cfg.get("weight_bits", 4)
    key = (cfg["name"], cfg["seed"], cfg["hidden"], cfg["inter"], layer, e, shared, bits, cfg["sigma_expert"])
    if key not in _qcache:
        quant = oracle.quantize_rows_int4 if bits == 4 else oracle.quantize_rows_int8
        mats = []
        for m in (synth.GATE, synth.UP, synth.DOWN):
            mats.extend(quant(synth.expert_matrix(cfg, layer, e, m, shared)))
        _qcache[key] = oracle.QExpert(*mats, bits=bits)
    return _qcache[key]


def oracle_layer_forward(cfg: dict, x: np.ndarray, layer: int = 0):
    """Oracle forward of layer `layer` on tokens x; returns (out, idx, w, scores)."""
    W, b = synth.router_w(cfg, layer), synth.bias(cfg, layer)
    scores, idx, _ = oracle.route(x, W, b, cfg["top_k"], cfg["norm_topk_prob"], cfg["routed_scaling_factor"])
    experts = {int(e): oracle_expert(cfg, layer, int(e)) for e in np.unique(idx)}
    shared = [oracle_expert(cfg, layer, s, shared=True) for s in range(cfg["n_shared"])]
    out, idx2, w = oracle.moe_layer(cfg, W, b, experts, shared, x)
    assert np.array_equal(idx, idx2)
    return out, idx, w, scores


def oracle_stack_forward(cfg: dict, x: np.ndarray, n_layers: int, expert_fn=None) -> np.ndarray:
    """The pre-norm stack by the oracle: for l = 0..n_layers-1,
    x <- x + MoE_l(RMSNorm(x)) (layer l's seeded weights).  expert_fn(layer,
    e, shared) may supply the experts instead of the generator."""
    eps = cfg.get("rms_eps", 1e-5)
    xo = np.ascontiguousarray(x, np.float32)
    for l in range(n_layers):
        xn = oracle.rmsnorm(xo, eps)
        if expert_fn is None:
            m, _, _, _ = oracle_layer_forward(cfg, xn, l)
        else:
            W, b = synth.router_w(cfg, l), synth.bias(cfg, l)
            experts = {e: expert_fn(l, e, False) for e in range(cfg["n_experts"])}
            shared = [expert_fn(l, s, True) for s in range(cfg["n_shared"])]
            m, _, _ = oracle.moe_layer(cfg, W, b, experts, shared, xn)
        xo = oracle.residual_add(xo, m)
    return xo


def rms(a) -> float:
    a = np.asarray(a, np.float64)
    return float(np.sqrt((a * a).mean()))


def assert_layer_close(got: np.ndarray, want: np.ndarray, rel: float = 2e-3):
    """The layer-output bar: max |got - want| <= rel * RMS(want)."""
    err = float(np.abs(got.astype(np.float64) - want.astype(np.float64)).max())
    bound = rel * rms(want)
    assert err <= bound, f"max abs err {err:.3e} > {rel} * RMS = {bound:.3e}"
    return err


def bits_equal(a: np.ndarray, b: np.ndarray) -> bool:
    a = np.ascontiguousarray(a)
    b = np.ascontiguousarray(b)
    return a.shape == b.shape and a.dtype == b.dtype and np.array_equal(a.view(np.uint8), b.view(np.uint8))
