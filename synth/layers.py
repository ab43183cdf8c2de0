"""Synthetic MoE layers resident in HBM, built on the GPU.

F32 weights come from the device generator (``synth_dev.cu``, the same
numbers as the host generator) and are packed to int4 by the library's own
quantiser (``coli_quantize_rows_int4``), one matrix at a time through a
reusable F32 staging buffer (cfg["weight_bits"] 8: int8 rows by
coli_quantize_rows_int8 instead; prepare=True also makes the layer's
streaming copy with coli_moe_prepare).  Each layer's packed weights live in one
allocation: experts e = 0..E-1 then the shared experts, each as
[gate | up | down] blocks of inter*hidden/2 bytes (row-major [out x in]).
"""
from __future__ import annotations

import synth


def device_layer(cfg: dict, layer: int = 0, device="cuda", staging=None, prepare: bool = False):
    import torch

    import int4_weight_only_sigmoid_b200 as coli

    H, I, E, S = cfg["hidden"], cfg["inter"], cfg["n_experts"], cfg["n_shared"]
    bits = cfg.get("weight_bits", 4)
    assert cfg["shared_inter"] == I
    n = E + S
    mat_bytes = I * H * bits // 8
    qbuf = torch.empty(n, 3, mat_bytes, dtype=torch.uint8 if bits == 4 else torch.int8, device=device)
    s_gu = torch.empty(n, 2, I, dtype=torch.float32, device=device)
    s_dn = torch.empty(n, H, dtype=torch.float32, device=device)
    tmp = staging if staging is not None else torch.empty(I * H, dtype=torch.float32, device=device)
    experts = []
    for j in range(n):
        shared = j >= E
        e = j - E if shared else j
        for m in (synth.GATE, synth.UP, synth.DOWN):
            rows, cols = synth.expert_shape(cfg, m, shared)
            w = tmp[:rows * cols].view(rows, cols)
            synth.dev_expert_matrix(w, cfg, layer, e, m, shared)
            q = qbuf[j, m].view(rows, cols * bits // 8)
            s = s_dn[j] if m == synth.DOWN else s_gu[j, m]
            if bits == 4:
                coli.quantize_rows_int4(w, q_out=q, s_out=s)
            else:
                coli.quantize_rows_int8(w, q_out=q, s_out=s)
        experts.append(coli.QExpert(qbuf[j, 0].view(I, H * bits // 8), s_gu[j, 0], qbuf[j, 1].view(I, H * bits // 8),
                                    s_gu[j, 1], qbuf[j, 2].view(H, I * bits // 8), s_dn[j]))
    ccfg = coli.make_config(H, I, E, cfg["top_k"], S, cfg["shared_inter"], cfg["norm_topk_prob"],
                            cfg["routed_scaling_factor"], bits)
    L = coli.MoeLayer(ccfg, synth.dev_router_w(cfg, layer, device), synth.dev_bias(cfg, layer, device),
                      experts[:E], experts[E:])
    L._storage = (qbuf, s_gu, s_dn)
    if prepare:
        coli.prepare(L)
    return L
