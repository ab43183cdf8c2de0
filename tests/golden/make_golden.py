"""Writes tests/golden/tiny_layer.txt: the tiny MoE layer (hidden 256, inter
128, 16 experts, top-4, 1 shared, 8 tokens, seed 0) as computed by the oracle
from the seeded generator.  Calls only ``oracle`` and ``synth``; it records the
oracle's own results so later changes to the oracle cannot pass unnoticed.

Run from the repository root:  python tests/golden/make_golden.py
"""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import synth  # noqa: E402


def qexpert(cfg, layer, e, shared=False):
    mats = []
    for m in (synth.GATE, synth.UP, synth.DOWN):
        mats.extend(oracle.quantize_rows_int4(synth.expert_matrix(cfg, layer, e, m, shared)))
    return oracle.QExpert(*mats)


def main():
    cfg = synth.config("tiny")
    experts = {e: qexpert(cfg, 0, e) for e in range(cfg["n_experts"])}
    shared = [qexpert(cfg, 0, 0, shared=True)]
    x = synth.tokens(cfg)
    out, idx, w = oracle.moe_layer(cfg, synth.router_w(cfg), synth.bias(cfg), experts, shared, x)
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_layer.txt")
    with open(path, "w") as f:
        f.write("# tiny MoE layer (seed 0), oracle output; written by make_golden.py\n")
        f.write("# idx: [8 tokens x top-4] rank order; w_bits / out_bits: binary32 bit patterns\n")
        f.write("idx = " + " ".join(str(v) for v in idx.ravel()) + "\n")
        f.write("w_bits = " + " ".join(f"{v:08x}" for v in w.view(np.uint32).ravel()) + "\n")
        f.write("out_bits = " + " ".join(f"{v:08x}" for v in out.view(np.uint32).ravel()) + "\n")
    print("wrote", path, "rms(out) =", float(np.sqrt((out.astype(np.float64) ** 2).mean())))


if __name__ == "__main__":
    main()
