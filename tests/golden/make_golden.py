"""Writes tests/golden/tiny_oracle.txt from the CPU oracle only.

Usage: python tests/golden/make_golden.py
Fixture: the tiny correctness workload (16 tokens, hidden 256, intermediate 128,
8 experts, top-2, seed 0), block_m 16: the oracle's routing tensors and the layer's
bf16 output. It pins the oracle against regressions; its values come from the oracle
(no page prints a worked example of this layer).
"""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from w4a16_int4_mixture_align_b200 import inputs  # noqa: E402

BLOCK_M = 16


def main():
    d = inputs.make_inputs(inputs.CONFIGS["tiny"])
    cfg = d["cfg"]
    s, eids, ntp, offs = oracle.moe_align(d["topk_ids"], cfg.E, BLOCK_M)
    out = oracle.moe_forward(d["x"], d["topk_ids"], d["topk_weights"], d["qw13"], d["s13"],
                             d["qw2"], d["s2"])
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_oracle.txt")
    with open(path, "w") as fh:
        fh.write("# tiny workload (T=16 H=256 I=128 E=8 top-2 seed 0), block_m=16; written by make_golden.py from the oracle\n")
        fh.write("num_tokens_padded %d\n" % ntp)
        fh.write("sorted_ids " + " ".join(map(str, s.tolist())) + "\n")
        fh.write("expert_ids " + " ".join(map(str, eids.tolist())) + "\n")
        fh.write("expert_offsets " + " ".join(map(str, offs.tolist())) + "\n")
        for r in range(out.shape[0]):
            fh.write("out %d " % r + " ".join("%04x" % v for v in out[r].tolist()) + "\n")


if __name__ == "__main__":
    main()
