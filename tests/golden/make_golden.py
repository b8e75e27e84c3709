"""Writes tests/golden/tiny_oracle.txt and tiny_route_ex.txt from the CPU oracle alone.

The source pages print no worked example of the MoE FFN, so the stored values
here are the oracle's own output on the seeded "tiny" workload (T=16, H=256,
I=128, E=8, top-2, seed 0).  They pin the oracle against later unintended
changes; a deliberate change of the oracle's arithmetic regenerates this file
in the same commit and names the passage that justifies it.

Run:  python tests/golden/make_golden.py
"""
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
from mixture_experts_ffn_sort_b200 import workloads  # noqa: E402


def main():
    w = workloads.make_workload("tiny", threads=1)
    o = oracle.workload(w)
    lines = ["# oracle output, workload tiny (T=16 H=256 I=128 E=8 K=2 seed 0)",
             "# written by tests/golden/make_golden.py (calls oracle/ only)"]
    lines.append("ids " + " ".join(map(str, o["ids"].ravel())))
    lines.append("w " + " ".join("%.17g" % v for v in o["w"].ravel()))
    lines.append("offsets " + " ".join(map(str, o["offsets"])))
    lines.append("sorted_route " + " ".join(map(str, o["sorted_route"])))
    for t in range(4):
        lines.append("out%d " % t + " ".join("%.17g" % v for v in o["out"][t, :16]))
    with open(os.path.join(HERE, "tiny_oracle.txt"), "w") as f:
        f.write("\n".join(lines) + "\n")
    # Routing variants on the tiny workload's logits: sigmoid scores, a
    # selection-only bias, 4 groups of 2 experts with 2 kept, scaling 2.5.
    bias = workloads.selection_bias(w.shape.E, seed=1, std=0.05)
    ids, wt = oracle.route_ex(w.logits, w.shape.K, score=oracle.SCORE_SIGMOID, bias=bias, n_group=4,
                              topk_group=2, scaling=2.5)
    lines = ["# oracle route_ex, workload tiny logits; sigmoid, bias selection_bias(8, seed=1, std=0.05),",
             "# 4 groups / 2 kept, renormalised, scaling 2.5; written by tests/golden/make_golden.py",
             "ids " + " ".join(map(str, ids.ravel())),
             "w " + " ".join("%.17g" % v for v in wt.ravel())]
    with open(os.path.join(HERE, "tiny_route_ex.txt"), "w") as f:
        f.write("\n".join(lines) + "\n")


if __name__ == "__main__":
    main()
