"""Writes tests/golden/oracle_regression.txt from the float64 oracle only.

The fixture freezes the oracle's output on one small seeded case so that a
later change to the oracle's arithmetic cannot pass unnoticed: such a change
must regenerate this file on purpose, and its commit names the passage of the
method that justifies it. Run from the repository root:
    python tests/golden/make_golden.py
"""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from gated_linear_recurrence_rglru_b200.workloads import WORKLOADS, generate  # noqa: E402
from oracle import rglru_oracle as orc  # noqa: E402

CASE = dict(B=2, T=7, D=8, H=2, h0_var=0.25, bias_std=0.5)


def case_inputs():
    wl = WORKLOADS["tiny_f32"].with_shape(**CASE)
    return generate(wl)


def main():
    t = case_inputs()
    y, hT, cs = orc.rglru_fwd(t["x"], t["conv_w"], t["W_a"], t["b_a"], t["W_x"], t["b_x"],
                              t["Lambda"], h0=t["h0"])
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_regression.txt")
    with open(path, "w") as f:
        f.write("# RG-LRU float64 oracle on workload tiny_f32 recipe with %s\n" % CASE)
        f.write("# (the RG-LRU layer with its width-4 Conv1D, as defined in include/rglru.h)\n")
        f.write("# rows: y[b, t, :] for b, t in order, then h_T[b, :]\n")
        for b in range(CASE["B"]):
            for tt in range(CASE["T"]):
                f.write(" ".join("%.17g" % v for v in y[b, tt]) + "\n")
        for b in range(CASE["B"]):
            f.write(" ".join("%.17g" % v for v in hT[b]) + "\n")
    print("wrote", path)


if __name__ == "__main__":
    main()
