"""Writes tests/golden/tiny_oracle.txt from the CPU oracle alone.

The pages print no worked example with numbers, so this fixture is the
oracle's own record for the tiny workload (B=1, d=256, V=4096, H ~ N(0,1),
W ~ N(0, 1/d), T=1, seed 0, no mask; steps 0..31), kept to catch unintended
changes to the oracle and to give the GPU smoke check fixed expected tokens.
Run: python tests/golden/make_golden.py
"""
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
from lm_head_exact_fmms_b200 import synth  # noqa: E402


def main():
    wl = synth.WORKLOADS["tiny"]
    H = synth.make_hidden(1, wl.d)
    W = synth.make_weight(wl.V, wl.d, wl.w_std)
    lines = ["# FMMS oracle record, tiny workload: B=1 d=256 V=4096 T=1 seed=0 no mask",
             "# (synth.make_hidden(1, 256), synth.make_weight(4096, 256, 1/16)).",
             "# Written by tests/golden/make_golden.py, which calls only oracle/.",
             "# Method: Gumbel-max over h W^T / T with Philox4x32-10 noise (FlashSampling,",
             "# arXiv:2603.15854, abstract; readus.org page, Gumbel Max Trick section).",
             "# columns: step token best_score second_score"]
    for step in range(32):
        idx, best, second = oracle.sample(H, W, T=wl.temperature, seed=0, step=step)
        lines.append("%d %d %.17g %.17g" % (step, idx[0], best[0], second[0]))
    with open(os.path.join(HERE, "tiny_oracle.txt"), "w") as f:
        f.write("\n".join(lines) + "\n")


if __name__ == "__main__":
    main()
