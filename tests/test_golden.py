"""The oracle reproduces its stored record of the tiny workload
(tests/golden/tiny_oracle.txt, written by tests/golden/make_golden.py)."""
import os

import numpy as np

from lm_head_exact_fmms_b200 import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "tiny_oracle.txt")


def load_golden():
    rows = [l.split() for l in open(GOLDEN) if l.strip() and not l.startswith("#")]
    return [(int(a), int(b), float(c), float(d)) for a, b, c, d in rows]


def test_oracle_matches_golden(oracle):
    wl = synth.WORKLOADS["tiny"]
    H = synth.make_hidden(1, wl.d)
    W = synth.make_weight(wl.V, wl.d, wl.w_std)
    for step, tok, best, second in load_golden():
        idx, b1, b2 = oracle.sample(H, W, T=wl.temperature, seed=0, step=step)
        assert idx[0] == tok
        assert np.isclose(b1[0], best, rtol=1e-14) and np.isclose(b2[0], second, rtol=1e-14)
