"""Regression fixture: the seeded tiny workload's inputs and oracle output
match what ``tests/golden/make_golden.py`` (oracle only) wrote."""
import os

import numpy as np

import oracle
from exact_io_aware_52_b200 import workloads
from tests.golden.make_golden import ROWS, input_digest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "config1_oracle.txt")


def _read():
    out = {}
    for line in open(GOLDEN):
        if line.startswith("#"):
            continue
        key, *vals = line.split()
        out[key] = vals
    return out


def test_golden_inputs_and_oracle():
    g = _read()
    w = workloads.WORKLOADS[1]
    q, k, v, _ = workloads.make_inputs(w)
    assert input_digest(q, k, v) == g["sha256"][0], "seeded input generator drifted"
    o, lse = oracle.attention_f64(q, k, v, w.causal, w.scale)
    np.testing.assert_allclose(lse, np.array(g["lse"], dtype=np.float64), rtol=0, atol=1e-13)
    for r in ROWS:
        np.testing.assert_allclose(o[r], np.array(g["o%d" % r], dtype=np.float64), rtol=0, atol=1e-13)
