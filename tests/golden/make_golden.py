"""Write ``config1_oracle.txt``: the fp64 oracle's output on the seeded tiny
workload (B=1, H=1, N=128, d=64, non-causal, scale = float32(1/8)).

Calls only ``oracle/`` and the seeded input generator.  The file is a
regression fixture for the oracle and the inputs: it holds the SHA-256 of the
input bits, lse for all 128 rows and O for rows 0, 1, 64 and 127.

    python tests/golden/make_golden.py
"""
import hashlib
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import numpy as np  # noqa: E402
import torch  # noqa: E402

import oracle  # noqa: E402
from exact_io_aware_52_b200 import workloads  # noqa: E402

ROWS = (0, 1, 64, 127)


def input_digest(q, k, v) -> str:
    h = hashlib.sha256()
    for t in (q, k, v):
        h.update(t.contiguous().view(torch.int16).numpy().tobytes())
    return h.hexdigest()


def main(path=os.path.join(HERE, "config1_oracle.txt")):
    w = workloads.WORKLOADS[1]
    q, k, v, _ = workloads.make_inputs(w)
    o, lse = oracle.attention_f64(q, k, v, w.causal, w.scale)
    with open(path, "w") as f:
        f.write("# fp64 oracle output, workload: %s, seed %d, scale %r\n" % (w.name, w.seed, w.scale))
        f.write("# written by tests/golden/make_golden.py (oracle only)\n")
        f.write("sha256 %s\n" % input_digest(q, k, v))
        f.write("lse " + " ".join(repr(float(x)) for x in lse) + "\n")
        for r in ROWS:
            f.write("o%d " % r + " ".join(repr(float(x)) for x in o[r]) + "\n")


if __name__ == "__main__":
    main()
