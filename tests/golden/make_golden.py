"""Writes tests/golden/tiny_oracle.json: a digest of the fp64 oracle on the
tiny workload (2 frames of 98x98, one head, d=64, hidden 128, seed 0), row-wise
renormalisation.  Calls only the oracle and the seeded input generator.

    python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle as O  # noqa: E402
from recon_chunk_ttt_b200 import workloads as wl  # noqa: E402


def main():
    x = wl.make_inputs("tiny")
    Wh = O.ttt_update(x.W1, x.W2, x.W3, x.K, x.V, x.eta, O.RENORM_ROW)
    out = O.ttt_apply(*Wh, x.Q)
    g = {"_about": "fp64 oracle digest on the tiny workload (row renorm); regenerate with make_golden.py"}
    for i, (name, W) in enumerate((("dW1", x.W1), ("dW2", x.W2), ("dW3", x.W3))):
        d = Wh[i] - W
        g[name + "_fro"] = float(np.linalg.norm(d))
        g[name + "_head8"] = [float(v) for v in d.reshape(-1)[:8]]
    g["O_fro"] = float(np.linalg.norm(out))
    g["O_head8"] = [float(v) for v in out.reshape(-1)[:8]]
    with open(os.path.join(HERE, "tiny_oracle.json"), "w") as f:
        json.dump(g, f, indent=1)


if __name__ == "__main__":
    main()
