"""Writes tests/golden/c1_expected.json from the oracle alone.

The tiny integer-valued decode workload (1 sequence, L=256, queries at
252..255, H_I=4, d_I=32, K=32, 4 MLA heads, d_c=64, d_rope=16) is run through
the fp64 oracle; its scores are exact integers, so the stored indices are the
unique correct selection. Run: python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from indexed_sparse_attention_relu_b200 import workloads as W  # noqa: E402


def main():
    wl = W.make("c1")
    sc, idx, out, lse = oracle.dsa(wl)
    nv = wl.n_valid()
    doc = {
        "workload": "c1: tiny integer-valued decode (seed 1)",
        "source": "oracle/ (fp64), written by tests/golden/make_golden.py",
        "n_valid": nv.tolist(),
        "scores": [[int(v) for v in sc[t, :nv[t]]] for t in range(wl.T)],
        "idx": idx.tolist(),
        "out": [[[float.hex(float(x)) for x in out[t, h]] for h in range(wl.H)] for t in range(wl.T)],
        "lse": [[float.hex(float(x)) for x in lse[t]] for t in range(wl.T)],
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "c1_expected.json")
    with open(path, "w") as f:
        json.dump(doc, f, indent=0)
    print("wrote", path)


if __name__ == "__main__":
    main()
