"""Writes tests/golden/oracle_tiny.json: the fp64 oracle's outputs on the tiny workload.

Regression fixture only: the values come from oracle/ alone (no CUDA code is involved)
and freeze the oracle's arithmetic, so a later change to it shows up as a failing CPU test
that must name the passage justifying the change.  The oracle's independent pins are in
tests/test_oracle_pins.py.  Run from the repository root:

    python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from recurrent_vision_backbone_only_b200 import synth  # noqa: E402


# spatial token rows kept: the first three, one in the middle, the last
TOKENS = [0, 1, 2, 35, 63]


def main():
    wl = synth.WORKLOADS["tiny"]
    x = synth.make_inputs(wl, seed=0)
    out = {"workload": "tiny: 8x8 grid, B=1, H=1, d_k=d_v=32, fp32 inputs from synth.make_inputs(seed=0)",
           "generator": "tests/golden/make_golden.py (oracle/ only)",
           "tokens": TOKENS, "directions": {}}
    for d in range(4):
        u = oracle.gla_forward(x["q"], x["k"], x["v"], x["a"], x["g"], x["w"], wl.grid_h, wl.grid_w, d)
        u = np.asarray(u, dtype=np.float64)[0, TOKENS, 0, :]          # [tokens, d_v]
        out["directions"][str(d)] = [[float(f"{val:.17g}") for val in row] for row in u]
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_tiny.json")
    with open(path, "w") as f:
        json.dump(out, f)
    print("wrote", path)


if __name__ == "__main__":
    main()
