"""Fixtures under tests/golden/: the constants the pages fix, and a frozen copy of the
oracle's output on the tiny workload (a regression guard written by
tests/golden/make_golden.py from oracle/ alone)."""
import json
import os

import numpy as np

import oracle
from recurrent_vision_backbone_only_b200 import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_oracle_uses_the_page_constants():
    with open(os.path.join(GOLDEN, "page_constants.json")) as f:
        c = json.load(f)
    assert oracle.TAU == c["tau"] == 16


def test_oracle_matches_its_frozen_tiny_outputs():
    with open(os.path.join(GOLDEN, "oracle_tiny.json")) as f:
        g = json.load(f)
    wl = synth.WORKLOADS["tiny"]
    x = synth.make_inputs(wl, seed=0)
    for d, vals in g["directions"].items():
        u = oracle.gla_forward(x["q"], x["k"], x["v"], x["a"], x["g"], x["w"], wl.grid_h, wl.grid_w,
                               int(d))
        u = np.asarray(u, dtype=np.float64)[0, g["tokens"], 0, :]
        np.testing.assert_allclose(u, np.asarray(vals), rtol=1e-12, atol=1e-14)
