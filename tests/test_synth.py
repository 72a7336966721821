"""The seeded input generator: deterministic, right shapes, dtypes and distributions."""
import numpy as np

from recurrent_vision_backbone_only_b200 import synth


def test_deterministic_and_shaped():
    wl = synth.WORKLOADS["gtr640"]
    x1, x2 = synth.make_inputs(wl), synth.make_inputs(wl)
    for name in ("q", "k", "v", "a", "g", "w"):
        np.testing.assert_array_equal(x1[name], x2[name])
    assert x1["q"].shape == (1, 1600, 6, 64) and x1["q"].dtype == np.float16
    assert x1["w"].shape == (64,) and x1["w"].dtype == np.float32
    x3 = synth.make_inputs(wl, seed=1)
    assert not np.array_equal(x1["q"], x3["q"])


def test_distributions_follow_workload():
    wl = synth.WORKLOADS["batched"].with_(B=2)
    x = synth.make_inputs(wl)
    a = x["a"].astype(np.float64)
    assert abs(a.mean()) < 0.05 and abs(a.std() - 3.0) < 0.05
    q = x["q"].astype(np.float64)
    assert abs(q.std() - 2 ** -0.5) < 0.01
    wl = synth.WORKLOADS["stress"].with_(grid_h=16, grid_w=16)
    x = synth.make_inputs(wl)
    assert abs(x["a"].astype(np.float64).mean() - 4.0) < 0.05
    assert abs(x["k"].astype(np.float64).std() - 0.5) < 0.01


def test_workload_bookkeeping():
    wl = synth.WORKLOADS["gtr640"]
    assert wl.tokens == 9600 and wl.bytes_per_token == 768
    assert synth.WORKLOADS["stress"].bytes_per_token == 1536
    t = synth.WORKLOADS["tiny"]
    assert t.dtype == "f32" and t.L == 64 and t.chunk == 16
