"""The gate projection's precision plan, emulated on the CPU (no GPU, shares no code with the
kernel): fp32 accumulation of x W1, the rank-16 intermediate split into fp16 high and low parts,
both multiplied by W2 with fp32 accumulation, bias added, one rounding to fp16.

GTR paper, method section, GLA recurrence paragraph (the gate's low-rank projection).  The plan
meets the bound the GPU parity test uses (half an fp16 ulp + 2^-16 of the magnitude); with one
fp16 operand for the intermediate (no low part) it does not, which is why the kernel splits.
"""
import numpy as np

import oracle
from recurrent_vision_backbone_only_b200 import synth


def half_ulp(v):
    e = np.floor(np.log2(np.maximum(np.abs(v), 2.0 ** -14)))
    return 2.0 ** (e - 11)


def emulate(inp, split=True):
    x, w1, w2 = (inp[k].astype(np.float32) for k in ("x", "w1", "w2"))
    t = (x @ w1).astype(np.float32)                      # fp32 accumulation
    hi = t.astype(np.float16).astype(np.float32)
    lo = (t - hi).astype(np.float16).astype(np.float32) if split else np.zeros_like(t)
    d = (hi @ w2).astype(np.float32) + (lo @ w2).astype(np.float32)
    return (d + inp["b"]).astype(np.float16).astype(np.float64)


def excess(inp, got):
    ref = oracle.gate_projection(*(inp[k].astype(np.float64) for k in ("x", "w1", "w2", "b")))
    mag = (np.abs(inp["x"].astype(np.float64)) @ np.abs(inp["w1"].astype(np.float64))) @ \
        np.abs(inp["w2"].astype(np.float64)) + np.abs(inp["b"])
    bound = half_ulp(np.maximum(np.abs(got), np.abs(ref))) + 2.0 ** -16 * mag
    return float(np.max(np.abs(got - ref) - bound))


def test_split_plan_meets_the_bound():
    for T, d, n, seed in [(1600, 384, 384, 0), (512, 1024, 256, 1), (300, 64, 128, 2)]:
        inp = synth.make_gate_inputs(T, d, n, seed=seed)
        assert excess(inp, emulate(inp)) <= 0.0


def test_single_fp16_intermediate_misses_it():
    inp = synth.make_gate_inputs(1600, 384, 384, seed=0)
    assert excess(inp, emulate(inp, split=False)) > 0.0
