"""The retention gate's low-rank projection a = x W1 W2 + b on the GPU (gla_gate_proj).

GTR paper, method section, GLA recurrence paragraph: gamma_t = sigma(x_t W_alpha^(1)
W_alpha^(2) + b_alpha)^(1/tau) with rank r = 16.  Every output element is compared with the
fp64 oracle.  Bound: the kernel accumulates in fp32 and splits the rank-16 intermediate into
fp16 high and low parts (exact to ~2^-22 relative), then rounds once to fp16.  So
|a - ref| <= half an fp16 ulp of the result + 2^-16 * (|x| |W1| |W2| + |b|), the second term
covering fp32 accumulation over up to 1024 products with margin.
"""
import numpy as np
import pytest

import oracle
from recurrent_vision_backbone_only_b200 import gla, synth

pytestmark = pytest.mark.gpu


def run_gate(x, w1, w2, b, stream=None):
    import torch
    t = [torch.from_numpy(np.ascontiguousarray(v)).cuda() for v in (x, w1, w2, b)]
    a = torch.empty((x.shape[0], w2.shape[1]), dtype=torch.float16, device="cuda")
    gla.gate_proj(*t, a, stream=stream)
    status = gla.get_status(stream)
    return a.cpu().numpy(), status


def half_ulp(v):
    v = np.abs(v).astype(np.float64)
    e = np.floor(np.log2(np.maximum(v, 2.0 ** -14)))
    return 2.0 ** (e - 11)


def check(a, inp):
    x, w1, w2, b = (inp[k].astype(np.float64) for k in ("x", "w1", "w2", "b"))
    ref = oracle.gate_projection(x, w1, w2, b)
    mag = (np.abs(x) @ np.abs(w1)) @ np.abs(w2) + np.abs(b)
    got = a.astype(np.float64)
    err = np.abs(got - ref)
    bound = half_ulp(np.maximum(np.abs(got), np.abs(ref))) + 2.0 ** -16 * mag
    worst = np.unravel_index(np.argmax(err - bound), err.shape)
    assert np.all(err <= bound), (worst, got[worst], ref[worst], bound[worst])
    d = got - ref
    assert np.max(np.abs(d)) <= 1e-2
    assert np.linalg.norm(d) <= 2e-3 * np.linalg.norm(ref)


# Each CTA takes a contiguous range of the (128-token tile, 128-column chunk) units: ranges
# start and end inside tiles, and short inputs give one unit per CTA (1600 tokens: 13 tiles x 3
# chunks = 39 CTAs; 129 tokens: 2 x 8 = 16 CTAs).
@pytest.mark.parametrize("T,d,n", [
    (1600, 384, 384),        # GTR-L at 640 px: 40x40 tokens, width 384, 6 heads of 64
    (300, 64, 128),          # ragged last tile (300 = 2 x 128 + 44)
    (1, 128, 128),           # a single token
    (127, 192, 256),
    (129, 1024, 1024),       # widest model and output
    (6400, 192, 256),
    (5000, 128, 640),        # 40 tiles x 5 chunks over 148 CTAs: ranges of 1 or 2 units
])
def test_gate_matches_oracle(T, d, n):
    inp = synth.make_gate_inputs(T, d, n, seed=T + d + n)
    a, status = run_gate(inp["x"], inp["w1"], inp["w2"], inp["b"])
    assert status == 0, gla.status_string(status)
    check(a, inp)


def test_more_tiles_than_sms():
    # 40,000 tokens = 313 tiles x 3 chunks on 148 CTAs: ranges of 6 or 7 units over 3 or 4
    # tiles each, the X ring wrapping many times and both TMEM output buffers reused
    inp = synth.make_gate_inputs(40000, 128, 384, seed=5)
    a, status = run_gate(inp["x"], inp["w1"], inp["w2"], inp["b"])
    assert status == 0, gla.status_string(status)
    check(a, inp)


def test_feeds_the_operator():
    # a straight into gla_fwd as its gate pre-activation, against the oracle chain with the
    # oracle's gate rounded to fp16 (the operator's input dtype)
    import torch
    wl = synth.WORKLOADS["gtr640"].with_(B=1, H=6)
    x = synth.make_inputs(wl, seed=11)
    gi = synth.make_gate_inputs(wl.B * wl.L, 384, wl.H * wl.d_k, seed=12)
    a, status = run_gate(gi["x"], gi["w1"], gi["w2"], gi["b"])
    assert status == 0
    t = {k: torch.from_numpy(np.ascontiguousarray(x[k])).cuda() for k in ("q", "k", "v", "g", "w")}
    ta = torch.from_numpy(a.reshape(x["a"].shape)).cuda()
    out = torch.empty_like(t["v"])
    gla.gla_fwd(t["q"], t["k"], t["v"], ta, t["g"], t["w"], out, 40, 40, 2)
    assert gla.get_status() == 0
    a_ref = oracle.gate_projection(*(gi[k].astype(np.float64) for k in ("x", "w1", "w2", "b")))
    a16 = a_ref.astype(np.float16).reshape(x["a"].shape)
    ref = oracle.gla_forward(x["q"], x["k"], x["v"], a16, x["g"], x["w"], 40, 40, 2)
    d = out.cpu().numpy().astype(np.float64) - ref
    assert np.max(np.abs(d)) <= 1e-2 and np.linalg.norm(d) <= 2e-3 * np.linalg.norm(ref)


def test_out_of_range_intermediate_is_latched():
    # x W1 = 1000 * 128 = 128,000 > 65,504: the fp16 split cannot hold it
    T, d, n = 128, 128, 128
    x = np.full((T, d), 1000.0, np.float16)
    w1 = np.ones((d, 16), np.float16)
    w2 = np.zeros((16, n), np.float16)
    b = np.zeros(n, np.float32)
    _, status = run_gate(x, w1, w2, b)
    assert status == 8, gla.status_string(status)          # GLA_ERR_RANGE
    inp = synth.make_gate_inputs(T, d, n, seed=1)           # the next call is clean
    a, status = run_gate(inp["x"], inp["w1"], inp["w2"], inp["b"])
    assert status == 0
    check(a, inp)


def test_on_a_side_stream():
    import torch
    s = torch.cuda.Stream()
    inp = synth.make_gate_inputs(1000, 256, 512, seed=9)
    with torch.cuda.stream(s):
        a, status = run_gate(inp["x"], inp["w1"], inp["w2"], inp["b"], stream=s)
    assert status == 0
    check(a, inp)
