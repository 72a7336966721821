"""Spatial SwiGLU's fused mixing step on the GPU (gla_sswiglu) against the fp64 oracle.

GTR paper, method section, Spatial SwiGLU paragraph: h = SiLU(gate) * (DWConv3x3(value) + b)
on the patch grid.  Every output element is compared.  Bound: the kernel sums the nine taps in
fp32 and evaluates SiLU with the fast exponential and division (a few ulp of fp32), then rounds
once to fp16, so |h - ref| <= half an fp16 ulp of the result + 2^-16 * |SiLU(g)| (|b| + sum |w v|).
"""
import numpy as np
import pytest

import oracle
from recurrent_vision_backbone_only_b200 import gla, synth

pytestmark = pytest.mark.gpu


def run(inp, gh, gw, stream=None):
    import torch
    t = {k: torch.from_numpy(np.ascontiguousarray(v)).cuda() for k, v in inp.items()}
    out = torch.empty_like(t["value"])
    gla.sswiglu(t["value"], t["gate"], t["conv_w"], t["conv_b"], out, gh, gw, stream=stream)
    status = gla.get_status(stream)
    return out.cpu().numpy(), status


def half_ulp(v):
    e = np.floor(np.log2(np.maximum(np.abs(v), 2.0 ** -14)))
    return 2.0 ** (e - 11)


def check(h, inp, gh, gw):
    v, g, w, b = (inp[k].astype(np.float64) for k in ("value", "gate", "conv_w", "conv_b"))
    ref = oracle.spatial_swiglu_mix(v, g, w, b, gh, gw)
    mag = np.abs(oracle.spatial_swiglu_mix(np.abs(v), g, np.abs(w), np.abs(b), gh, gw))
    got = h.astype(np.float64)
    err = np.abs(got - ref)
    bound = half_ulp(np.maximum(np.abs(got), np.abs(ref))) + 2.0 ** -16 * mag
    worst = np.unravel_index(np.argmax(err - bound), err.shape)
    assert np.all(err <= bound), (worst, got[worst], ref[worst], bound[worst])
    d = got - ref
    assert np.max(np.abs(d)) <= 1e-2
    assert np.linalg.norm(d) <= 2e-3 * np.linalg.norm(ref)


# Tiles are near-equal blocks of at most 8 rows x 16 columns x 64 channels, values with a
# one-token halo: 40 columns -> 3 blocks of 14 (ragged last block), 33 rows -> 5 of 7, 17
# columns -> 2 of 9, 256 columns -> 16 of 16.
@pytest.mark.parametrize("B,gh,gw,C", [
    (1, 40, 40, 1536),       # GTR-L at 640 px: width 384, expansion 4
    (2, 7, 5, 64),
    (1, 1, 1, 64),           # a single token: every neighbour is padding
    (1, 3, 256, 64),         # widest box, 16 column blocks
    (2, 33, 17, 128),
    (1, 80, 80, 256),
    (3, 16, 16, 192),
    (1, 1, 37, 64),          # one grid row: the rows above and below are padding
])
def test_sswiglu_matches_oracle(B, gh, gw, C):
    inp = synth.make_sswiglu_inputs(B, gh, gw, C, seed=B * 1000 + gh * 10 + gw)
    h, status = run(inp, gh, gw)
    assert status == 0, gla.status_string(status)
    check(h, inp, gh, gw)


def test_more_tiles_than_ctas():
    # 16 x 40x40 x 512 channels = 16 x 15 x 8 = 1920 tiles on 296 CTAs (a multiple of the 8
    # slabs): both stages reused many times, one slab per CTA
    inp = synth.make_sswiglu_inputs(16, 40, 40, 512, seed=3)
    h, status = run(inp, 40, 40)
    assert status == 0
    check(h, inp, 40, 40)


def test_out_of_range_is_latched():
    inp = synth.make_sswiglu_inputs(1, 8, 8, 64, seed=4)
    inp["value"][:] = 1000.0
    inp["gate"][:] = 10.0
    inp["conv_w"][:] = 10.0                                 # 9 x 10 x 1000 x ~10 > 65504
    _, status = run(inp, 8, 8)
    assert status == 8, gla.status_string(status)           # GLA_ERR_RANGE
    inp = synth.make_sswiglu_inputs(1, 8, 8, 64, seed=5)
    h, status = run(inp, 8, 8)
    assert status == 0
    check(h, inp, 8, 8)


def test_on_a_side_stream():
    import torch
    s = torch.cuda.Stream()
    inp = synth.make_sswiglu_inputs(2, 20, 12, 128, seed=6)
    with torch.cuda.stream(s):
        h, status = run(inp, 20, 12, stream=s)
    assert status == 0
    check(h, inp, 20, 12)
