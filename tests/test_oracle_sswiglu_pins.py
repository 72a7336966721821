"""Pins of the oracle's Spatial SwiGLU mixing step h = SiLU(gate) * (DWConv3x3(value) + b) (CPU).

GTR paper, method section, Spatial SwiGLU paragraph: the value branch goes through a 3x3
depthwise convolution on the patch grid, the gating branch stays tokenwise.  The pins do not
retype the oracle: a framework depthwise convolution and SiLU in fp64, brute force with explicit
bounds checks on tiny grids, the identity and shift kernels (which fix the orientation of the
taps and the zero border), channel independence, and the kernel size the pages fix.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle


def rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def test_kernel_size_is_the_pages_value():
    d = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_constants.json")))
    assert oracle.SSWIGLU_KERNEL == d["sswiglu_kernel"] == 3


@pytest.mark.parametrize("B,gh,gw,C", [(2, 5, 7, 3), (1, 1, 1, 2), (1, 2, 9, 4), (3, 6, 1, 1)])
def test_matches_framework_depthwise_conv(B, gh, gw, C):
    v, g = rand((B, gh * gw, C), 1), rand((B, gh * gw, C), 2)
    w, b = rand((C, 3, 3), 3), rand((C,), 4)
    h = oracle.spatial_swiglu_mix(v, g, w, b, gh, gw)
    vt = torch.from_numpy(v).reshape(B, gh, gw, C).permute(0, 3, 1, 2)
    conv = torch.nn.functional.conv2d(vt, torch.from_numpy(w)[:, None], torch.from_numpy(b),
                                      padding=1, groups=C)
    conv = conv.permute(0, 2, 3, 1).reshape(B, gh * gw, C)
    want = torch.nn.functional.silu(torch.from_numpy(g)) * conv
    np.testing.assert_allclose(h, want.numpy(), rtol=1e-12, atol=1e-12)


def test_brute_force_tiny():
    B, gh, gw, C = 1, 3, 4, 2
    v, g = rand((B, gh * gw, C), 5), rand((B, gh * gw, C), 6)
    w, b = rand((C, 3, 3), 7), rand((C,), 8)
    h = oracle.spatial_swiglu_mix(v, g, w, b, gh, gw)
    for y in range(gh):
        for x in range(gw):
            for c in range(C):
                acc = b[c]
                for i in range(3):
                    for j in range(3):
                        yy, xx = y + i - 1, x + j - 1
                        if 0 <= yy < gh and 0 <= xx < gw:
                            acc += w[c][i][j] * v[0][yy * gw + xx][c]
                gv = g[0][y * gw + x][c]
                want = gv / (1.0 + np.exp(-gv)) * acc
                assert abs(h[0][y * gw + x][c] - want) <= 1e-12 * (1 + abs(want))


def test_identity_kernel_is_tokenwise_swiglu():
    v, g = rand((2, 12, 3), 9), rand((2, 12, 3), 10)
    w = np.zeros((3, 3, 3))
    w[:, 1, 1] = 1.0
    b = np.zeros(3)
    h = oracle.spatial_swiglu_mix(v, g, w, b, 3, 4)
    np.testing.assert_allclose(h, g / (1 + np.exp(-g)) * v, rtol=1e-13)


def test_shift_kernel_orientation_and_zero_border():
    # tap (0, 0) alone: h[y][x] = SiLU(g) * v[y-1][x-1] (cross-correlation), zero off the grid
    gh, gw = 4, 5
    v = np.arange(gh * gw, dtype=np.float64).reshape(1, gh * gw, 1) + 1.0
    g = np.full((1, gh * gw, 1), 50.0)                  # SiLU(50) = 50 to 1e-20
    w = np.zeros((1, 3, 3))
    w[0, 0, 0] = 1.0
    h = oracle.spatial_swiglu_mix(v, g, w, np.zeros(1), gh, gw)[0, :, 0] / 50.0
    for y in range(gh):
        for x in range(gw):
            want = v[0, (y - 1) * gw + (x - 1), 0] if y >= 1 and x >= 1 else 0.0
            assert h[y * gw + x] == pytest.approx(want, abs=1e-12)


def test_channels_are_independent_and_zero_gate_gives_zero():
    v, g = rand((1, 20, 4), 11), rand((1, 20, 4), 12)
    w, b = rand((4, 3, 3), 13), rand((4,), 14)
    h0 = oracle.spatial_swiglu_mix(v, g, w, b, 4, 5)
    v2 = v.copy()
    v2[:, :, 2] += 7.0
    h1 = oracle.spatial_swiglu_mix(v2, g, w, b, 4, 5)
    np.testing.assert_array_equal(h1[:, :, [0, 1, 3]], h0[:, :, [0, 1, 3]])
    assert np.max(np.abs(h1[:, :, 2] - h0[:, :, 2])) > 0.1
    assert not np.any(oracle.spatial_swiglu_mix(v, np.zeros_like(g), w, b, 4, 5))
