"""Seeded synthetic inputs for the GLA token mixer.

This module only draws random numbers and rounds them to the I/O dtype; it
holds none of the method's arithmetic, so both the CUDA path (through the
tests and the bench) and the CPU oracle consume exactly the same values.

Workload shapes follow the GTR paper (arXiv 2609.26590): stride-16 patch
grids of 640 px (40x40), 1280 px (80x80) and ~2048 px (128x128, the 16.4K-token
case of the isolated-operator comparison), head dim 64 for the S/L backbones
(H=6 for GTR-L at dim 384).  No dataset is involved; every tensor is drawn
from the distributions listed per workload below.

Draw order is fixed: q, k, v, a (retention-gate pre-activation), g (output
gate pre-activation), w (RMSNorm weight).  Values are produced in fp32 with a
numpy PCG64 generator and then rounded once to the workload's dtype.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Dict, Tuple

import numpy as np

DIR_NAMES = {0: "L2R", 1: "R2L", 2: "T2B", 3: "B2T", 4: "CYCLE"}


@dataclass(frozen=True)
class Workload:
    name: str
    grid_h: int
    grid_w: int
    B: int
    H: int
    d_k: int
    d_v: int
    dtype: str                      # "f16" or "f32"
    qkv_std: float
    a_mean: float
    a_std: float
    w_std: float                    # w = 1 + w_std * N(0,1)
    directions: Tuple[int, ...] = (0,)
    chunk: int = 0                  # 0: the kernel's own choice
    seed: int = 0

    @property
    def L(self) -> int:
        return self.grid_h * self.grid_w

    @property
    def tokens(self) -> int:
        """Tokens in the sense of the throughput metric: B * H * L."""
        return self.B * self.H * self.L

    @property
    def elem_bytes(self) -> int:
        return 2 if self.dtype == "f16" else 4

    @property
    def bytes_per_token(self) -> int:
        """Algorithmic HBM bytes per (b, h, t): q, k, a, v, g read once, u written once."""
        return self.elem_bytes * (3 * self.d_k + 3 * self.d_v)

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS: Dict[str, Workload] = {
    # one head over an 8x8 grid, fp32, the tight-tolerance correctness case
    "tiny": Workload("tiny", 8, 8, 1, 1, 32, 32, "f32", 1.0, 0.0, 1.0, 0.0, (0,), 16),
    # GTR-like 640 px input: 40x40 patches, GTR-L heads
    "gtr640": Workload("gtr640", 40, 40, 1, 6, 64, 64, "f16", 2 ** -0.5, 2.0, 1.0, 0.1,
                       (0, 1, 2, 3)),
    # 1280 px input
    "highres": Workload("highres", 80, 80, 1, 8, 64, 64, "f16", 2 ** -0.5, 2.0, 1.0, 0.1,
                        (0, 1, 2, 3)),
    # batched throughput, directions cycling with the batch index
    "batched": Workload("batched", 40, 40, 16, 12, 64, 64, "f16", 2 ** -0.5, 0.0, 3.0, 0.1,
                        (4,)),
    # long sequence, wide heads, long retention
    "stress": Workload("stress", 128, 128, 2, 8, 128, 128, "f16", 0.5, 4.0, 1.0, 0.1,
                       (2, 3)),
}


def np_dtype(dtype: str):
    return {"f16": np.float16, "f32": np.float32}[dtype]


def make_inputs(wl: Workload, seed: int | None = None) -> Dict[str, np.ndarray]:
    """Draw q, k, v, a, g (token-major [B, L, H, d]) and w ([d_v], fp32).

    Returned arrays already carry the workload dtype (w stays fp32); the same
    rounded values feed the GPU kernel and the oracle.
    """
    rng = np.random.Generator(np.random.PCG64(wl.seed if seed is None else seed))
    B, L, H, dk, dv = wl.B, wl.L, wl.H, wl.d_k, wl.d_v
    dt = np_dtype(wl.dtype)

    def normal(shape, mean, std):
        x = rng.standard_normal(size=shape, dtype=np.float32)
        return (x * np.float32(std) + np.float32(mean)).astype(dt)

    q = normal((B, L, H, dk), 0.0, wl.qkv_std)
    k = normal((B, L, H, dk), 0.0, wl.qkv_std)
    v = normal((B, L, H, dv), 0.0, wl.qkv_std)
    a = normal((B, L, H, dk), wl.a_mean, wl.a_std)
    g = normal((B, L, H, dv), 0.0, 1.0)
    w = (np.float32(1.0) + np.float32(wl.w_std) *
         rng.standard_normal(size=(dv,), dtype=np.float32)).astype(np.float32)
    return {"q": q, "k": k, "v": v, "a": a, "g": g, "w": w}


def make_gate_inputs(tokens: int, d_model: int, n_out: int, rank: int = 16, seed: int = 0,
                     x_std: float = 1.0, b_mean: float = 2.0, b_std: float = 0.5) -> Dict[str, np.ndarray]:
    """Draw the retention gate's projection inputs: x [tokens][d_model], w1 [d_model][rank],
    w2 [rank][n_out] (fp16) and b [n_out] (fp32).

    x is the block's normalised input, N(0, x_std); w1 ~ N(0, 1/d_model) and w2 ~ N(0, 1/rank)
    keep the product near unit scale, and b ~ N(b_mean, b_std) puts the pre-activation where the
    recurrence workloads draw it (mean 2: per-step retention sigma(2)^(1/16) ~ 0.992).  Draw
    order: x, w1, w2, b.
    """
    rng = np.random.Generator(np.random.PCG64(seed))

    def normal(shape, mean, std, dt):
        x = rng.standard_normal(size=shape, dtype=np.float32)
        return (x * np.float32(std) + np.float32(mean)).astype(dt)

    x = normal((tokens, d_model), 0.0, x_std, np.float16)
    w1 = normal((d_model, rank), 0.0, d_model ** -0.5, np.float16)
    w2 = normal((rank, n_out), 0.0, rank ** -0.5, np.float16)
    b = normal((n_out,), b_mean, b_std, np.float32)
    return {"x": x, "w1": w1, "w2": w2, "b": b}


def make_sswiglu_inputs(B: int, grid_h: int, grid_w: int, channels: int, seed: int = 0,
                        w_std: float = 1.0 / 3.0, b_std: float = 0.1) -> Dict[str, np.ndarray]:
    """Draw Spatial SwiGLU's mixing-step inputs: value and gate [B][grid_h*grid_w][channels]
    (fp16, the two branches' projections, N(0, 1)), conv_w [channels][3][3] (fp32,
    N(0, w_std): fan-in 9) and conv_b [channels] (fp32, N(0, b_std)).  Draw order: value,
    gate, conv_w, conv_b."""
    rng = np.random.Generator(np.random.PCG64(seed))
    L = grid_h * grid_w

    def normal(shape, std, dt):
        return (rng.standard_normal(size=shape, dtype=np.float32) * np.float32(std)).astype(dt)

    value = normal((B, L, channels), 1.0, np.float16)
    gate = normal((B, L, channels), 1.0, np.float16)
    conv_w = normal((channels, 3, 3), w_std, np.float32)
    conv_b = normal((channels,), b_std, np.float32)
    return {"value": value, "gate": gate, "conv_w": conv_w, "conv_b": conv_b}


def make_linear_inputs(rows: int, k_dim: int, n_dim: int, seed: int = 0, bias: bool = False) -> Dict[str, np.ndarray]:
    """Draw a dense projection's inputs: x [rows][k_dim] fp16 ~ N(0, 1), w [k_dim][n_dim] fp16
    ~ N(0, 1/k_dim) (unit-scale outputs) and, if asked, bias [n_dim] fp32 ~ N(0, 0.1).  Draw
    order: x, w, bias."""
    rng = np.random.Generator(np.random.PCG64(seed))

    def normal(shape, std, dt):
        return (rng.standard_normal(size=shape, dtype=np.float32) * np.float32(std)).astype(dt)

    out = {"x": normal((rows, k_dim), 1.0, np.float16), "w": normal((k_dim, n_dim), k_dim ** -0.5, np.float16)}
    if bias:
        out["b"] = normal((n_dim,), 0.1, np.float32)
    return out
