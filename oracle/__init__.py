"""CPU oracle for the key-only GLA token mixer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The
product path (``recurrent_vision_backbone_only_b200``) never imports it and
shares no code with it.

The arithmetic lives in ``gla_oracle.c`` (plain sequential fp64 recurrence,
OpenMP over independent (batch, head) pairs); this module only compiles it
with gcc and marshals numpy arrays.  Source: "GTR: Gated Token Recurrence for
Efficient Dense Prediction" (arXiv 2609.26590), method section (GLA
recurrence, retention gate, output gate, scan directions).

Parity status: the recurrence, gate, scale, epilogue and direction map are
pinned by tests/test_oracle_pins.py against closed forms, the brute-force
quadratic form, library routines and direction invariants.  Parity with the
authors' own (unpublished) outputs is unpinned: the pages print no numbers
for the operator.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gla_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

TAU = 16.0
EPS = 1e-6
DIR_L2R, DIR_R2L, DIR_T2B, DIR_B2T, DIR_CYCLE = 0, 1, 2, 3, 4


def build(force: bool = False) -> str:
    """Compile gla_oracle.c into liboracle.so (gcc, OpenMP) when stale."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def load_library(path: str):
    """Open a compiled oracle library and declare its signatures."""
    lib = ctypes.CDLL(path)
    dp = ctypes.POINTER(ctypes.c_double)
    lib.gla_oracle_fwd.restype = ctypes.c_int
    lib.gla_oracle_fwd.argtypes = [dp] * 8 + [ctypes.c_int] * 7 + [
        ctypes.c_double, ctypes.c_double, ctypes.c_int]
    lib.gla_oracle_spatial_index.restype = ctypes.c_long
    lib.gla_oracle_spatial_index.argtypes = [ctypes.c_int, ctypes.c_long,
                                             ctypes.c_long, ctypes.c_long]
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = load_library(build())
    return _lib


def _f64(x):
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(x):
    return x.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def spatial_index(direction: int, p: int, grid_h: int, grid_w: int) -> int:
    """Scan position p -> row-major spatial index (the oracle's own map)."""
    return int(_load().gla_oracle_spatial_index(direction, p, grid_h, grid_w))


def gla_forward(q, k, v, a, g, w, grid_h: int, grid_w: int, direction: int,
                eps: float = EPS, tau: float = TAU, threads: int = 0,
                return_o: bool = False, lib=None):
    """Run the fp64 recurrence.

    q, k, a: [B, L, H, d_k]; v, g: [B, L, H, d_v]; w: [d_v]; L = grid_h*grid_w.
    Inputs of any float dtype are widened to fp64 (exactly, for fp16/fp32).
    Returns u (fp64, same shape as v), and o (pre-epilogue readout) when
    ``return_o``.  ``lib`` selects another compiled copy (used by the
    mutation tests, which compile deliberately broken variants).
    """
    q, k, v, a, g, w = (_f64(t) for t in (q, k, v, a, g, w))
    if q.ndim != 4:
        raise ValueError("q must be [B, L, H, d_k]")
    B, L, H, d_k = q.shape
    d_v = v.shape[-1]
    if L != grid_h * grid_w:
        raise ValueError("L must equal grid_h * grid_w")
    for t, d in ((k, d_k), (a, d_k), (v, d_v), (g, d_v)):
        if t.shape != (B, L, H, d):
            raise ValueError("inconsistent input shapes")
    if w.shape != (d_v,):
        raise ValueError("w must be [d_v]")
    out = np.empty((B, L, H, d_v), dtype=np.float64)
    o = np.empty_like(out) if return_o else None
    rc = (lib or _load()).gla_oracle_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(a), _ptr(g), _ptr(w),
                                _ptr(out), _ptr(o) if o is not None else None,
                                B, H, grid_h, grid_w, d_k, d_v, direction,
                                float(eps), float(tau), int(threads))
    if rc != 0:
        raise RuntimeError("gla_oracle_fwd failed with code %d" % rc)
    return (out, o) if return_o else out


GATE_RANK = 16


def gate_projection(x, w1, w2, b):
    """Retention-gate pre-activation a = x W1 W2 + b, fp64.

    GTR paper (arXiv 2609.26590), method section, GLA recurrence paragraph: the gate is
    gamma_t = sigma(x_t W_alpha^(1) W_alpha^(2) + b_alpha)^(1/tau), a low-rank projection of
    rank r = 16 built the way GLA builds its gate.  Reading taken here (the paragraph writes one head, d_k key
    channels): as in GLA, one first factor W1 [d][r] is shared by the heads and the second factor
    W2 [r][H d_k] maps to every head's key channels, with one bias per key channel.

    x [T][d] (T tokens, d the model width), w1 [d][r], w2 [r][n], b [n]  ->  a [T][n], with
    n = H d_k laid out head-major, i.e. exactly the gate_preact layout [B][L][H][d_k] of the
    operator.  Two library matmuls in the paragraph's order; no reassociation.
    """
    x64 = np.asarray(x, dtype=np.float64)
    w1_64 = np.asarray(w1, dtype=np.float64)
    w2_64 = np.asarray(w2, dtype=np.float64)
    b64 = np.asarray(b, dtype=np.float64)
    if x64.ndim != 2 or w1_64.shape[0] != x64.shape[1] or w2_64.shape[0] != w1_64.shape[1] \
            or b64.shape != (w2_64.shape[1],):
        raise ValueError("gate_projection: shapes x [T][d], w1 [d][r], w2 [r][n], b [n] expected")
    return (x64 @ w1_64) @ w2_64 + b64


SSWIGLU_KERNEL = 3


def spatial_swiglu_mix(value, gate, conv_w, conv_b, grid_h, grid_w):
    """Spatial SwiGLU's token mixing step, fp64: h = SiLU(gate) * (DWConv3x3(value) + conv_b).

    GTR paper (arXiv 2609.26590), method section, Spatial SwiGLU paragraph: the value branch is
    reshaped to the 2-D patch grid, passed through a 3x3 depthwise convolution and restored to
    sequence order; the gating branch stays tokenwise.  The block's equation itself is missing
    from the text; reading taken: SwiGLU's SiLU-activated gating branch multiplies the
    convolved value branch, the convolution being a framework depthwise Conv2d (per-channel
    3x3 cross-correlation, zero padding of one token, one bias per channel).

    value, gate [B][L][C] with L = grid_h * grid_w row-major (s = y * grid_w + x),
    conv_w [C][3][3], conv_b [C]  ->  h [B][L][C].  The nine taps are summed in the order
    (dy, dx) = (-1,-1), (-1,0), ..., (1,1) over a zero-padded copy of the grid.
    """
    v = np.asarray(value, dtype=np.float64)
    g = np.asarray(gate, dtype=np.float64)
    w = np.asarray(conv_w, dtype=np.float64)
    b = np.asarray(conv_b, dtype=np.float64)
    if v.ndim != 3 or g.shape != v.shape or v.shape[1] != grid_h * grid_w:
        raise ValueError("spatial_swiglu_mix: value, gate [B][grid_h*grid_w][C] expected")
    B, L, C = v.shape
    if w.shape != (C, SSWIGLU_KERNEL, SSWIGLU_KERNEL) or b.shape != (C,):
        raise ValueError("spatial_swiglu_mix: conv_w [C][3][3], conv_b [C] expected")
    grid = v.reshape(B, grid_h, grid_w, C)
    padded = np.zeros((B, grid_h + 2, grid_w + 2, C), dtype=np.float64)
    padded[:, 1:grid_h + 1, 1:grid_w + 1, :] = grid
    conv = np.broadcast_to(b, (B, grid_h, grid_w, C)).copy()
    for dy in (-1, 0, 1):
        for dx in (-1, 0, 1):
            conv += w[:, dy + 1, dx + 1] * padded[:, 1 + dy:1 + dy + grid_h, 1 + dx:1 + dx + grid_w, :]
    silu = g / (1.0 + np.exp(-g))
    return silu * conv.reshape(B, L, C)


def linear(x, w, bias=None):
    """y = x W (+ bias), fp64: one library matmul.

    The block's dense projections (GTR paper, arXiv 2609.26590, method section): the input
    projections Q = X W_Q, K = X W_K, V = X W_V and the output gate's x_t W_r (GLA recurrence
    and output-gate paragraphs, no bias written), and the output projection that maps the
    concatenated heads back to the model dimension (output-gate paragraph).  x [T][K],
    w [K][N], bias [N] or None  ->  y [T][N].
    """
    x64 = np.asarray(x, dtype=np.float64)
    w64 = np.asarray(w, dtype=np.float64)
    if x64.ndim != 2 or w64.ndim != 2 or x64.shape[1] != w64.shape[0]:
        raise ValueError("linear: x [T][K], w [K][N] expected")
    y = x64 @ w64
    if bias is not None:
        b64 = np.asarray(bias, dtype=np.float64)
        if b64.shape != (w64.shape[1],):
            raise ValueError("linear: bias [N] expected")
        y = y + b64
    return y


def input_projections(x, w_q, w_k, w_v, w_r):
    """The block's input side, fp64: q = x W_Q, k = x W_K, v = x W_V and the output gate's
    pre-activation x W_r, all heads at once.

    GTR paper, method section, GLA recurrence paragraph (Q = X W_Q, K = X W_K, V = X W_V per
    head, W_Q, W_K in R^{d x d_k}, W_V in R^{d x d_v}) and output-gate paragraph
    (r_t = SiLU(x_t W_r)).  Each weight holds every head's columns head-major, [d][H d], so
    each result is [T][H d] = the operator's [B][L][H][d] layout.  Returns (q, k, v, g).
    """
    return tuple(linear(x, w) for w in (w_q, w_k, w_v, w_r))


def output_projection(u, w_o):
    """Heads concatenated and projected back to the model dimension, fp64: y = concat_h(u_h) W_O.

    GTR paper, method section, output-gate paragraph.  u [T][H d_v] is the operator's output
    [B][L][H][d_v] viewed per token (the concatenation is that layout), w_o [H d_v][d]."""
    return linear(u, w_o)
