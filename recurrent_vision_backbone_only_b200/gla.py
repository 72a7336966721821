"""ctypes binding of libgla.so -- argument marshalling only.

Every step of the GLA token mixer runs in libgla.so's CUDA kernels; this
module checks tensor shapes/dtypes, passes raw device pointers and the
current CUDA stream, and turns status codes into exceptions.  There is no
fallback: if the library is missing or the device is not an sm_100 GPU the
call raises.

Tensor layout (token-major, head interleaved): q, k, a: [B, L, H, d_k];
v, g, out: [B, L, H, d_v]; w: [d_v] float32; L = grid_h * grid_w row-major.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libgla.so")
# the same library with every computed index checked before use (-DGLA_CHECKED)
LIB_CHECKED_PATH = os.path.join(PKG, "libgla_checked.so")
HEADER = os.path.join(os.path.dirname(PKG), "include", "gla.h")

GLA_OK = 0
STATUS_NAMES = {0: "GLA_OK", 1: "GLA_ERR_NULL", 2: "GLA_ERR_SHAPE", 3: "GLA_ERR_UNSUPPORTED",
                4: "GLA_ERR_DIRECTION", 5: "GLA_ERR_ALIAS", 6: "GLA_ERR_CUDA",
                7: "GLA_ERR_TIMEOUT", 8: "GLA_ERR_RANGE", 9: "GLA_ERR_NO_DEVICE",
                10: "GLA_ERR_CHECK"}
DIR_L2R, DIR_R2L, DIR_T2B, DIR_B2T, DIR_CYCLE = 0, 1, 2, 3, 4

_lib = None


class GLAError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__("%s failed: %s" % (where, status_string(code)))


def load() -> ctypes.CDLL:
    """Open libgla.so (built in-tree by build.py); raise if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libgla.so is not built (run recurrent_vision_backbone_only_b200"
                               ".build or __graft_entry__.build()); there is no fallback path")
        lib = ctypes.CDLL(LIB_PATH)
        vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
        common = [vp] * 7 + [i] * 7
        lib.gla_fwd.argtypes = common + [vp]
        lib.gla_fwd_f32.argtypes = common + [vp]
        lib.gla_fwd_host.argtypes = common + [i, vp]
        lib.gla_fwd_ex.argtypes = common + [i, i, i, f, i, vp]
        lib.gla_get_status.argtypes = [vp, ctypes.POINTER(ctypes.c_int)]
        lib.gla_status_string.argtypes = [i]
        lib.gla_status_string.restype = ctypes.c_char_p
        lib.gla_version.argtypes = []
        lib.gla_selftest_mma.argtypes = [i, vp, vp, vp, vp]
        lib.gla_selftest_timeout.argtypes = [ctypes.c_longlong, vp]
        lib.gla_selftest_timeout.restype = ctypes.c_int
        lib.gla_empty_launch.argtypes = [ctypes.c_int] * 4 + [vp]
        lib.gla_empty_launch.restype = ctypes.c_int
        ip = ctypes.POINTER(ctypes.c_int)
        lib.gla_plan.argtypes = [i] * 7 + [ip] * 5
        lib.gla_plan.restype = ctypes.c_int
        ll = ctypes.c_longlong
        lib.gla_selftest_chunk.argtypes = [i, i, vp, vp, vp, vp]
        lib.gla_selftest_chunk.restype = ctypes.c_int
        lib.gla_selftest_load.argtypes = [vp] * 5 + [i] * 7 + [vp, vp, vp]
        lib.gla_selftest_load.restype = ctypes.c_int
        lib.gla_scan_layout.argtypes = [i] * 5 + [vp, vp]
        lib.gla_scan_layout.restype = ctypes.c_int
        lib.gla_gate_proj.argtypes = [vp] * 5 + [i] * 4 + [vp]
        lib.gla_gate_proj.restype = ctypes.c_int
        lib.gla_sswiglu.argtypes = [vp] * 5 + [i] * 4 + [vp]
        lib.gla_sswiglu.restype = ctypes.c_int
        lib.gla_linear.argtypes = [vp] * 4 + [i] * 4 + [vp]
        lib.gla_linear.restype = ctypes.c_int
        lib.gla_selftest_fault.argtypes = [vp] * 7 + [i] * 7 + [ll, i, i, vp]
        lib.gla_selftest_rcp.argtypes = [vp, vp, i, vp]
        lib.gla_selftest_rcp.restype = ctypes.c_int
        lib.gla_selftest_fault.restype = ctypes.c_int
        for fn in (lib.gla_fwd, lib.gla_fwd_f32, lib.gla_fwd_host, lib.gla_fwd_ex,
                   lib.gla_get_status, lib.gla_version, lib.gla_selftest_mma):
            fn.restype = ctypes.c_int
        _lib = lib
    return _lib


def header_functions() -> list:
    """Names of the functions declared in include/gla.h."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gla_[a-z0-9_]+)\s*\(", text)))


def status_string(code: int) -> str:
    try:
        return load().gla_status_string(int(code)).decode()
    except Exception:  # library missing: still give a readable message
        return STATUS_NAMES.get(code, "status %d" % code)


def _check(rc: int, where: str):
    if rc != GLA_OK:
        raise GLAError(rc, where)


def _dtype_code(t) -> int:
    """0 for float16 I/O, 1 for float32 I/O."""
    import torch
    if t.dtype == torch.float16:
        return 0
    if t.dtype == torch.float32:
        return 1
    raise ValueError("q must be float16 or float32, not %s" % t.dtype)


def _stream_ptr(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dims(q, v, grid_h, grid_w):
    if q.dim() != 4 or v.dim() != 4:
        raise ValueError("q and v must be [B, L, H, d]")
    B, L, H, dk = q.shape
    dv = v.shape[-1]
    if L != grid_h * grid_w:
        raise ValueError("L = %d does not equal grid_h*grid_w = %d" % (L, grid_h * grid_w))
    return int(B), int(H), int(dk), int(dv)


def _check_tensors(q, k, v, a, g, w, out, dtype, on_device: bool = True):
    """Every tensor has the shape, dtype and placement the library reads and writes through its
    raw pointer (device tensors for gla_fwd*, host tensors for gla_fwd_host)."""
    import torch
    where = "CUDA" if on_device else "host (CPU)"
    B, L, H, dk = q.shape
    dv = v.shape[-1]
    for name, t, d in (("q", q, dk), ("k", k, dk), ("a", a, dk), ("v", v, dv),
                       ("g", g, dv), ("out", out, dv)):
        if tuple(t.shape) != (B, L, H, d):
            raise ValueError("%s has shape %s, expected %s" % (name, tuple(t.shape), (B, L, H, d)))
        if t.dtype != dtype or t.is_cuda != on_device or not t.is_contiguous():
            raise ValueError("%s must be a contiguous %s %s tensor" % (name, where, dtype))
    if (tuple(w.shape) != (dv,) or w.dtype != torch.float32 or w.is_cuda != on_device
            or not w.is_contiguous()):
        raise ValueError("w must be a contiguous %s float32 tensor of shape [d_v]" % where)


def gla_fwd(q, k, v, a, g, w, out, grid_h: int, grid_w: int, direction: int, stream=None):
    """u = GLA(q, k, v; gate a) with SiLU(g) * RMSNorm epilogue, into `out` (fp16 or fp32)."""
    import torch
    B, H, dk, dv = _dims(q, v, grid_h, grid_w)
    _check_tensors(q, k, v, a, g, w, out, q.dtype)
    args = [ctypes.c_void_p(t.data_ptr()) for t in (q, k, v, a, g, w, out)]
    args += [B, H, grid_h, grid_w, dk, dv, direction, _stream_ptr(stream)]
    if q.dtype == torch.float16:
        _check(load().gla_fwd(*args), "gla_fwd")
    elif q.dtype == torch.float32:
        _check(load().gla_fwd_f32(*args), "gla_fwd_f32")
    else:
        raise ValueError("q must be float16 or float32")
    return out


KERNEL_AUTO, KERNEL_TC128, KERNEL_SIMT, KERNEL_TC64, KERNEL_PIPE64 = 0, 1, 2, 3, 4
KERNEL_NAMES = {1: "tensor-core 128-row", 2: "cuda-core", 3: "tensor-core 64-row",
                4: "tensor-core 64-row pipelined"}


def gla_fwd_ex(q, k, v, a, g, w, out, grid_h: int, grid_w: int, direction: int,
               chunk: int = 0, segments: int = 0, eps: float = 1e-6, kernel: int = 0,
               stream=None):
    """gla_fwd with the kernel, chunk length, segments per pair and epsilon exposed (tests)."""
    import torch
    B, H, dk, dv = _dims(q, v, grid_h, grid_w)
    _check_tensors(q, k, v, a, g, w, out, q.dtype)
    dtype = _dtype_code(q)
    args = [ctypes.c_void_p(t.data_ptr()) for t in (q, k, v, a, g, w, out)]
    args += [B, H, grid_h, grid_w, dk, dv, direction, dtype, chunk, segments,
             ctypes.c_float(eps), kernel, _stream_ptr(stream)]
    _check(load().gla_fwd_ex(*args), "gla_fwd_ex")
    return out


def gla_fwd_host(q, k, v, a, g, w, out, grid_h: int, grid_w: int, direction: int, stream=None):
    """The same operation on HOST tensors (CPU, ideally pinned); synchronous."""
    B, H, dk, dv = _dims(q, v, grid_h, grid_w)
    dtype = _dtype_code(q)
    _check_tensors(q, k, v, a, g, w, out, q.dtype, on_device=False)
    args = [ctypes.c_void_p(t.data_ptr()) for t in (q, k, v, a, g, w, out)]
    args += [B, H, grid_h, grid_w, dk, dv, direction, dtype, _stream_ptr(stream)]
    _check(load().gla_fwd_host(*args), "gla_fwd_host")
    return out


def plan(B: int, H: int, grid_h: int, grid_w: int, d_k: int = 64, d_v: int = 64,
         dtype: int = 0) -> dict:
    """The launch schedule the library picks for these shapes on the current device."""
    vals = [ctypes.c_int(0) for _ in range(5)]
    _check(load().gla_plan(B, H, grid_h, grid_w, d_k, d_v, dtype, *[ctypes.byref(v) for v in vals]),
           "gla_plan")
    kernel, segs, seg_len, ctas, mac = (v.value for v in vals)
    return {"kernel": KERNEL_NAMES.get(kernel, kernel), "segments": segs,
            "seg_len": seg_len, "ctas": ctas, "max_active_clusters": mac}


def scan_layout(grid_h: int, grid_w: int, direction: int, chunk: int = 0,
                kernel: int = KERNEL_PIPE64):
    """Spatial index of the token the kernel's chunk tiles place at each scan position (host only).

    Returns (spatial: list of grid_h * grid_w ints, box_rows)."""
    L = grid_h * grid_w
    buf = (ctypes.c_int * L)()
    rows = ctypes.c_int(0)
    _check(load().gla_scan_layout(kernel, grid_h, grid_w, direction, chunk, buf, ctypes.byref(rows)),
           "gla_scan_layout")
    return list(buf), rows.value


def gate_proj(x, w1, w2, bias, a, stream=None):
    """a = x W1 W2 + bias (the retention gate's pre-activation, gla_fwd's gate_preact).

    x [tokens, d_model] fp16, w1 [d_model, 16] fp16, w2 [16, n_out] fp16, bias [n_out] fp32,
    a [tokens, n_out] fp16; CUDA tensors, contiguous.  Any leading dims of x / a are tokens."""
    import torch
    tokens = x.numel() // x.shape[-1] if x.dim() else 0
    d_model, rank, n_out = x.shape[-1], w1.shape[-1], w2.shape[-1]
    for t, dt, shape in ((x, torch.float16, None), (w1, torch.float16, (d_model, rank)),
                         (w2, torch.float16, (rank, n_out)), (bias, torch.float32, (n_out,)),
                         (a, torch.float16, None)):
        if not (t.is_cuda and t.is_contiguous() and t.dtype == dt):
            raise ValueError("gate_proj: contiguous CUDA tensors of the documented dtypes expected")
        if shape is not None and tuple(t.shape) != shape:
            raise ValueError("gate_proj: shape %s expected, got %s" % (shape, tuple(t.shape)))
    if a.numel() != tokens * n_out or a.shape[-1] != n_out:
        raise ValueError("gate_proj: a must hold [tokens, n_out]")
    _check(load().gla_gate_proj(*[ctypes.c_void_p(t.data_ptr()) for t in (x, w1, w2, bias, a)],
                                tokens, d_model, rank, n_out, _stream_ptr(stream)), "gla_gate_proj")
    return a


def linear(x, w, y, bias=None, n_part: int = 0, stream=None):
    """y = x W (+ bias): the block's dense projections on tensor cores.

    x [rows, K] fp16, w [K, N] fp16, bias [N] fp32 or None; y holds N / n_part parts of
    [rows, n_part] one after another (default n_part = N: y is [rows, N]).  Leading dims of x
    are rows.  CUDA tensors, contiguous."""
    import torch
    K, N = w.shape
    rows = x.numel() // K if x.dim() else 0
    n_part = n_part or N
    for t, dt in ((x, torch.float16), (w, torch.float16), (y, torch.float16)):
        if not (t.is_cuda and t.is_contiguous() and t.dtype == dt):
            raise ValueError("linear: contiguous fp16 CUDA tensors expected")
    if x.shape[-1] != K or y.numel() != rows * N:
        raise ValueError("linear: x [rows, K] and y holding rows x N expected")
    if bias is not None and not (bias.is_cuda and bias.is_contiguous() and bias.dtype == torch.float32
                                 and tuple(bias.shape) == (N,)):
        raise ValueError("linear: bias must be a contiguous fp32 CUDA tensor [N]")
    _check(load().gla_linear(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(w.data_ptr()),
                             ctypes.c_void_p(bias.data_ptr()) if bias is not None else None,
                             ctypes.c_void_p(y.data_ptr()), rows, K, N, n_part, _stream_ptr(stream)),
           "gla_linear")
    return y


def sswiglu(value, gate, conv_w, conv_b, out, grid_h: int, grid_w: int, stream=None):
    """h = SiLU(gate) * (DWConv3x3(value) + conv_b): Spatial SwiGLU's mixing step.

    value, gate, out [B, grid_h * grid_w, C] fp16; conv_w [C, 3, 3] and conv_b [C] fp32; CUDA
    tensors, contiguous."""
    import torch
    if value.dim() != 3 or value.shape[1] != grid_h * grid_w:
        raise ValueError("sswiglu: value must be [B, grid_h * grid_w, C]")
    B, _, C = value.shape
    for t, dt, shape in ((value, torch.float16, None), (gate, torch.float16, tuple(value.shape)),
                         (out, torch.float16, tuple(value.shape)), (conv_w, torch.float32, (C, 3, 3)),
                         (conv_b, torch.float32, (C,))):
        if not (t.is_cuda and t.is_contiguous() and t.dtype == dt):
            raise ValueError("sswiglu: contiguous CUDA tensors of the documented dtypes expected")
        if shape is not None and tuple(t.shape) != shape:
            raise ValueError("sswiglu: shape %s expected, got %s" % (shape, tuple(t.shape)))
    _check(load().gla_sswiglu(*[ctypes.c_void_p(t.data_ptr()) for t in (value, gate, conv_w, conv_b, out)],
                              B, grid_h, grid_w, C, _stream_ptr(stream)), "gla_sswiglu")
    return out


def empty_launch(B: int, H: int, grid_h: int, grid_w: int, stream=None):
    """Launch the do-nothing kernel with gla_fwd's exact launch shape for these dimensions
    (fp16, d_k = d_v = 64): timing a run of these gives the per-launch floor."""
    _check(load().gla_empty_launch(B, H, grid_h, grid_w, _stream_ptr(stream)), "gla_empty_launch")


def get_status(stream=None) -> int:
    """Synchronise `stream` and return (and clear) the latched device status."""
    val = ctypes.c_int(0)
    _check(load().gla_get_status(_stream_ptr(stream), ctypes.byref(val)), "gla_get_status")
    return val.value


def raw_call(name: str, *args) -> int:
    """Call an entry point with raw ctypes-compatible arguments (host-side error tests)."""
    return getattr(load(), name)(*args)
