"""Host-side checks of the C ABI (no GPU needed).

The library must load on a machine without a GPU, export every function
declared in include/gla.h, and reject bad arguments synchronously with the
documented status codes before touching CUDA.
"""
import ctypes
import os

import pytest

from recurrent_vision_backbone_only_b200 import build, gla

ALIGNED = [0x10000 * (i + 1) for i in range(7)]   # fake, never dereferenced


@pytest.fixture(scope="module")
def lib():
    build.build()
    return gla.load()


def test_exports_every_declared_symbol(lib):
    names = gla.header_functions()
    assert {"gla_fwd", "gla_fwd_f32", "gla_fwd_ex", "gla_fwd_host", "gla_get_status",
            "gla_status_string", "gla_version", "gla_selftest_mma", "gla_selftest_timeout",
            "gla_empty_launch",
            "gla_plan"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n


@pytest.mark.parametrize("checked", [False, True])
def test_exports_via_nm(checked):
    # the release library and its index-checked twin (-DGLA_CHECKED) export the same calls
    import subprocess
    path = build.build(checked=checked)
    assert path == (gla.LIB_CHECKED_PATH if checked else gla.LIB_PATH)
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for n in gla.header_functions():
        assert n in exported, n


def test_version_and_strings(lib):
    assert lib.gla_version() >= 100
    for code in range(11):
        s = gla.status_string(code)
        assert s.startswith(gla.STATUS_NAMES[code])
    assert "unknown" in gla.status_string(99)


def call(fn, ptrs=None, B=1, H=2, gh=4, gw=5, dk=64, dv=64, direction=0, extra=()):
    ptrs = ALIGNED if ptrs is None else ptrs
    args = [ctypes.c_void_p(p) if p is not None else None for p in ptrs]
    args += [B, H, gh, gw, dk, dv, direction, *extra, None]
    return gla.raw_call(fn, *args)


@pytest.mark.parametrize("fn,extra", [("gla_fwd", ()), ("gla_fwd_f32", ()),
                                      ("gla_fwd_host", (0,)),
                                      ("gla_fwd_ex", (0, 0, 0, ctypes.c_float(1e-6), 0))])
def test_argument_errors(lib, fn, extra):
    for i in range(7):
        ptrs = list(ALIGNED)
        ptrs[i] = None
        assert call(fn, ptrs, extra=extra) == 1            # GLA_ERR_NULL
    for kw in (dict(B=0), dict(H=-1), dict(gh=0), dict(gw=0)):
        assert call(fn, extra=extra, **kw) == 2            # GLA_ERR_SHAPE
    assert call(fn, extra=extra, gh=1 << 16, gw=1 << 15) == 2
    for d in (16, 48, 96, 256):
        assert call(fn, extra=extra, dk=d) == 3            # GLA_ERR_UNSUPPORTED
        assert call(fn, extra=extra, dv=d) == 3
    for d in (-1, 5, 100):
        assert call(fn, extra=extra, direction=d) == 4     # GLA_ERR_DIRECTION
    if fn != "gla_fwd_host":
        mis = list(ALIGNED)
        mis[2] += 8
        assert call(fn, mis, extra=extra) == 3             # misaligned
        alias = list(ALIGNED)
        alias[6] = alias[0]                                # out == q
        assert call(fn, alias, extra=extra) == 5           # GLA_ERR_ALIAS


def test_selftest_rejects_bad_arguments(lib):
    f = lib.gla_selftest_mma
    f.argtypes = [ctypes.c_int] + [ctypes.c_void_p] * 4
    assert f(0, None, 16, 16, None) == 1
    assert f(4, 16, 16, 16, None) == 3
    assert f(-1, 16, 16, 16, None) == 3


def test_timeout_selftest_rejects_bad_bound(lib):
    assert lib.gla_empty_launch(0, 6, 40, 40, None) == 2     # GLA_ERR_SHAPE, before any device call
    assert lib.gla_empty_launch(1, 6, 40, -1, None) == 2
    assert lib.gla_selftest_timeout(0, None) == 3
    assert lib.gla_selftest_timeout(1 << 40, None) == 3


def test_plan_rejects_bad_arguments(lib):
    ip = ctypes.POINTER(ctypes.c_int)
    vals = [ctypes.c_int(0) for _ in range(5)]
    args = [1, 6, 40, 40, 64, 64, 0] + [ctypes.byref(v) for v in vals]
    bad = list(args)
    bad[7] = None
    assert lib.gla_plan(*bad) == 1
    assert lib.gla_plan(*([1, 6, 40, 40, 64, 48, 0] + args[7:])) == 3
    assert lib.gla_plan(*([1, 0, 40, 40, 64, 64, 0] + args[7:])) == 2
    assert lib.gla_plan(*([1, 6, 40, 40, 64, 64, 5] + args[7:])) == 3


def test_ex_rejects_bad_schedule(lib):
    bad = [(5, 0, 0, 0), (0, 0, 17, 0), (0, -1, 0, 0), (1, 0, -2, 0),   # dtype, chunk, segs,
           (0, 0, 0, 5), (0, 0, 0, -1), (1, 0, 0, 1), (1, 0, 0, 3), (1, 0, 0, 4)]   # kernel
    for dtype, chunk, segs, kernel in bad:
        rc = call("gla_fwd_ex", extra=(dtype, chunk, segs, ctypes.c_float(1e-6), kernel))
        assert rc == 3, (dtype, chunk, segs, kernel, rc)


def test_no_device_is_reported_not_faked(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert call("gla_fwd") == 9                            # GLA_ERR_NO_DEVICE
    assert call("gla_fwd_f32") == 9


def test_binding_raises_when_library_missing(monkeypatch, tmp_path):
    monkeypatch.setattr(gla, "_lib", None)
    monkeypatch.setattr(gla, "LIB_PATH", os.path.join(str(tmp_path), "missing.so"))
    with pytest.raises(RuntimeError, match="no fallback"):
        gla.load()


def test_binding_rejects_unsupported_dtypes_before_any_call():
    import torch
    x = torch.zeros(1, 4, 1, 64, dtype=torch.bfloat16)
    w = torch.zeros(64)
    with pytest.raises(ValueError):
        gla.gla_fwd_host(x, x, x, x, x, w, x, 2, 2, 0)
    with pytest.raises(ValueError):
        gla.gla_fwd_ex(x, x, x, x, x, w, x, 2, 2, 0)


@pytest.mark.parametrize("bad", ["w_fp16", "out_small", "k_other_d", "g_fp32", "v_strided"])
def test_host_entry_checks_every_tensor_before_any_call(bad):
    # gla_fwd_host copies whole host buffers by raw pointer: a tensor of the wrong shape or
    # dtype must be refused in the binding, before the library reads or writes past its end
    import torch
    B, H, gh, gw, d = 1, 2, 3, 4, 64
    L = gh * gw
    t = {n: torch.zeros(B, L, H, d, dtype=torch.float16) for n in ("q", "k", "v", "a", "g", "out")}
    w = torch.zeros(d, dtype=torch.float32)
    if bad == "w_fp16":
        w = w.half()
    elif bad == "out_small":
        t["out"] = torch.zeros(B, L - 1, H, d, dtype=torch.float16)
    elif bad == "k_other_d":
        t["k"] = torch.zeros(B, L, H, 32, dtype=torch.float16)
    elif bad == "g_fp32":
        t["g"] = t["g"].float()
    else:
        t["v"] = torch.zeros(B, L, H, d, dtype=torch.float16)[..., : d // 2]   # not contiguous
    with pytest.raises(ValueError):
        gla.gla_fwd_host(t["q"], t["k"], t["v"], t["a"], t["g"], w, t["out"], gh, gw, 0)


def test_gate_projection_argument_errors(lib):
    def gate(ptrs=ALIGNED[:5], T=128, d=128, r=16, n=128):
        args = [ctypes.c_void_p(p) if p is not None else None for p in ptrs]
        return gla.raw_call("gla_gate_proj", *args, T, d, r, n, None)
    for i in range(5):
        ptrs = list(ALIGNED[:5])
        ptrs[i] = None
        assert gate(ptrs) == 1                             # GLA_ERR_NULL
    for kw in (dict(T=0), dict(d=-64), dict(n=0), dict(T=(1 << 31) - 1, d=1024)):
        assert gate(**kw) == 2                             # GLA_ERR_SHAPE
    for kw in (dict(r=8), dict(r=32), dict(d=96), dict(d=2048), dict(n=64), dict(n=2048)):
        assert gate(**kw) == 3                             # GLA_ERR_UNSUPPORTED
    mis = list(ALIGNED[:5])
    mis[1] += 4
    assert gate(mis) == 3                                  # misaligned w1
    alias = list(ALIGNED[:5])
    alias[4] = alias[0] + 64                               # a overlaps x
    assert gate(alias) == 5                                # GLA_ERR_ALIAS
    import torch
    if not torch.cuda.is_available():
        assert gate() == 9                                 # GLA_ERR_NO_DEVICE, nothing faked


def test_sswiglu_argument_errors(lib):
    def sw(ptrs=ALIGNED[:5], B=1, gh=4, gw=5, C=64):
        args = [ctypes.c_void_p(p) if p is not None else None for p in ptrs]
        return gla.raw_call("gla_sswiglu", *args, B, gh, gw, C, None)
    for i in range(5):
        ptrs = list(ALIGNED[:5])
        ptrs[i] = None
        assert sw(ptrs) == 1                               # GLA_ERR_NULL
    for kw in (dict(B=0), dict(gh=-1), dict(gw=0), dict(C=0), dict(B=1 << 20, gh=1 << 10, gw=1 << 10, C=1024)):
        assert sw(**kw) == 2                               # GLA_ERR_SHAPE
    for kw in (dict(C=32), dict(C=96)):
        assert sw(**kw) == 3                               # GLA_ERR_UNSUPPORTED
    mis = list(ALIGNED[:5])
    mis[1] += 8
    assert sw(mis) == 3                                    # gate not 16-byte aligned
    alias = list(ALIGNED[:5])
    alias[4] = alias[1] + 16                               # out overlaps gate
    assert sw(alias) == 5                                  # GLA_ERR_ALIAS
    import torch
    if not torch.cuda.is_available():
        assert sw() == 9                                   # GLA_ERR_NO_DEVICE


def test_linear_argument_errors(lib):
    def ln(ptrs=ALIGNED[:4], rows=128, K=64, N=256, n_part=256):
        args = [ctypes.c_void_p(p) if p is not None else None for p in ptrs]
        return gla.raw_call("gla_linear", *args, rows, K, N, n_part, None)
    for i in (0, 1, 3):
        ptrs = list(ALIGNED[:4])
        ptrs[i] = None
        assert ln(ptrs) == 1                               # GLA_ERR_NULL (x, w or y)
    for kw in (dict(rows=0), dict(K=-64), dict(N=0), dict(n_part=0), dict(rows=1 << 30, K=2048)):
        assert ln(**kw) == 2                               # GLA_ERR_SHAPE
    for kw in (dict(K=96), dict(N=320, n_part=320), dict(N=256, n_part=96), dict(N=512, n_part=384)):
        assert ln(**kw) == 3                               # GLA_ERR_UNSUPPORTED
    mis = list(ALIGNED[:4])
    mis[2] += 8
    assert ln(mis) == 3                                    # bias not 16-byte aligned
    alias = list(ALIGNED[:4])
    alias[3] = alias[0] + 32                               # y overlaps x
    assert ln(alias) == 5                                  # GLA_ERR_ALIAS
    import torch
    if not torch.cuda.is_available():
        assert ln() == 9                                   # GLA_ERR_NO_DEVICE
        nb = list(ALIGNED[:4])
        nb[2] = None                                       # no bias is allowed
        assert ln(nb) == 9


def test_new_bindings_check_tensors_before_any_call():
    # host (CPU) tensors and wrong dtypes are rejected in Python, before the library is called
    import torch
    x = torch.zeros(128, 64, dtype=torch.float16)
    with pytest.raises(ValueError):
        gla.gate_proj(x, torch.zeros(64, 16, dtype=torch.float16), torch.zeros(16, 128, dtype=torch.float16),
                      torch.zeros(128), torch.zeros(128, 128, dtype=torch.float16))
    with pytest.raises(ValueError):
        gla.linear(x, torch.zeros(64, 128, dtype=torch.float16), torch.zeros(128, 128, dtype=torch.float16))
    v = torch.zeros(1, 20, 64, dtype=torch.float16)
    with pytest.raises(ValueError):
        gla.sswiglu(v, v, torch.zeros(64, 3, 3), torch.zeros(64), torch.zeros_like(v), 4, 5)
    with pytest.raises(ValueError):
        gla.sswiglu(v, v, torch.zeros(64, 3, 3), torch.zeros(64), torch.zeros_like(v), 5, 5)   # L != 25
