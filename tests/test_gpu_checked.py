"""The index-checked build (libgla_checked.so, -DGLA_CHECKED) on the GPU.

Every computed index that addresses memory -- gathered and stored token rows, TMA box
coordinates, remote exchange rows, chunk geometry -- is checked before use in that build, and
a violation latches GLA_ERR_CHECK instead of touching memory.  These cases run every kernel
over the shapes whose index arithmetic differs (ragged and packed grids, reversed and cycling
directions, 1 to 16 segments, a partial-wave split, d = 32 / 64 / 128, fp16 and fp32, and the
gate projection's ragged tiles and split unit ranges, Spatial SwiGLU's ragged tiles and padding, the projections' row and column tiles and parts) and
require that no check fires and that the results still match the oracle.  This stands in for
a device memory checker, which cannot run on this hardware.
"""
import numpy as np
import pytest

import oracle
from recurrent_vision_backbone_only_b200 import build, gla, synth

pytestmark = pytest.mark.gpu

TOL = {"f16": dict(max_abs=1e-2, rel_l2=2e-3), "f32": dict(max_abs=1e-5, rel_l2=1e-5)}
TC128, SIMT, TC64, PIPE64 = gla.KERNEL_TC128, gla.KERNEL_SIMT, gla.KERNEL_TC64, gla.KERNEL_PIPE64


@pytest.fixture(scope="module", autouse=True)
def checked_library():
    """Route every gla call of this module through libgla_checked.so, then restore."""
    path = build.build(checked=True)
    saved = (gla.LIB_PATH, gla._lib)
    gla.LIB_PATH, gla._lib = path, None
    gla.load()
    yield
    gla.LIB_PATH, gla._lib = saved


def run_checked(x, gh, gw, direction, kernel, segments=0, chunk=0):
    import torch
    t = {n: torch.from_numpy(np.ascontiguousarray(x[n])).cuda() for n in ("q", "k", "v", "a", "g", "w")}
    out = torch.empty_like(t["v"])
    if kernel == 0:                                   # fp16 or fp32 by the tensors' dtype
        gla.gla_fwd(t["q"], t["k"], t["v"], t["a"], t["g"], t["w"], out, gh, gw, direction)
    else:
        gla.gla_fwd_ex(t["q"], t["k"], t["v"], t["a"], t["g"], t["w"], out, gh, gw, direction,
                       chunk=chunk, segments=segments, kernel=kernel)
    torch.cuda.synchronize()
    status = gla.get_status()
    assert status == 0, gla.status_string(status)
    return out.cpu().numpy().astype(np.float64)


def check(u, x, gh, gw, direction, dtype):
    ref = oracle.gla_forward(x["q"], x["k"], x["v"], x["a"], x["g"], x["w"], gh, gw, direction)
    d = u - ref
    max_abs = float(np.max(np.abs(d)))
    rel = float(np.linalg.norm(d) / max(np.linalg.norm(ref), 1e-30))
    assert max_abs <= TOL[dtype]["max_abs"] and rel <= TOL[dtype]["rel_l2"], (max_abs, rel)


def test_the_checked_library_is_loaded():
    assert gla.LIB_PATH == gla.LIB_CHECKED_PATH


@pytest.mark.parametrize("kernel,d", [(TC128, 64), (TC64, 64), (TC64, 128), (PIPE64, 64), (SIMT, 32)])
@pytest.mark.parametrize("grid,segments", [((24, 37), 0), ((40, 40), 3), ((16, 20), 9), ((7, 5), 0)])
def test_kernels_shapes_and_directions(kernel, d, grid, segments):
    gh, gw = grid
    wl = synth.WORKLOADS["gtr640"].with_(grid_h=gh, grid_w=gw, H=2, B=2, d_k=d, d_v=d)
    x = synth.make_inputs(wl, seed=gh * gw + d)
    segs = segments if kernel in (TC64, PIPE64) else 0     # the others plan their own
    for direction in (0, 1, 2, 3, 4):
        u = run_checked(x, gh, gw, direction, kernel, segments=segs)
        check(u, x, gh, gw, direction, "f16")


@pytest.mark.parametrize("kernel", [TC64, PIPE64])
def test_sixteen_segments_and_short_chunks(kernel):
    wl = synth.WORKLOADS["gtr640"].with_(grid_h=32, grid_w=40, H=1, B=1)
    x = synth.make_inputs(wl, seed=3)
    for direction in (1, 2):
        u = run_checked(x, 32, 40, direction, kernel, segments=16, chunk=16)
        check(u, x, 32, 40, direction, "f16")


def test_partial_wave_split():
    # more pairs than one wave of the pipelined kernel: a second, segmented launch
    wl = synth.WORKLOADS["batched"].with_(B=3, H=53, grid_h=16, grid_w=24)
    x = synth.make_inputs(wl)
    u = run_checked(x, 16, 24, 4, PIPE64)
    check(u, x, 16, 24, 4, "f16")


def test_fp32_cuda_cores():
    wl = synth.WORKLOADS["tiny"].with_(grid_h=12, grid_w=9, B=2, H=2)
    x = synth.make_inputs(wl)
    for direction in (0, 3, 4):
        u = run_checked(x, 12, 9, direction, 0)
        check(u, x, 12, 9, direction, "f32")


@pytest.mark.parametrize("T,d,n", [(300, 64, 128), (1600, 384, 384), (5000, 128, 640), (40000, 128, 256)])
def test_gate_projection(T, d, n):
    import torch
    inp = synth.make_gate_inputs(T, d, n, seed=T)
    t = [torch.from_numpy(np.ascontiguousarray(inp[k])).cuda() for k in ("x", "w1", "w2", "b")]
    a = torch.empty((T, n), dtype=torch.float16, device="cuda")
    gla.gate_proj(*t, a)
    status = gla.get_status()
    assert status == 0, gla.status_string(status)
    ref = oracle.gate_projection(*(inp[k].astype(np.float64) for k in ("x", "w1", "w2", "b")))
    d_ = a.cpu().numpy().astype(np.float64) - ref
    assert np.max(np.abs(d_)) <= 1e-2 and np.linalg.norm(d_) <= 2e-3 * np.linalg.norm(ref)


@pytest.mark.parametrize("B,gh,gw,C", [(2, 33, 17, 128), (1, 40, 40, 256), (1, 1, 1, 64), (1, 3, 256, 64)])
def test_sswiglu(B, gh, gw, C):
    import torch
    inp = synth.make_sswiglu_inputs(B, gh, gw, C, seed=gh)
    t = {k: torch.from_numpy(np.ascontiguousarray(v)).cuda() for k, v in inp.items()}
    out = torch.empty_like(t["value"])
    gla.sswiglu(t["value"], t["gate"], t["conv_w"], t["conv_b"], out, gh, gw)
    status = gla.get_status()
    assert status == 0, gla.status_string(status)
    ref = oracle.spatial_swiglu_mix(*(inp[k].astype(np.float64) for k in ("value", "gate", "conv_w", "conv_b")), gh, gw)
    d_ = out.cpu().numpy().astype(np.float64) - ref
    assert np.max(np.abs(d_)) <= 1e-2 and np.linalg.norm(d_) <= 2e-3 * np.linalg.norm(ref)


@pytest.mark.parametrize("rows,K,N,n_part", [(300, 64, 128, 128), (1600, 384, 1536, 384), (129, 192, 576, 192)])
def test_linear(rows, K, N, n_part):
    import torch
    inp = synth.make_linear_inputs(rows, K, N, seed=rows, bias=True)
    x, w, b = (torch.from_numpy(inp[k]).cuda() for k in ("x", "w", "b"))
    y = torch.empty((N // n_part, rows, n_part), dtype=torch.float16, device="cuda")
    gla.linear(x, w, y, bias=b, n_part=n_part)
    status = gla.get_status()
    assert status == 0, gla.status_string(status)
    ref = oracle.linear(inp["x"].astype(np.float64), inp["w"].astype(np.float64), inp["b"].astype(np.float64))
    got = np.concatenate(list(y.cpu().numpy()), axis=1).astype(np.float64)
    assert np.max(np.abs(got - ref)) <= 1e-2
