"""GPU parity: libgla.so (through the C ABI) against the fp64 CPU oracle.

Tolerances (on u, the kernel's final output): fp16 I/O with fp32
accumulation -- max-abs <= 1e-2 and relative L2 <= 2e-3; fp32 I/O -- max-abs
<= 1e-5.  Every workload runs at its full size in the launch configuration
the bench uses, and every element of every output is compared with the oracle
(the stress workload, L = 16384 and d = 128, included).
"""
import os

import numpy as np
import pytest

import oracle
from recurrent_vision_backbone_only_b200 import gla, synth

pytestmark = pytest.mark.gpu

TOL = {"f16": dict(max_abs=1e-2, rel_l2=2e-3), "f32": dict(max_abs=1e-5, rel_l2=1e-5)}


def torch_dev(x):
    import torch
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


TC128, SIMT, TC64, PIPE64 = gla.KERNEL_TC128, gla.KERNEL_SIMT, gla.KERNEL_TC64, gla.KERNEL_PIPE64


def run_gpu(x, gh, gw, direction, chunk=0, segments=0, eps=1e-6, kernel=0):
    import torch
    t = {n: torch_dev(x[n]) for n in ("q", "k", "v", "a", "g", "w")}
    out = torch.empty_like(t["v"])
    if chunk or segments or eps != 1e-6 or kernel:
        gla.gla_fwd_ex(t["q"], t["k"], t["v"], t["a"], t["g"], t["w"], out, gh, gw, direction,
                       chunk=chunk, segments=segments, eps=eps, kernel=kernel)
    else:
        gla.gla_fwd(t["q"], t["k"], t["v"], t["a"], t["g"], t["w"], out, gh, gw, direction)
    torch.cuda.synchronize()
    assert gla.get_status() == 0
    return out.cpu().numpy()


def errors(u, ref):
    u = u.astype(np.float64)
    d = u - ref
    return float(np.max(np.abs(d))), float(np.linalg.norm(d) / max(np.linalg.norm(ref), 1e-30))


def _report(max_abs, rel, dtype):
    """Append the error to $GLA_PARITY_REPORT (one JSON line per comparison)."""
    path = os.environ.get("GLA_PARITY_REPORT")
    if path:
        import json
        with open(path, "a") as f:
            f.write(json.dumps({"test": os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0],
                                "dtype": dtype, "max_abs": max_abs, "rel_l2": rel}) + "\n")


def assert_close(u, ref, dtype):
    assert np.all(np.isfinite(u))
    max_abs, rel = errors(u, ref)
    _report(max_abs, rel, dtype)
    tol = TOL[dtype]
    assert max_abs <= tol["max_abs"] and rel <= tol["rel_l2"], (max_abs, rel)


def oracle_ref(x, gh, gw, direction):
    return oracle.gla_forward(x["q"], x["k"], x["v"], x["a"], x["g"], x["w"], gh, gw, direction)


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_ok):
    from recurrent_vision_backbone_only_b200 import build
    build.build()
    gla.load()


@pytest.mark.parametrize("direction", [0, 1, 2, 3])
def test_tiny_fp32(direction):
    wl = synth.WORKLOADS["tiny"]
    x = synth.make_inputs(wl)
    u = run_gpu(x, wl.grid_h, wl.grid_w, direction, chunk=wl.chunk)
    assert_close(u, oracle_ref(x, wl.grid_h, wl.grid_w, direction), "f32")
    u2 = run_gpu(x, wl.grid_h, wl.grid_w, direction)
    assert_close(u2, oracle_ref(x, wl.grid_h, wl.grid_w, direction), "f32")


@pytest.mark.parametrize("kernel", [0, TC64, PIPE64])
@pytest.mark.parametrize("name", ["gtr640", "highres"])
def test_full_workloads_all_directions(name, kernel):
    # kernel 0: the one gla_fwd picks (128-row kernel at 40 x 40, pipelined at 80 x 80)
    wl = synth.WORKLOADS[name]
    x = synth.make_inputs(wl)
    for d in wl.directions:
        assert_close(run_gpu(x, wl.grid_h, wl.grid_w, d, kernel=kernel),
                     oracle_ref(x, wl.grid_h, wl.grid_w, d), wl.dtype)


def test_batched_plan_splits_the_partial_wave():
    # 192 pairs on the pipelined kernel: whole waves one CTA per pair, the remainder in segments
    import torch
    wl = synth.WORKLOADS["batched"]
    pl = gla.plan(wl.B, wl.H, wl.grid_h, wl.grid_w, wl.d_k, wl.d_v, 0)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    pairs = wl.B * wl.H
    assert pl["kernel"] == gla.KERNEL_NAMES[PIPE64]
    if pairs > sms and 2 * (pairs % sms) <= sms:
        assert pl["ctas"] > pairs


@pytest.mark.parametrize("B,H", [(3, 53), (1, 149), (5, 40)])
def test_partial_wave_split_parity(B, H):
    # pair counts just above and around a wave: the tail launch starts mid-batch
    wl = synth.WORKLOADS["batched"].with_(B=B, H=H, grid_h=16, grid_w=24)
    x = synth.make_inputs(wl)
    u = run_gpu(x, wl.grid_h, wl.grid_w, 4, kernel=PIPE64)
    assert_close(u, oracle_ref(x, wl.grid_h, wl.grid_w, 4), wl.dtype)


@pytest.mark.parametrize("kernel", [0, TC64, PIPE64])
def test_batched_cycle(kernel):
    wl = synth.WORKLOADS["batched"]
    x = synth.make_inputs(wl)
    u = run_gpu(x, wl.grid_h, wl.grid_w, 4, kernel=kernel)
    assert_close(u, oracle_ref(x, wl.grid_h, wl.grid_w, 4), wl.dtype)


@pytest.mark.parametrize("direction", [2, 3])
def test_stress_all_pairs(direction):
    # every (b, h) pair of the 128x128, d = 128 workload against one oracle call
    wl = synth.WORKLOADS["stress"]
    x = synth.make_inputs(wl)
    u = run_gpu(x, wl.grid_h, wl.grid_w, direction)
    assert_close(u, oracle_ref(x, wl.grid_h, wl.grid_w, direction), wl.dtype)


@pytest.mark.parametrize("dtype,kernel", [("f16", TC128), ("f16", TC64), ("f16", PIPE64),
                                          ("f16", SIMT), ("f32", SIMT)])
def test_chunk_and_segment_invariance(dtype, kernel):
    wl = synth.WORKLOADS["gtr640"].with_(H=2, dtype=dtype, grid_h=24, grid_w=37)
    x = synth.make_inputs(wl)
    gh, gw = wl.grid_h, wl.grid_w
    ref = oracle_ref(x, gh, gw, 1)
    outs = []
    for chunk in (16, 32, 64):
        for segs in (1, 3, 16):
            u = run_gpu(x, gh, gw, 1, chunk=chunk, segments=segs, kernel=kernel)
            assert_close(u, ref, dtype)
            outs.append(u.astype(np.float64))
    for u in outs[1:]:
        assert_close(u, outs[0], dtype)


@pytest.mark.parametrize("gh,gw,dk,dv", [(1, 1, 64, 64), (7, 9, 64, 64), (1, 33, 32, 128),
                                         (17, 3, 128, 32), (5, 5, 128, 128)])
@pytest.mark.parametrize("dtype", ["f16", "f32"])
def test_ragged_and_mixed_dims(gh, gw, dk, dv, dtype):
    wl = synth.WORKLOADS["gtr640"].with_(grid_h=gh, grid_w=gw, d_k=dk, d_v=dv, B=2, H=3,
                                         dtype=dtype, a_std=3.0, a_mean=0.0)
    x = synth.make_inputs(wl, seed=gh * 100 + gw)
    for d in (0, 3, 4):
        assert_close(run_gpu(x, gh, gw, d), oracle_ref(x, gh, gw, d), dtype)


@pytest.mark.parametrize("dtype", ["f16", "f32"])
def test_extreme_gates(dtype):
    # gamma ~ 0 (a = -30) and gamma ~ 1 (a = +30) mixed per channel and token
    wl = synth.WORKLOADS["gtr640"].with_(grid_h=12, grid_w=12, H=2, dtype=dtype)
    x = synth.make_inputs(wl, seed=3)
    rng = np.random.default_rng(3)
    x["a"] = np.where(rng.random(x["a"].shape) < 0.5, -30.0, 30.0).astype(x["a"].dtype)
    for d in (0, 2):
        assert_close(run_gpu(x, 12, 12, d), oracle_ref(x, 12, 12, d), dtype)


def test_zero_keys_exact_zero():
    wl = synth.WORKLOADS["gtr640"].with_(grid_h=10, grid_w=13, H=2)
    x = synth.make_inputs(wl, seed=4)
    x["k"][:] = 0
    u = run_gpu(x, 10, 13, 1)
    assert np.all(u == 0)


def test_many_pairs_small_grid():
    wl = synth.WORKLOADS["gtr640"].with_(grid_h=4, grid_w=4, B=64, H=4)
    x = synth.make_inputs(wl, seed=5)
    assert_close(run_gpu(x, 4, 4, 4), oracle_ref(x, 4, 4, 4), "f16")


def test_host_entry_matches_device_entry():
    import torch
    wl = synth.WORKLOADS["gtr640"].with_(grid_h=16, grid_w=20, H=3)
    x = synth.make_inputs(wl, seed=6)
    dev = run_gpu(x, 16, 20, 2)
    h = {n: torch.from_numpy(np.ascontiguousarray(x[n])).pin_memory()
         for n in ("q", "k", "v", "a", "g", "w")}
    out = torch.empty_like(h["v"]).pin_memory()
    gla.gla_fwd_host(h["q"], h["k"], h["v"], h["a"], h["g"], h["w"], out, 16, 20, 2)
    np.testing.assert_array_equal(out.numpy(), dev)


def test_eps_is_honoured():
    # tiny inputs: |o|^2 is comparable to eps, so eps changes the answer
    wl = synth.WORKLOADS["tiny"].with_(qkv_std=0.02)
    x = synth.make_inputs(wl)
    for eps in (1e-6, 1e-3):
        u = run_gpu(x, 8, 8, 0, eps=eps)
        ref = oracle.gla_forward(x["q"], x["k"], x["v"], x["a"], x["g"], x["w"], 8, 8, 0,
                                 eps=eps)
        assert_close(u, ref, "f32")


@pytest.mark.parametrize("d,kernel", [(64, TC64), (128, TC64), (64, PIPE64)])
@pytest.mark.parametrize("segs", [2, 5, 7, 12, 13, 15, 16])
def test_segment_counts_64_row_kernel(segs, d, kernel):
    # the state exchange deals key channel c to scanner c % segs: counts that do not divide d
    # give scanners unequal channel counts.  chunk 64 gives segments of one or two chunks,
    # chunk 16 segments of several (state-only pass, exchange, full pass)
    wl = synth.WORKLOADS["gtr640"].with_(H=2, grid_h=24, grid_w=37, d_k=d, d_v=d)
    x = synth.make_inputs(wl, seed=segs)
    ref = oracle_ref(x, 24, 37, 2)
    for chunk in (16, 64):
        assert_close(run_gpu(x, 24, 37, 2, chunk=chunk, segments=segs, kernel=kernel), ref, "f16")


@pytest.mark.parametrize("segs", [2, 5, 7, 12])
def test_segment_counts_128_row_kernel(segs):
    # the 128-row kernel splits the 16 four-channel key groups over the segments; counts that
    # do not divide 16 give some scanners two or more groups.  chunk 128 keeps each segment in
    # one chunk (exchange mid-chunk), chunk 32 gives several chunks per segment
    wl = synth.WORKLOADS["gtr640"].with_(H=2, grid_h=24, grid_w=37)
    x = synth.make_inputs(wl, seed=segs)
    ref = oracle_ref(x, 24, 37, 2)
    for chunk in (32, 128):
        assert_close(run_gpu(x, 24, 37, 2, chunk=chunk, segments=segs, kernel=TC128), ref, "f16")


@pytest.mark.parametrize("kernel,chunk,segs,d", [(TC64, 128, 0, 64), (TC64, 40, 0, 64), (TC64, 64, 17, 64),
                                                 (TC128, 0, 13, 64), (TC128, 0, 15, 64),
                                                 (TC128, 144, 0, 64), (TC128, 0, 0, 128)])
def test_unsupported_schedules_are_refused(kernel, chunk, segs, d):
    import torch
    wl = synth.WORKLOADS["gtr640"].with_(H=1, grid_h=16, grid_w=16, d_k=d, d_v=d)
    x = synth.make_inputs(wl, seed=1)
    t = {n: torch_dev(x[n]) for n in ("q", "k", "v", "a", "g", "w")}
    out = torch.empty_like(t["v"])
    with pytest.raises(gla.GLAError):
        gla.gla_fwd_ex(t["q"], t["k"], t["v"], t["a"], t["g"], t["w"], out, 16, 16, 0,
                       chunk=chunk, segments=segs, kernel=kernel)


@pytest.mark.parametrize("kernel,d,segs,chunk", [(PIPE64, 64, 3, 64), (PIPE64, 64, 16, 64),
                                                 (PIPE64, 64, 5, 32),
                                                 (TC64, 64, 3, 64), (TC64, 64, 16, 64),
                                                 (TC64, 64, 5, 32), (TC64, 128, 3, 64),
                                                 (TC64, 128, 16, 64), (TC64, 128, 5, 32),
                                                 (TC128, 64, 3, 128), (TC128, 64, 16, 128),
                                                 (TC128, 64, 5, 32)])
def test_extreme_gates_with_exchange(kernel, d, segs, chunk):
    # gates of -30 make a chunk's decay range exceed what the 16-bit (64-row kernel) or tf32
    # (128-row kernel) score operands carry, so P is evaluated exactly on CUDA cores; combined
    # here with the cluster state exchange
    wl = synth.WORKLOADS["gtr640"].with_(grid_h=16, grid_w=20, H=2, d_k=d, d_v=d)
    x = synth.make_inputs(wl, seed=7)
    rng = np.random.default_rng(7)
    x["a"] = np.where(rng.random(x["a"].shape) < 0.5, -30.0, 30.0).astype(x["a"].dtype)
    for dr in (1, 3):
        assert_close(run_gpu(x, 16, 20, dr, chunk=chunk, segments=segs, kernel=kernel),
                     oracle_ref(x, 16, 20, dr), "f16")


def test_empty_launch_runs_clean():
    import torch
    gla.empty_launch(1, 6, 40, 40)
    gla.empty_launch(16, 12, 40, 40)
    torch.cuda.synchronize()
    assert gla.get_status() == 0
    assert gla.raw_call("gla_empty_launch", 0, 1, 1, 1, None) == 2      # GLA_ERR_SHAPE


@pytest.mark.parametrize("kernel,gh,gw,chunk,segs", [(TC128, 16, 20, 32, 9), (TC128, 42, 50, 128, 16),
                                                     (TC128, 42, 50, 0, 0), (PIPE64, 16, 20, 32, 9),
                                                     (PIPE64, 42, 50, 64, 16), (TC64, 16, 20, 32, 9),
                                                     (TC64, 42, 50, 64, 16), (TC64, 42, 50, 0, 0)])
def test_shorter_last_segment(kernel, gh, gw, chunk, segs):
    # a last segment shorter than the others (128-row kernel, 16x20: 9 segments of 36 tokens
    # with chunk 32, the last of 32; 42x50: 16 segments of 132, the last of 120; and the
    # automatic plan).  For the 128-row kernel every CTA of a cluster must take the same
    # exchange layout; for the 64-row kernel the last segment holds fewer chunks.
    wl = synth.WORKLOADS["gtr640"].with_(H=2, grid_h=gh, grid_w=gw)
    x = synth.make_inputs(wl, seed=gh + gw)
    for dr in (0, 2):
        assert_close(run_gpu(x, gh, gw, dr, chunk=chunk, segments=segs, kernel=kernel),
                     oracle_ref(x, gh, gw, dr), "f16")
