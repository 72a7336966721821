"""Device-side failure detection, tested without faulting the GPU.

A one-thread kernel waits, with the kernels' bounded-wait loop, on a barrier nothing
ever signals; the wait must run out after its bound, latch GLA_ERR_TIMEOUT in the
device status word, and return.  The operator's own tensor-core kernel is then run with
the loads of one chunk withheld and a short wait bound: its wait on those tiles must
expire, the kernel must skip its remaining waits and products and return promptly, and
GLA_ERR_TIMEOUT must be latched.  The status is read (and cleared) on the host, and the
context must still run the operator correctly afterwards.
"""
import time

import numpy as np
import pytest

import oracle
from recurrent_vision_backbone_only_b200 import build, gla, synth

pytestmark = pytest.mark.gpu


def test_bounded_wait_expires_and_context_survives(cuda_ok):
    import torch
    build.build()
    lib = gla.load()
    assert gla.get_status() == 0
    rc = lib.gla_selftest_timeout(2_000_000, None)      # ~1 ms of SM clocks
    assert rc == 0
    assert gla.get_status() == 7                         # GLA_ERR_TIMEOUT latched
    assert gla.get_status() == 0                         # and cleared by the read
    # the context still works: a small forward matches the oracle
    wl = synth.WORKLOADS["gtr640"].with_(grid_h=8, grid_w=10, H=2)
    x = synth.make_inputs(wl, seed=9)
    t = {n: torch.from_numpy(x[n]).cuda() for n in ("q", "k", "v", "a", "g", "w")}
    out = torch.empty_like(t["v"])
    gla.gla_fwd(t["q"], t["k"], t["v"], t["a"], t["g"], t["w"], out, 8, 10, 1)
    torch.cuda.synchronize()
    assert gla.get_status() == 0
    ref = oracle.gla_forward(x["q"], x["k"], x["v"], x["a"], x["g"], x["w"], 8, 10, 1)
    assert np.max(np.abs(out.cpu().numpy().astype(np.float64) - ref)) < 1e-2


@pytest.mark.parametrize("kernel,d,segments", [(gla.KERNEL_PIPE64, 64, 1), (gla.KERNEL_PIPE64, 64, 4),
                                               (gla.KERNEL_TC64, 64, 1), (gla.KERNEL_TC64, 64, 4),
                                               (gla.KERNEL_TC64, 128, 3), (gla.KERNEL_TC128, 64, 1),
                                               (gla.KERNEL_TC128, 64, 4)])
def test_operator_wait_expires_and_returns_promptly(cuda_ok, kernel, d, segments):
    import torch
    build.build()
    lib = gla.load()
    wl = synth.WORKLOADS["gtr640"].with_(grid_h=24, grid_w=24, H=2, d_k=d, d_v=d)
    x = synth.make_inputs(wl, seed=11)
    t = {n: torch.from_numpy(x[n]).cuda() for n in ("q", "k", "v", "a", "g", "w")}
    out = torch.empty_like(t["v"])
    ptrs = [t[n].data_ptr() for n in ("q", "k", "v", "a", "g", "w")] + [out.data_ptr()]
    torch.cuda.synchronize()
    assert gla.get_status() == 0
    t0 = time.perf_counter()
    # full-pass chunk 1 of every segment is never gathered; waits are bounded by 2e6 clocks
    rc = lib.gla_selftest_fault(*ptrs, 1, 2, 24, 24, d, 0, segments, 2_000_000, 1, kernel, None)
    assert rc == 0, gla.status_string(rc)
    status = gla.get_status()
    elapsed = time.perf_counter() - t0
    assert status == 7                                   # GLA_ERR_TIMEOUT latched
    assert elapsed < 1.0, elapsed                        # the default bound is ~2 s per wait
    assert gla.get_status() == 0
    # the context still works: the same shapes through gla_fwd match the oracle
    gla.gla_fwd(t["q"], t["k"], t["v"], t["a"], t["g"], t["w"], out, 24, 24, 0)
    torch.cuda.synchronize()
    assert gla.get_status() == 0
    ref = oracle.gla_forward(x["q"], x["k"], x["v"], x["a"], x["g"], x["w"], 24, 24, 0)
    assert np.max(np.abs(out.cpu().numpy().astype(np.float64) - ref)) < 1e-2


def test_newton_reciprocal_error_bound(cuda_ok):
    # the 128-row kernel's 1/x (integer-subtraction seed, three Newton steps) over the range its
    # argument 2^(r - b) takes (|r - b| <= 86 in log2 units) stays within 2 ulp of 1/x
    import torch
    build.build()
    lib = gla.load()
    rng = np.random.default_rng(12)
    e = rng.uniform(-86.0, 86.0, 1 << 16)
    x = np.exp2(e).astype(np.float32)
    x[:4] = [1.0, 2.0 ** -86, 2.0 ** 86, 1.5]
    dx = torch.from_numpy(x).cuda()
    dy = torch.empty_like(dx)
    assert lib.gla_selftest_rcp(dx.data_ptr(), dy.data_ptr(), x.size, None) == 0
    torch.cuda.synchronize()
    y = dy.cpu().numpy().astype(np.float64)
    rel = np.abs(y * x.astype(np.float64) - 1.0)
    assert np.max(rel) <= 2.0 ** -22, np.max(rel)
