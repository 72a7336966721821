"""Device-side failure detection, tested without faulting the GPU.

A one-thread kernel waits, with the kernels' bounded-wait loop, on a barrier nothing
ever signals; the wait must run out after its bound, latch GLA_ERR_TIMEOUT in the
device status word, and return.  The operator's own tensor-core kernel is then run with
the gathers of one chunk withheld and a short wait bound: its wait on those tiles must
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


@pytest.mark.parametrize("d,segments", [(64, 1), (64, 4), (128, 3)])
def test_operator_wait_expires_and_returns_promptly(cuda_ok, d, segments):
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
    rc = lib.gla_selftest_fault(*ptrs, 1, 2, 24, 24, d, 0, segments, 2_000_000, 1, None)
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
