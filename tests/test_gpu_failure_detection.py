"""Device-side failure detection, tested without faulting the GPU.

A one-thread kernel waits, with the kernels' bounded-wait loop, on a barrier nothing
ever signals; the wait must run out after its bound, latch GLA_ERR_TIMEOUT in the
device status word, and return.  The status is read (and cleared) on the host, and
the context must still run the operator correctly afterwards.
"""
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
