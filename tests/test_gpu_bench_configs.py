"""Parity at the exact configurations `bench.py --op` times (same shapes, same seeded inputs,
same launch path), against the fp64 oracle on every output element.

GTR paper, method section: the retention gate's low-rank projection (GLA recurrence
paragraph), the dense projections (GLA recurrence and output-gate paragraphs) and Spatial
SwiGLU's mixing step (Spatial SwiGLU paragraph).  Tolerances are the fp16 ones of the operator:
max-abs <= 1e-2 and relative L2 <= 2e-3.
"""
import numpy as np
import pytest

import bench
import oracle
from recurrent_vision_backbone_only_b200 import gla, synth

pytestmark = pytest.mark.gpu
D_MODEL = 384


def close(got, ref):
    got = got.astype(np.float64)
    d = got - ref
    max_abs = float(np.max(np.abs(d)))
    rel = float(np.linalg.norm(d) / np.linalg.norm(ref))
    assert max_abs <= 1e-2 and rel <= 2e-3, (max_abs, rel)


@pytest.mark.parametrize("workload", ["batched", "gtr640"])
def test_gate_bench_config(workload):
    import torch
    wl = synth.WORKLOADS[workload]
    T, d, n = bench.gate_shape(wl, D_MODEL)
    inp = synth.make_gate_inputs(T, d, n, seed=wl.seed)
    a = torch.empty((T, n), dtype=torch.float16, device="cuda")
    gla.gate_proj(*(torch.from_numpy(inp[k]).cuda() for k in ("x", "w1", "w2", "b")), a)
    assert gla.get_status() == 0
    close(a.cpu().numpy(), oracle.gate_projection(*(inp[k].astype(np.float64) for k in ("x", "w1", "w2", "b"))))


@pytest.mark.parametrize("workload", ["batched", "gtr640", "highres", "stress"])
def test_sswiglu_bench_config(workload):
    import torch
    wl = synth.WORKLOADS[workload]
    C = bench.SSWIGLU_EXPANSION * D_MODEL
    inp = synth.make_sswiglu_inputs(wl.B, wl.grid_h, wl.grid_w, C, seed=wl.seed)
    t = {k: torch.from_numpy(v).cuda() for k, v in inp.items()}
    h = torch.empty_like(t["value"])
    gla.sswiglu(t["value"], t["gate"], t["conv_w"], t["conv_b"], h, wl.grid_h, wl.grid_w)
    assert gla.get_status() == 0
    ref = oracle.spatial_swiglu_mix(*(inp[k].astype(np.float64) for k in ("value", "gate", "conv_w", "conv_b")),
                                    wl.grid_h, wl.grid_w)
    close(h.cpu().numpy(), ref)


@pytest.mark.parametrize("side", ["in", "out"])
@pytest.mark.parametrize("workload", ["batched", "gtr640"])
def test_projection_bench_config(workload, side):
    import torch
    wl = synth.WORKLOADS[workload]
    T, n = wl.B * wl.L, wl.H * wl.d_k
    rows, K, N, n_part = (T, D_MODEL, 4 * n, n) if side == "in" else (T, wl.H * wl.d_v, D_MODEL, D_MODEL)
    inp = synth.make_linear_inputs(rows, K, N, seed=wl.seed)
    y = torch.empty((N // n_part, rows, n_part), dtype=torch.float16, device="cuda")
    gla.linear(torch.from_numpy(inp["x"]).cuda(), torch.from_numpy(inp["w"]).cuda(), y, n_part=n_part)
    assert gla.get_status() == 0
    got = np.concatenate(list(y.cpu().numpy()), axis=1)
    close(got, oracle.linear(inp["x"].astype(np.float64), inp["w"].astype(np.float64)))
