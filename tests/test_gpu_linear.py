"""The block's dense projections on the GPU (gla_linear) against the fp64 oracle.

GTR paper, method section: Q = X W_Q, K = X W_K, V = X W_V and x W_r (input side), the
concatenated heads projected back to the model dimension (output side).  Every output element
is compared.  Bound: fp16 products accumulated in fp32 over K <= 1024 terms, rounded once to
fp16: |y - ref| <= half an fp16 ulp of the result + 2^-14 * (|x| |W| + |b|).
"""
import numpy as np
import pytest

import oracle
from recurrent_vision_backbone_only_b200 import gla, synth

pytestmark = pytest.mark.gpu


def run(inp, n_part=0, stream=None):
    import torch
    x, w = (torch.from_numpy(inp[k]).cuda() for k in ("x", "w"))
    b = torch.from_numpy(inp["b"]).cuda() if "b" in inp else None
    rows, N = x.shape[0], w.shape[1]
    n_part = n_part or N
    y = torch.empty((N // n_part, rows, n_part), dtype=torch.float16, device="cuda")
    gla.linear(x, w, y, bias=b, n_part=n_part, stream=stream)
    return y.cpu().numpy(), gla.get_status(stream)


def half_ulp(v):
    e = np.floor(np.log2(np.maximum(np.abs(v), 2.0 ** -14)))
    return 2.0 ** (e - 11)


def check(y_parts, inp):
    x, w = inp["x"].astype(np.float64), inp["w"].astype(np.float64)
    b = inp["b"].astype(np.float64) if "b" in inp else None
    ref = oracle.linear(x, w, b)
    mag = oracle.linear(np.abs(x), np.abs(w), None if b is None else np.abs(b))
    got = np.concatenate(list(y_parts), axis=1).astype(np.float64)   # parts side by side
    err = np.abs(got - ref)
    bound = half_ulp(np.maximum(np.abs(got), np.abs(ref))) + 2.0 ** -14 * mag
    worst = np.unravel_index(np.argmax(err - bound), err.shape)
    assert np.all(err <= bound), (worst, got[worst], ref[worst], bound[worst])


# column tiles of 256, 192 or 128 (the largest dividing N); rows in 128-row tiles
@pytest.mark.parametrize("rows,K,N,n_part,bias", [
    (1600, 384, 1536, 384, False),   # GTR-L input side at 640 px: q, k, v, W_r as four parts
    (1600, 384, 384, 384, True),     # GTR-L output projection (192-column tiles)
    (300, 64, 128, 128, True),       # ragged last row tile
    (1, 128, 256, 256, False),       # a single row
    (5000, 1024, 768, 256, False),   # K = 1024, three parts
    (129, 192, 576, 192, True),      # 192-column tiles, three parts
])
def test_linear_matches_oracle(rows, K, N, n_part, bias):
    inp = synth.make_linear_inputs(rows, K, N, seed=rows + K + N, bias=bias)
    y, status = run(inp, n_part)
    assert status == 0, gla.status_string(status)
    check(y, inp)


def test_more_tiles_than_sms():
    inp = synth.make_linear_inputs(40000, 128, 512, seed=7, bias=True)   # 313 x 2 tiles
    y, status = run(inp)
    assert status == 0
    check(y, inp)


def test_input_side_writes_the_operator_layout():
    # W = [W_Q | W_K | W_V | W_r]: the four parts are q, k, v and g exactly as the oracle's
    # input_projections gives them per token, [B][L][H][d] = [T][H d]
    T, d, n = 640, 128, 256
    inp = synth.make_linear_inputs(T, d, 4 * n, seed=8)
    y, status = run(inp, n)
    assert status == 0
    ws = [inp["w"][:, i * n:(i + 1) * n] for i in range(4)]
    refs = oracle.input_projections(inp["x"].astype(np.float64), *[w.astype(np.float64) for w in ws])
    for part, ref in zip(y, refs):
        assert np.max(np.abs(part.astype(np.float64) - ref)) <= 4e-3


def test_block_token_mixer_end_to_end():
    # x -> q, k, v, g (gla_linear) and a (gla_gate_proj) -> gla_fwd -> y = u W_O (gla_linear),
    # against the oracle chain with every intermediate rounded to fp16 where the GPU path
    # stores one
    import torch
    B, gh, gw, H, dh, d = 1, 24, 20, 4, 64, 256
    T, n = B * gh * gw, H * dh
    rng = np.random.default_rng(9)
    x = rng.standard_normal((T, d)).astype(np.float16)
    w_in = (rng.standard_normal((d, 4 * n)) * d ** -0.5).astype(np.float16)
    w_o = (rng.standard_normal((n, d)) * n ** -0.5).astype(np.float16)
    gi = synth.make_gate_inputs(T, d, n, seed=10)
    w_norm = np.ones(dh, np.float32)
    for direction in (0, 3):
        xt, wt, wo = (torch.from_numpy(v).cuda() for v in (x, w_in, w_o))
        qkvg = torch.empty((4, T, n), dtype=torch.float16, device="cuda")
        gla.linear(xt, wt, qkvg, n_part=n)
        a = torch.empty((T, n), dtype=torch.float16, device="cuda")
        gla.gate_proj(xt, *(torch.from_numpy(gi[k]).cuda() for k in ("w1", "w2", "b")), a)
        shp = (B, gh * gw, H, dh)
        u = torch.empty(shp, dtype=torch.float16, device="cuda")
        gla.gla_fwd(qkvg[0].view(shp), qkvg[1].view(shp), qkvg[2].view(shp), a.view(shp), qkvg[3].view(shp),
                    torch.from_numpy(w_norm).cuda(), u, gh, gw, direction)
        y = torch.empty((T, d), dtype=torch.float16, device="cuda")
        gla.linear(u.view(T, n), wo, y)
        assert gla.get_status() == 0
        x64 = x.astype(np.float64)
        q, k, v, g = (r.astype(np.float16) for r in oracle.input_projections(
            x64, *[w_in[:, i * n:(i + 1) * n].astype(np.float64) for i in range(4)]))
        a16 = oracle.gate_projection(x64, *(gi[kk].astype(np.float64) for kk in ("w1", "w2", "b"))).astype(np.float16)
        u_ref = oracle.gla_forward(*(t.reshape(shp) for t in (q, k, v, a16, g)), w_norm, gh, gw, direction)
        y_ref = oracle.output_projection(u_ref.astype(np.float16).astype(np.float64).reshape(T, n), w_o.astype(np.float64))
        dlt = y.cpu().numpy().astype(np.float64) - y_ref
        assert np.max(np.abs(dlt)) <= 2e-2 and np.linalg.norm(dlt) <= 3e-3 * np.linalg.norm(y_ref), \
            (np.max(np.abs(dlt)), np.linalg.norm(dlt) / np.linalg.norm(y_ref))


def test_on_a_side_stream():
    import torch
    s = torch.cuda.Stream()
    inp = synth.make_linear_inputs(700, 256, 384, seed=11, bias=True)
    with torch.cuda.stream(s):
        y, status = run(inp, stream=s)
    assert status == 0
    check(y, inp)
