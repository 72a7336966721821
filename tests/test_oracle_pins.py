"""Pins for the CPU oracle (oracle/gla_oracle.c), all CPU-only.

Each check reaches the oracle's result by a route other than the oracle's own
recurrence: the unrolled quadratic form with explicit gate products computed
through ``np.power``, the causal-linear-attention special case (gamma = 1), the
memoryless special case (gamma = 0), the one-token closed form, the zero-key
case, the direction maps built from numpy slicing, and the RMSNorm / SiLU
epilogue from torch's library routines.  Together they catch a dropped or
misplaced decay, an exclusive-instead-of-inclusive state, a transposed state,
a wrong gate exponent, a wrong scale position, and an index error in any scan
direction.

Source of every formula: GTR paper (arXiv 2609.26590), method section -- GLA
recurrence and readout, retention gate sigma(.)^(1/tau) with tau = 16,
key-side decay only, output gate u = SiLU(g) * RMSNorm(o), four scan
directions with spatial order restored.
"""
import numpy as np
import pytest
import torch

import oracle

EPS = 1e-6


def rand_inputs(rng, B, gh, gw, H, dk, dv, a_mean=0.0, a_std=2.0, scale=1.0):
    L = gh * gw
    q = rng.standard_normal((B, L, H, dk)) * scale
    k = rng.standard_normal((B, L, H, dk)) * scale
    v = rng.standard_normal((B, L, H, dv)) * scale
    a = rng.standard_normal((B, L, H, dk)) * a_std + a_mean
    g = rng.standard_normal((B, L, H, dv))
    w = 1.0 + 0.3 * rng.standard_normal(dv)
    return q, k, v, a, g, w


def gate_gamma(a):
    """gamma = sigma(a)^(1/16) via the power function (not the oracle's log form)."""
    sig = 1.0 / (1.0 + np.exp(-a))
    return np.power(sig, 1.0 / 16.0)


def epilogue(o, g, w):
    """SiLU(g) * RMSNorm(o) with torch's own library routines in fp64."""
    ot = torch.from_numpy(np.ascontiguousarray(o))
    n = torch.nn.functional.rms_norm(ot, (o.shape[-1],), weight=torch.from_numpy(w), eps=EPS)
    return (n * torch.nn.functional.silu(torch.from_numpy(np.ascontiguousarray(g)))).numpy()


# ---- direction maps built from numpy slicing of the [gh, gw] grid ----------
def scan_perm(direction, gh, gw):
    """perm[p] = spatial index visited at scan position p."""
    idx = np.arange(gh * gw).reshape(gh, gw)
    if direction == 0:
        return idx.reshape(-1)
    if direction == 1:
        return idx[:, ::-1].reshape(-1)
    if direction == 2:
        return idx.T.reshape(-1)
    if direction == 3:
        return idx[::-1, :].T.reshape(-1)
    raise ValueError(direction)


def brute_force_o(q, k, v, gam):
    """o_t = d_k^-1/2 sum_{s<=t} (q_t * prod_{j=s+1..t} gamma_j) . k_s  v_s, one sequence.

    q, k, gam: [L, d_k]; v: [L, d_v].  The gate product is taken explicitly.
    """
    L, dk = q.shape
    o = np.zeros((L, v.shape[1]))
    for t in range(L):
        for s in range(t + 1):
            decay = np.prod(gam[s + 1:t + 1], axis=0) if t > s else np.ones(dk)
            o[t] += np.dot(q[t] * decay, k[s]) * v[s]
    return o / np.sqrt(dk)


def brute_force(q, k, v, a, g, w, gh, gw, direction):
    B, L, H, dk = q.shape
    dv = v.shape[-1]
    gam = gate_gamma(a)
    o = np.zeros((B, L, H, dv))
    for b in range(B):
        d = b % 4 if direction == 4 else direction
        perm = scan_perm(d, gh, gw)
        for h in range(H):
            o_seq = brute_force_o(q[b, perm, h], k[b, perm, h], v[b, perm, h], gam[b, perm, h])
            o[b, perm, h] = o_seq
    return epilogue(o, g, w), o


@pytest.mark.parametrize("direction", [0, 1, 2, 3])
def test_spatial_index_matches_slicing(direction):
    for gh, gw in [(3, 5), (4, 4), (1, 7), (6, 1)]:
        perm = scan_perm(direction, gh, gw)
        got = [oracle.spatial_index(direction, p, gh, gw) for p in range(gh * gw)]
        assert got == perm.tolist()


@pytest.mark.parametrize("direction", [0, 1, 2, 3, 4])
def test_brute_force_quadratic_form(direction):
    rng = np.random.default_rng(100 + direction)
    gh, gw, B, H, dk, dv = 3, 5, 4 if direction == 4 else 1, 2, 6, 10
    q, k, v, a, g, w = rand_inputs(rng, B, gh, gw, H, dk, dv)
    u, o = oracle.gla_forward(q, k, v, a, g, w, gh, gw, direction, return_o=True)
    u_ref, o_ref = brute_force(q, k, v, a, g, w, gh, gw, direction)
    np.testing.assert_allclose(o, o_ref, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(u, u_ref, rtol=1e-10, atol=1e-12)


def test_brute_force_long_and_fast_decay():
    # 64 tokens, gates from fast forgetting to near-1 retention
    rng = np.random.default_rng(7)
    gh, gw, dk, dv = 8, 8, 8, 5
    q, k, v, a, g, w = rand_inputs(rng, 1, gh, gw, 1, dk, dv, a_mean=-2.0, a_std=6.0)
    u, o = oracle.gla_forward(q, k, v, a, g, w, gh, gw, 0, return_o=True)
    u_ref, o_ref = brute_force(q, k, v, a, g, w, gh, gw, 0)
    np.testing.assert_allclose(o, o_ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(u, u_ref, rtol=1e-9, atol=1e-12)


def test_tiny_magnitudes_scale_before_rmsnorm():
    # |o|^2 comparable to eps: the d_k^-1/2 factor is visible through eps
    rng = np.random.default_rng(3)
    gh, gw, dk, dv = 2, 4, 16, 8
    q, k, v, a, g, w = rand_inputs(rng, 1, gh, gw, 1, dk, dv, scale=0.02)
    u, o = oracle.gla_forward(q, k, v, a, g, w, gh, gw, 0, return_o=True)
    u_ref, o_ref = brute_force(q, k, v, a, g, w, gh, gw, 0)
    assert np.mean(o_ref ** 2) < 1e-4  # eps = 1e-6 matters at this size
    np.testing.assert_allclose(u, u_ref, rtol=1e-10, atol=1e-14)
    # moving the scale after the norm would give a visibly different answer
    o_unscaled = o_ref * np.sqrt(dk)
    u_wrong = epilogue(o_unscaled, g, w)
    assert np.max(np.abs(u_wrong - u)) > 1e-4


def test_gamma_one_is_causal_linear_attention():
    rng = np.random.default_rng(11)
    gh, gw, B, H, dk, dv = 4, 6, 2, 3, 7, 9
    q, k, v, _, g, w = rand_inputs(rng, B, gh, gw, H, dk, dv)
    a = np.full(q.shape, np.inf)           # sigma(+inf) = 1 -> gamma = 1
    u, o = oracle.gla_forward(q, k, v, a, g, w, gh, gw, 0, return_o=True)
    kv = np.einsum("blhc,blhj->blhcj", k, v)
    S = np.cumsum(kv, axis=1)               # S_t = sum_{s<=t} k_s^T v_s
    o_ref = np.einsum("blhc,blhcj->blhj", q, S) / np.sqrt(dk)
    np.testing.assert_allclose(o, o_ref, rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(u, epilogue(o_ref, g, w), rtol=1e-10, atol=1e-12)


def test_gamma_zero_is_memoryless():
    rng = np.random.default_rng(12)
    gh, gw, dk, dv = 3, 3, 5, 4
    q, k, v, _, g, w = rand_inputs(rng, 2, gh, gw, 2, dk, dv)
    a = np.full(q.shape, -np.inf)          # sigma(-inf) = 0 -> gamma = 0
    for d in range(4):
        u, o = oracle.gla_forward(q, k, v, a, g, w, gh, gw, d, return_o=True)
        o_ref = np.sum(q * k, axis=-1, keepdims=True) * v / np.sqrt(dk)
        np.testing.assert_allclose(o, o_ref, rtol=1e-12, atol=1e-13)


def test_single_token_closed_form():
    rng = np.random.default_rng(13)
    dk, dv = 12, 6
    q, k, v, a, g, w = rand_inputs(rng, 1, 1, 1, 1, dk, dv)
    u, o = oracle.gla_forward(q, k, v, a, g, w, 1, 1, 0, return_o=True)
    o_ref = np.dot(q[0, 0, 0], k[0, 0, 0]) * v[0, 0, 0] / np.sqrt(dk)
    np.testing.assert_allclose(o[0, 0, 0], o_ref, rtol=1e-13)
    np.testing.assert_allclose(u, epilogue(o, g, w), rtol=1e-12)


def test_zero_keys_give_zero_output():
    rng = np.random.default_rng(14)
    q, k, v, a, g, w = rand_inputs(rng, 2, 5, 4, 3, 8, 8)
    k[:] = 0.0
    for d in range(5):
        u = oracle.gla_forward(q, k, v, a, g, w, 5, 4, d)
        assert np.all(u == 0.0)


def _mirror_cols(x, gh, gw):   # x -> x mirrored left/right on the grid
    B, L, H, d = x.shape
    return x.reshape(B, gh, gw, H, d)[:, :, ::-1].reshape(B, L, H, d)


def _mirror_rows(x, gh, gw):   # x -> x mirrored top/bottom on the grid
    B, L, H, d = x.shape
    return x.reshape(B, gh, gw, H, d)[:, ::-1].reshape(B, L, H, d)


def _transpose_grid(x, gh, gw):
    B, L, H, d = x.shape
    return x.reshape(B, gh, gw, H, d).transpose(0, 2, 1, 3, 4).reshape(B, L, H, d)


def test_direction_invariants():
    rng = np.random.default_rng(15)
    gh, gw = 4, 7
    q, k, v, a, g, w = rand_inputs(rng, 2, gh, gw, 2, 6, 5)
    run = lambda d, gh_, gw_, *xs: oracle.gla_forward(*xs, w, gh_, gw_, d)

    def tf(f, *xs):
        return [f(x, gh, gw) for x in xs]

    l2r = run(0, gh, gw, q, k, v, a, g)
    # R->L equals L->R on the row-mirrored grid, mirrored back
    r2l = run(1, gh, gw, q, k, v, a, g)
    r2l_via = _mirror_cols(run(0, gh, gw, *tf(_mirror_cols, q, k, v, a, g)), gh, gw)
    np.testing.assert_allclose(r2l, r2l_via, rtol=1e-13, atol=1e-14)
    # T->B equals L->R on the transposed grid, transposed back
    t2b = run(2, gh, gw, q, k, v, a, g)
    t2b_via = _transpose_grid(run(0, gw, gh, *tf(_transpose_grid, q, k, v, a, g)), gw, gh)
    np.testing.assert_allclose(t2b, t2b_via, rtol=1e-13, atol=1e-14)
    # B->T equals T->B on the column-mirrored grid, mirrored back
    b2t = run(3, gh, gw, q, k, v, a, g)
    b2t_via = _mirror_rows(run(2, gh, gw, *tf(_mirror_rows, q, k, v, a, g)), gh, gw)
    np.testing.assert_allclose(b2t, b2t_via, rtol=1e-13, atol=1e-14)
    # the four directions really differ (no accidental identity map)
    assert np.max(np.abs(l2r - r2l)) > 1e-3 and np.max(np.abs(l2r - t2b)) > 1e-3


def test_cycle_is_per_batch_direction():
    rng = np.random.default_rng(16)
    gh, gw = 3, 4
    q, k, v, a, g, w = rand_inputs(rng, 5, gh, gw, 2, 4, 4)
    cyc = oracle.gla_forward(q, k, v, a, g, w, gh, gw, 4)
    for b in range(5):
        sl = slice(b, b + 1)
        one = oracle.gla_forward(q[sl], k[sl], v[sl], a[sl], g[sl], w, gh, gw, b % 4)
        np.testing.assert_array_equal(cyc[sl], one)


def test_pairs_are_independent():
    rng = np.random.default_rng(17)
    gh, gw, B, H = 3, 3, 2, 3
    q, k, v, a, g, w = rand_inputs(rng, B, gh, gw, H, 4, 6)
    full = oracle.gla_forward(q, k, v, a, g, w, gh, gw, 2)
    for b in range(B):
        for h in range(H):
            sb, sh = slice(b, b + 1), slice(h, h + 1)
            one = oracle.gla_forward(q[sb, :, sh], k[sb, :, sh], v[sb, :, sh], a[sb, :, sh],
                                     g[sb, :, sh], w, gh, gw, 2)
            np.testing.assert_array_equal(full[sb, :, sh], one)


def test_threads_do_not_change_result():
    rng = np.random.default_rng(18)
    q, k, v, a, g, w = rand_inputs(rng, 3, 4, 4, 3, 8, 8)
    u1 = oracle.gla_forward(q, k, v, a, g, w, 4, 4, 4, threads=1)
    u4 = oracle.gla_forward(q, k, v, a, g, w, 4, 4, 4, threads=4)
    np.testing.assert_array_equal(u1, u4)


def test_bad_arguments_raise():
    rng = np.random.default_rng(19)
    q, k, v, a, g, w = rand_inputs(rng, 1, 2, 2, 1, 4, 4)
    with pytest.raises(ValueError):
        oracle.gla_forward(q, k, v, a, g, w, 3, 2, 0)
    with pytest.raises(RuntimeError):
        oracle.gla_forward(q, k, v, a, g, w, 2, 2, 7)
