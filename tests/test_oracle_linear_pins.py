"""Pins of the oracle's dense projections (CPU): linear, input_projections, output_projection.

GTR paper, method section: Q = X W_Q, K = X W_K, V = X W_V per head, the output gate's x W_r,
and the heads concatenated and projected back to the model dimension.  The pins do not retype
the oracle: explicit sums on tiny non-square inputs (a transposed operand fails them), the
per-head reading (head h's q is x times that head's own columns), the concatenation being the
[B][L][H][d] layout, identity weights, and the bias.
"""
import numpy as np
import pytest

import oracle


def rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


@pytest.mark.parametrize("T,K,N", [(3, 5, 4), (1, 1, 1), (4, 2, 7)])
def test_brute_force_sums(T, K, N):
    x, w, b = rand((T, K), T), rand((K, N), K), rand(N, N)
    y = oracle.linear(x, w, b)
    for t in range(T):
        for n in range(N):
            acc = b[n]
            for k in range(K):
                acc += x[t][k] * w[k][n]
            assert abs(y[t][n] - acc) <= 1e-12 * (1 + abs(acc))
    assert np.array_equal(oracle.linear(x, w), y - b) or np.allclose(oracle.linear(x, w), y - b, rtol=1e-14, atol=1e-14)


def test_identity_weight():
    x = rand((6, 8), 1)
    np.testing.assert_array_equal(oracle.linear(x, np.eye(8)), x)


def test_per_head_columns():
    # H = 3 heads of d_k = 4: head h's q is x W_Q^(h), the weight's columns [4h, 4h + 4)
    T, d, H, dk = 5, 7, 3, 4
    x = rand((T, d), 2)
    heads = [rand((d, dk), 10 + h) for h in range(H)]
    w_q = np.concatenate(heads, axis=1)
    q, k, v, g = oracle.input_projections(x, w_q, 2 * w_q, 3 * w_q, -w_q)
    for h in range(H):
        want = np.array([[sum(x[t][i] * heads[h][i][c] for i in range(d)) for c in range(dk)] for t in range(T)])
        np.testing.assert_allclose(q[:, h * dk:(h + 1) * dk], want, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(k, 2 * q, rtol=1e-13)
    np.testing.assert_allclose(v, 3 * q, rtol=1e-13)
    np.testing.assert_allclose(g, -q, rtol=1e-13)


def test_output_projection_concatenates_heads():
    # u in the operator's [B][L][H][d_v] layout: token t's row is heads 0..H-1 side by side
    B, L, H, dv, d = 2, 3, 2, 3, 4
    u = rand((B, L, H, dv), 3)
    w_o = rand((H * dv, d), 4)
    y = oracle.output_projection(u.reshape(B * L, H * dv), w_o)
    for b in range(B):
        for t in range(L):
            cat = np.concatenate([u[b, t, h] for h in range(H)])
            np.testing.assert_allclose(y[b * L + t], cat @ w_o, rtol=1e-12)
            want = sum(u[b, t, h] @ w_o[h * dv:(h + 1) * dv] for h in range(H))
            np.testing.assert_allclose(y[b * L + t], want, rtol=1e-12, atol=1e-12)


def test_shape_checks():
    with pytest.raises(ValueError):
        oracle.linear(np.zeros((2, 3)), np.zeros((4, 5)))
    with pytest.raises(ValueError):
        oracle.linear(np.zeros((2, 3)), np.zeros((3, 5)), np.zeros(4))
