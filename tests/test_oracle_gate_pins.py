"""Pins of the oracle's retention-gate projection a = x W1 W2 + b (CPU).

GTR paper, method section, GLA recurrence paragraph: the gate pre-activation is a low-rank
projection x_t W_alpha^(1) W_alpha^(2) + b_alpha of rank r = 16.  The pins do not retype the
oracle's formula: brute force with explicit sums on tiny inputs, the rank-1 closed form, the
zero and identity special cases, and the rank the pages fix.
"""
import json
import os

import numpy as np
import pytest

import oracle


def test_rank_is_the_pages_value():
    d = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_constants.json")))
    assert oracle.GATE_RANK == d["gate_rank"] == 16


@pytest.mark.parametrize("T,d,r,n", [(3, 5, 2, 4), (1, 1, 1, 1), (4, 7, 3, 6)])
def test_brute_force_sums(T, d, r, n):
    rng = np.random.default_rng(T * 100 + d)
    x, w1 = rng.standard_normal((T, d)), rng.standard_normal((d, r))
    w2, b = rng.standard_normal((r, n)), rng.standard_normal(n)
    a = oracle.gate_projection(x, w1, w2, b)
    for t in range(T):
        for c in range(n):
            want = b[c]
            for j in range(r):
                inner = 0.0
                for i in range(d):
                    inner += x[t][i] * w1[i][j]
                want += inner * w2[j][c]
            assert abs(a[t][c] - want) <= 1e-12 * (1 + abs(want))


def test_rank_one_closed_form():
    # r = 1: a[t][c] = (x_t . w1) w2[c] + b[c]
    rng = np.random.default_rng(7)
    x, w1, w2, b = rng.standard_normal((5, 9)), rng.standard_normal((9, 1)), rng.standard_normal((1, 4)), rng.standard_normal(4)
    a = oracle.gate_projection(x, w1, w2, b)
    dots = [sum(float(x[t][i]) * float(w1[i][0]) for i in range(9)) for t in range(5)]
    for t in range(5):
        for c in range(4):
            assert a[t][c] == pytest.approx(dots[t] * w2[0][c] + b[c], rel=1e-13, abs=1e-13)


def test_zero_first_factor_leaves_the_bias():
    x = np.ones((3, 8))
    a = oracle.gate_projection(x, np.zeros((8, 16)), np.ones((16, 5)), np.arange(5.0))
    assert np.array_equal(a, np.tile(np.arange(5.0), (3, 1)))


def test_identity_factors_pass_x_through():
    x = np.arange(12.0).reshape(3, 4)
    a = oracle.gate_projection(x, np.eye(4), np.eye(4), np.full(4, 0.5))
    assert np.array_equal(a, x + 0.5)


def test_shape_errors():
    with pytest.raises(ValueError):
        oracle.gate_projection(np.ones((2, 3)), np.ones((4, 16)), np.ones((16, 5)), np.ones(5))
    with pytest.raises(ValueError):
        oracle.gate_projection(np.ones((2, 3)), np.ones((3, 16)), np.ones((16, 5)), np.ones(4))
