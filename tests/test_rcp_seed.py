"""The reciprocal seed constant of the 128-row tensor-core kernel, derived again on the CPU.

rcp_nr starts Newton-Raphson for 1/x from bits(C - bits(x)), reading float bits as integers:
on every binade this is a linear function of the mantissa.  The kernel's comment states that
C = 0x7EF311C7 minimises the seed's largest relative error over a binade (5.05 %), so that three
Newton steps (each squares the error) reach fp32 rounding.  This test repeats that search.
"""
import numpy as np

C = 0x7EF311C7


def seed_max_rel_err(c, m_bits):
    y = (np.int64(c) - m_bits).astype(np.uint32).view(np.float32).astype(np.float64)
    x = m_bits.astype(np.uint32).view(np.float32).astype(np.float64)
    return float(np.max(np.abs(y * x - 1.0)))


def test_seed_constant_is_the_minimax_choice():
    # every mantissa of the binade [1, 2) (the error is the same on every binade)
    m_bits = (np.arange(0, 1 << 23, 7, dtype=np.int64) + (127 << 23))
    err = seed_max_rel_err(C, m_bits)
    assert 0.0500 < err < 0.0506
    # no constant nearby does better by more than a rounding hair
    for c in range(C - (1 << 16), C + (1 << 16), 1 << 9):
        assert seed_max_rel_err(c, m_bits) >= err - 1e-6, hex(c)
    # three Newton steps square the error three times: far below fp32 rounding
    assert err ** 8 < 2.0 ** -30
