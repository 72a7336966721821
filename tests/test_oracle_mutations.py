"""The oracle pins must catch plausible mistakes.

Each case below plants one mistake in a private copy of oracle/gla_oracle.c
(compiled with gcc into a temporary directory, CPU only) and runs the same
independent checks as tests/test_oracle_pins.py against it; at least one
check must fail for every mutant, while the unmodified source passes all.
"""
import os
import subprocess

import numpy as np
import pytest

import oracle
from tests.test_oracle_pins import (brute_force, epilogue, rand_inputs, scan_perm,
                                    _mirror_cols, _transpose_grid)

SRC = os.path.join(os.path.dirname(oracle.__file__), "gla_oracle.c")

# (name, original text, planted mistake)
MUTANTS = [
    ("exclusive_state",
     "            /* S_t = Diag(gamma_t) S_{t-1} + k_t^T v_t */",
     "            if (0) /* placeholder */ ;\n            /* S_t = Diag(gamma_t) S_{t-1} + k_t^T v_t */"),
    ("no_tau", "exp(oracle_log_sigmoid(a[rk + c]) / tau)", "exp(oracle_log_sigmoid(a[rk + c]))"),
    ("dropped_decay", "Sc[j] = gam[c] * Sc[j] + kc * v[rv + j];", "Sc[j] = Sc[j] + kc * v[rv + j];"),
    ("decay_on_value_side", "Sc[j] = gam[c] * Sc[j] + kc * v[rv + j];",
     "Sc[j] = gam[j % d_k] * Sc[j] + kc * v[rv + j];"),
    ("query_is_key", "const double qc = q[rk + c];", "const double qc = k[rk + c];"),
    ("no_scale", "for (int j = 0; j < d_v; ++j) o[j] *= scale;", ""),
    ("b2t_as_t2b", "default: x = p / gh; y = gh - 1 - p % gh; break;",
     "default: x = p / gh; y = p % gh; break;"),
    ("t2b_transposed", "case 2: x = p / gh; y = p % gh; break;",
     "case 2: x = p % gw; y = p / gw; break;"),
    ("r2l_off_by_one", "case 1: y = p / gw; x = gw - 1 - p % gw; break;",
     "case 1: y = p / gw; x = (gw - p % gw) % gw; break;"),
    ("sigmoid_not_silu", "const double silu = gj / (1.0 + exp(-gj));",
     "const double silu = 1.0 / (1.0 + exp(-gj));"),
    ("eps_outside_sqrt", "1.0 / sqrt(ms + eps)", "1.0 / (sqrt(ms) + eps)"),
    ("sum_not_mean", "ms /= (double)d_v;", ""),
    ("gate_sign", "return a - log1p(exp(a));", "return -a - log1p(exp(a));"),
    ("no_weight", "out[rv + j] = o[j] * inv_rms * w[j] * silu;",
     "out[rv + j] = o[j] * inv_rms * silu;"),
]


def _exclusive_patch(src):
    # move the readout above the state update: o_t = q_t S_{t-1}
    upd_start = src.index("            /* S_t = Diag(gamma_t) S_{t-1} + k_t^T v_t */")
    rd_start = src.index("            /* o_t = d_k^{-1/2} q_t S_t */")
    rd_end = src.index("            /* u_t = SiLU(g_t) * RMSNorm(o_t) */")
    upd, rd = src[upd_start:rd_start], src[rd_start:rd_end]
    return src[:upd_start] + rd + upd + src[rd_end:]


def build_variant(tmp_path, name, old, new):
    src = open(SRC).read()
    if name == "exclusive_state":
        src = _exclusive_patch(src)
    else:
        assert old in src, name
        src = src.replace(old, new)
    c = tmp_path / (name + ".c")
    so = tmp_path / (name + ".so")
    c.write_text(src)
    subprocess.check_call(["gcc", "-O1", "-shared", "-fPIC", "-o", str(so), str(c), "-lm"])
    return oracle.load_library(str(so))


def pin_checks(lib):
    """Return the names of the independent checks that this library fails."""
    failed = []
    run = lambda *args, **kw: oracle.gla_forward(*args, lib=lib, **kw)
    rng = np.random.default_rng(5)
    gh, gw = 3, 5
    q, k, v, a, g, w = rand_inputs(rng, 1, gh, gw, 2, 6, 10)
    for d in range(4):
        u = run(q, k, v, a, g, w, gh, gw, d)
        u_ref, _ = brute_force(q, k, v, a, g, w, gh, gw, d)
        if not np.allclose(u, u_ref, rtol=1e-9, atol=1e-12):
            failed.append("brute_force_dir%d" % d)
    # small magnitudes: eps and the scale position become visible
    qs, ks, vs = q * 0.02, k * 0.02, v * 0.02
    u = run(qs, ks, vs, a, g, w, gh, gw, 0)
    u_ref, _ = brute_force(qs, ks, vs, a, g, w, gh, gw, 0)
    if not np.allclose(u, u_ref, rtol=1e-9, atol=1e-14):
        failed.append("brute_force_small")
    # one token
    q1, k1, v1, a1, g1, w1 = rand_inputs(rng, 1, 1, 1, 1, 12, 6)
    u, o = run(q1, k1, v1, a1, g1, w1, 1, 1, 0, return_o=True)
    o_ref = np.dot(q1[0, 0, 0], k1[0, 0, 0]) * v1[0, 0, 0] / np.sqrt(12)
    if not (np.allclose(o[0, 0, 0], o_ref, rtol=1e-12) and
            np.allclose(u, epilogue(o, g1, w1), rtol=1e-12)):
        failed.append("single_token")
    # invariants
    r2l = run(q, k, v, a, g, w, gh, gw, 1)
    via = _mirror_cols(run(*[_mirror_cols(x, gh, gw) for x in (q, k, v, a, g)], w, gh, gw, 0),
                       gh, gw)
    if not np.allclose(r2l, via, rtol=1e-12, atol=1e-14):
        failed.append("invariant_r2l")
    t2b = run(q, k, v, a, g, w, gh, gw, 2)
    via = _transpose_grid(run(*[_transpose_grid(x, gh, gw) for x in (q, k, v, a, g)], w,
                              gw, gh, 0), gw, gh)
    if not np.allclose(t2b, via, rtol=1e-12, atol=1e-14):
        failed.append("invariant_t2b")
    return failed


def test_unmodified_oracle_passes_all_checks():
    assert pin_checks(oracle._load()) == []


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, old, new):
    lib = build_variant(tmp_path, name, old, new)
    assert pin_checks(lib), "mutant %s passed every pin" % name
