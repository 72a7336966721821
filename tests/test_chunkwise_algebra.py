"""The chunkwise form evaluated by the tensor-core kernel, restated in numpy and checked
against the fp64 oracle on the CPU (no GPU, no code shared with the kernels).

GTR paper (arXiv 2609.26590), method section and its chunkwise CUDA operator: the
recurrence S_t = Diag(gamma_t) S_{t-1} + k_t^T v_t, o_t = d_k^{-1/2} q_t S_t is evaluated
chunk by chunk.  With b_t the in-chunk cumulative log2-decay (inclusive), B its last row
and r a reference row:

    intra  O = tril(Q~ K~^T) V,   K~ = k 2^(r-b),   Q~ = d_k^{-1/2} q 2^(b-r)
    inter  O += Q~ (Diag(2^r) S_in)
    state  S_out = Diag(2^B) S_in + (k 2^(B-b))^T V

and a scan cut into segments combines (G, S) pairs as S_in' = Diag(2^G) S_in + S.

These tests pin three things.  (1) The factorisation is exact: it matches the recurrence in
fp64 for any chunk length, reference row, segment count and direction.  (2) The kernel's
precision plan keeps u within the fp16 tolerance, emulated at its rounding points: split
tf32 score operands (high part = the fp32 value with its low 13 mantissa bits cleared,
what the tensor core reads; low part = the remainder, read the same way), an exact fp32
diagonal, fp16 P and decayed keys, tf32 S~, fp32 accumulation, fp16 output.  A single
tf32 operand per side is shown to miss that tolerance on a first token whose readout
nearly cancels.  (3) A candidate plan with every product as kind::f16 -- split bf16
scores, a split fp16 inter operand against fp16 states, states exchanged in fp16 -- stays
within the tolerance, while bf16 states or one tf32 score operand per side do not.
"""
import math

import numpy as np
import pytest

import oracle
from tests.test_oracle_pins import rand_inputs, scan_perm

EPS = 1e-6
LN2 = math.log(2.0)


def log2_gate(a):
    """log2(sigma(a)) / 16 with the stable log-sigmoid."""
    return (np.minimum(a, 0.0) - np.log1p(np.exp(-np.abs(a)))) / LN2 / 16.0


def ref_row(n, where):
    return {"first": 0, "middle": n // 2, "last": n - 1}[where]


def chunk_exact(q, k, v, lg, S_in, where):
    """One chunk of the factorised form in fp64: (O, S_out, B)."""
    n, dk = q.shape
    b = np.cumsum(lg, axis=0)
    B, r = b[-1], b[ref_row(n, where)]
    x = np.exp2(r - b)
    Kt = k * x
    Qt = q / x / math.sqrt(dk)
    O = np.tril(Qt @ Kt.T) @ v + Qt @ (np.exp2(r)[:, None] * S_in)
    S_out = np.exp2(B)[:, None] * S_in + (k * np.exp2(B - b)).T @ v
    return O, S_out, B


def segmented_scan(q, k, v, lg, chunk, segs, chunk_fn, exchange_rnd=None):
    """A scan in scan order cut into `segs` equal segments of chunks: a state-only pass per
    segment, the (G, S) combine across segments, then the full pass.  `exchange_rnd`, if
    given, rounds the states exchanged in both directions and the combine runs in fp32."""
    L, dk = q.shape
    dv = v.shape[1]
    seg_len = -(-L // segs)
    bounds = [(s0, min(L, s0 + seg_len)) for s0 in range(0, L, seg_len)]

    def run(s0, s1, S):
        outs, G = [], np.zeros(dk)
        for c0 in range(s0, s1, chunk):
            c1 = min(s1, c0 + chunk)
            O, S, B = chunk_fn(q[c0:c1], k[c0:c1], v[c0:c1], lg[c0:c1], S)
            outs.append(O)
            G = G + B
        return np.concatenate(outs), S, G

    incoming, S_in = [], np.zeros((dk, dv))
    for s0, s1 in bounds:
        _, S_agg, G = run(s0, s1, np.zeros((dk, dv)))
        if exchange_rnd is None:
            incoming.append(S_in)
            S_in = np.exp2(G)[:, None] * S_in + S_agg
        else:
            incoming.append(exchange_rnd(S_in))
            S_in = f32(np.exp2(G)[:, None] * S_in + exchange_rnd(S_agg))
    return np.concatenate([run(s0, s1, S0)[0] for (s0, s1), S0 in zip(bounds, incoming)])


def chunkwise_o(q, k, v, a, gh, gw, direction, chunk, segs, chunk_fn, exchange_rnd=None):
    """o for every (b, h) pair, gathered in scan order and written back in spatial order."""
    B, L, H, _ = q.shape
    o = np.zeros(v.shape)
    lg = log2_gate(a)
    for bi in range(B):
        perm = scan_perm(direction, gh, gw)
        for h in range(H):
            o[bi, perm, h] = segmented_scan(q[bi, perm, h], k[bi, perm, h], v[bi, perm, h],
                                            lg[bi, perm, h], chunk, segs, chunk_fn, exchange_rnd)
    return o


def lookback_scan(q, k, v, lg, chunk, segs, chunk_fn):
    """The segment scan with every segment combining all earlier aggregates itself instead of
    receiving a running state: S_in(s) = sum_{j<s} Diag(2^{G_{j+1} + ... + G_{s-1}}) S_agg(j)
    -- the form a grid-wide exchange through a workspace would take, where all aggregates are
    published at once and no segment waits for its predecessor's combine."""
    L, dk = q.shape
    dv = v.shape[1]
    seg_len = -(-L // segs)
    bounds = [(s0, min(L, s0 + seg_len)) for s0 in range(0, L, seg_len)]

    def run(s0, s1, S):
        outs, G = [], np.zeros(dk)
        for c0 in range(s0, s1, chunk):
            c1 = min(s1, c0 + chunk)
            O, S, B = chunk_fn(q[c0:c1], k[c0:c1], v[c0:c1], lg[c0:c1], S)
            outs.append(O)
            G = G + B
        return np.concatenate(outs), S, G

    aggs = [run(s0, s1, np.zeros((dk, dv)))[1:] for s0, s1 in bounds]     # (S_agg, G) each
    outs = []
    for s, (s0, s1) in enumerate(bounds):
        S_in = np.zeros((dk, dv))
        for j in range(s):
            decay = np.sum([aggs[i][1] for i in range(j + 1, s)], axis=0) if j + 1 < s else np.zeros(dk)
            S_in = S_in + np.exp2(decay)[:, None] * aggs[j][0]
        outs.append(run(s0, s1, S_in)[0])
    return np.concatenate(outs)


@pytest.mark.parametrize("direction", [0, 3])
def test_lookback_combine_with_eighteen_segments_is_exact(direction):
    rng = np.random.default_rng(11)
    gh, gw = 24, 30                                  # 720 tokens: 18 segments of 40
    q, k, v, a, g, w = rand_inputs(rng, 1, gh, gw, 1, 32, 24, a_mean=0.0, a_std=3.0)
    _, o_ref = oracle.gla_forward(q, k, v, a, g, w, gh, gw, direction, return_o=True)
    lg = log2_gate(a)
    perm = scan_perm(direction, gh, gw)
    fn = lambda *t: chunk_exact(*t, where="middle")   # noqa: E731
    o = np.zeros(v.shape)
    o[0, perm, 0] = lookback_scan(q[0, perm, 0], k[0, perm, 0], v[0, perm, 0], lg[0, perm, 0], 16, 18, fn)
    assert np.max(np.abs(o - o_ref)) <= 1e-12 * max(1.0, np.max(np.abs(o_ref)))


@pytest.mark.parametrize("direction", [0, 1, 2, 3])
@pytest.mark.parametrize("chunk,segs,where", [(16, 1, "middle"), (32, 3, "first"),
                                              (64, 16, "middle"), (100, 5, "last"),
                                              (128, 2, "middle"), (32, 7, "middle")])
def test_factorised_form_is_exact(direction, chunk, segs, where):
    # (32, 7): segments of 35 tokens (two chunks) and a last one of 30 (one chunk)
    rng = np.random.default_rng(7)
    gh, gw = 12, 20
    q, k, v, a, g, w = rand_inputs(rng, 1, gh, gw, 2, 32, 24, a_mean=0.0, a_std=3.0)
    _, o_ref = oracle.gla_forward(q, k, v, a, g, w, gh, gw, direction, return_o=True)
    fn = lambda *t: chunk_exact(*t, where=where)   # noqa: E731
    o = chunkwise_o(q, k, v, a, gh, gw, direction, chunk, segs, fn)
    assert np.max(np.abs(o - o_ref)) <= 1e-12 * max(1.0, np.max(np.abs(o_ref)))


def test_decays_on_the_state_side_never_exceed_one():
    # every exponent the state update and the inter operand use is <= 0 (no overflow)
    rng = np.random.default_rng(3)
    for a_mean, a_std in ((2.0, 1.0), (0.0, 3.0), (-30.0, 1.0)):
        lg = log2_gate(rng.standard_normal((128, 64)) * a_std + a_mean)
        b = np.cumsum(lg, axis=0)
        B, r = b[-1], b[64]
        assert np.all(B - b <= 0) and np.all(r <= 0) and np.all(B <= 0)
        # the score operands carry exponents of either sign, bounded by the chunk's
        # half-range about the middle row
        half = np.maximum(b[0] - r, r - B)
        assert np.all(np.abs(r - b) <= half + 1e-12)


# ---- the kernel's precision plan, emulated ------------------------------------------
def tf32(x):
    """What the tensor core reads from an fp32 operand: the low 13 mantissa bits cleared."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32) & np.uint32(0xFFFFE000)
    return u.view(np.float32).astype(np.float64)


def f32(x):
    return np.asarray(x, dtype=np.float32).astype(np.float64)


def f16(x):
    return np.asarray(x, dtype=np.float16).astype(np.float64)


def chunk_rounded(q, k, v, lg, S_in, split=True):
    """One chunk with the kernel's rounding points (fp32 accumulation emulated by one
    rounding of each fp64 product sum, which is closer than any real accumulation order)."""
    n, dk = q.shape
    lg = f32(lg)
    b = np.cumsum(lg.astype(np.float32), axis=0).astype(np.float64)
    B, r = b[-1], b[n // 2]
    x = f32(np.exp2(r - b))
    Kt = f32(k * x)
    Qt = f32(q * f32(1.0 / x) / math.sqrt(dk))
    Kh, Qh = tf32(Kt), tf32(Qt)
    if split:
        Kl, Ql = tf32(Kt - Kh), tf32(Qt - Qh)
        A = f32(Qh @ Kh.T + Qh @ Kl.T + Ql @ Kh.T)
        np.fill_diagonal(A, f32(np.sum(q * k, axis=1) / math.sqrt(dk)))
        Qop = Qh + Ql
    else:
        A = f32(Qh @ Kh.T)
        Qop = Qh
    P = f16(np.tril(A))
    S_t = tf32(f32(np.exp2(r)[:, None] * S_in))
    O = f32(P @ v) + f32(Qop @ S_t)
    Ks = f16(k * f32(np.exp2(B - b)))
    S_out = f32(f32(np.exp2(B)[:, None] * S_in) + f32(Ks.T @ v))
    return O, S_out, B


def epilogue_f16(o, g, w):
    o = f32(o)
    n = f32(o / np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + EPS) * w)
    return f16(n * f32(g / (1.0 + np.exp(-g))))


def errors(u, ref):
    return float(np.max(np.abs(u - ref))), float(np.linalg.norm(u - ref) / np.linalg.norm(ref))


@pytest.mark.parametrize("direction", [0, 2])
def test_precision_plan_meets_the_fp16_tolerance(direction):
    # the 40x40 shape as the kernel runs it: 16 segments of one 100-token chunk each
    from recurrent_vision_backbone_only_b200 import synth
    wl = synth.WORKLOADS["gtr640"].with_(H=2)
    x = {n: t.astype(np.float64) for n, t in synth.make_inputs(wl, seed=0).items()}
    ref = oracle.gla_forward(x["q"], x["k"], x["v"], x["a"], x["g"], x["w"],
                             wl.grid_h, wl.grid_w, direction)
    o = chunkwise_o(x["q"], x["k"], x["v"], x["a"], wl.grid_h, wl.grid_w, direction,
                    128, 16, chunk_rounded)
    max_abs, rel = errors(epilogue_f16(o, x["g"], x["w"]), ref)
    assert max_abs <= 1e-2 and rel <= 2e-3, (max_abs, rel)


def test_single_tf32_scores_miss_the_tolerance_where_the_split_meets_it():
    # a first token whose readout q.k nearly cancels: o_0 = (q_0 . k_0) v_0 / 8 is small,
    # RMSNorm rescales it to O(1), and the relative error of q_0 . k_0 carries through
    rng = np.random.default_rng(11)
    gh, gw, d = 1, 64, 64
    q, k, v, a, g, w = rand_inputs(rng, 1, gh, gw, 1, d, d, a_mean=2.0, a_std=1.0,
                                   scale=1 / math.sqrt(2))
    q0, k0 = q[0, 0, 0], k[0, 0, 0]
    k0[-1] -= np.dot(q0, k0) / q0[-1]              # q_0 . k_0 = 0 before rounding
    q, k, v, a, g = (f16(t) for t in (q, k, v, a, g))
    w = f32(w)
    ref = oracle.gla_forward(q, k, v, a, g, w, gh, gw, 0)
    res = {}
    for split in (True, False):
        fn = lambda *t, s=split: chunk_rounded(*t, split=s)   # noqa: E731
        o = chunkwise_o(q, k, v, a, gh, gw, 0, 64, 1, fn)
        res[split] = errors(epilogue_f16(o, g, w), ref)[0]
    assert res[True] <= 1e-2, res
    assert res[False] > 1e-2, res


def _mutant(kind):
    def fn(q, k, v, lg, S_in):
        n, dk = q.shape
        b = np.cumsum(lg, axis=0) - (lg if kind == "exclusive decay" else 0.0)
        B, r = b[-1], b[n // 2]
        x = np.exp2(r - b)
        Qt, Kt = q / x / math.sqrt(dk), k * x
        O = np.tril(Qt @ Kt.T, -1 if kind == "strict mask" else 0) @ v
        if kind != "no inter term":
            O = O + Qt @ (np.exp2(r)[:, None] * S_in)
        return O, np.exp2(B)[:, None] * S_in + (k * np.exp2(B - b)).T @ v, B
    return fn


@pytest.mark.parametrize("kind", ["no inter term", "exclusive decay", "strict mask"])
def test_broken_factorisations_are_caught(kind):
    rng = np.random.default_rng(7)
    q, k, v, a, g, w = rand_inputs(rng, 1, 12, 20, 2, 32, 24, a_mean=0.0, a_std=3.0)
    _, o_ref = oracle.gla_forward(q, k, v, a, g, w, 12, 20, 1, return_o=True)
    o = chunkwise_o(q, k, v, a, 12, 20, 1, 32, 3, _mutant(kind))
    assert np.max(np.abs(o - o_ref)) > 1.0


# ---- a candidate plan with 16-bit operands, weighed the same way -----------------------
def bf16(x):
    """Round to bfloat16 (nearest even), returned as fp64."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def split(x, rnd):
    """High part and remainder, each rounded by `rnd`, summed (what two products see)."""
    hi = rnd(x)
    return hi + rnd(x - hi)


def chunk_candidate(q, k, v, lg, S_in, scores="split_bf16"):
    """Every product as kind::f16: scores from split bf16 Q~/K~ (same 8-bit exponent as
    tf32) with the exact fp32 diagonal; the inter product as split fp16(q 2^b / sqrt(d_k))
    against fp16 S_in (every exponent <= 0, so fp16 suffices), chained into P.V's
    accumulator."""
    n, dk = q.shape
    b = np.cumsum(f32(lg).astype(np.float32), axis=0).astype(np.float64)
    B, r = b[-1], b[n // 2]
    x = f32(np.exp2(r - b))
    Kt = f32(k * x)
    Qt = f32(q * f32(1.0 / x) / math.sqrt(dk))
    if scores == "split_bf16":
        Kh, Qh = bf16(Kt), bf16(Qt)
        A = f32(Qh @ Kh.T + Qh @ bf16(Kt - Kh).T + bf16(Qt - Qh) @ Kh.T)
    else:                                          # one tf32 operand per side
        A = f32(tf32(Qt) @ tf32(Kt).T)
    np.fill_diagonal(A, f32(np.sum(q * k, axis=1) / math.sqrt(dk)))
    Qi = split(f32(q * f32(np.exp2(b)) / math.sqrt(dk)), f16)
    O = f32(f16(np.tril(A)) @ v + Qi @ f16(S_in))
    Ks = f16(k * f32(np.exp2(B - b)))
    S_out = f32(f32(np.exp2(B)[:, None] * S_in) + f32(Ks.T @ v))
    return O, S_out, B


def worst_error(name, directions, segs, chunk_fn, exchange_rnd=None):
    from recurrent_vision_backbone_only_b200 import synth
    wl = synth.WORKLOADS[name]
    x = {n: t.astype(np.float64) for n, t in synth.make_inputs(wl, seed=0).items()}
    worst = (0.0, 0.0)
    for direction in directions:
        ref = oracle.gla_forward(x["q"], x["k"], x["v"], x["a"], x["g"], x["w"],
                                 wl.grid_h, wl.grid_w, direction)
        o = chunkwise_o(x["q"], x["k"], x["v"], x["a"], wl.grid_h, wl.grid_w, direction,
                        128, segs, chunk_fn, exchange_rnd)
        e = errors(epilogue_f16(o, x["g"], x["w"]), ref)
        worst = (max(worst[0], e[0]), max(worst[1], e[1]))
    return worst


def test_candidate_plan_with_fp16_states_meets_the_tolerance():
    for name, dirs, segs in (("gtr640", (0, 1, 2, 3), 16), ("highres", (0,), 10)):
        max_abs, rel = worst_error(name, dirs, segs, chunk_candidate, exchange_rnd=f16)
        assert max_abs <= 6e-3 and rel <= 4e-4, (name, max_abs, rel)


def test_bf16_states_miss_the_tolerance():
    max_abs, _ = worst_error("gtr640", (0, 1, 2, 3), 16, chunk_rounded, exchange_rnd=bf16)
    assert max_abs > 1e-2, max_abs


def test_single_operand_scores_miss_the_tolerance_on_80x80():
    # the exact diagonal alone does not rescue one tf32 operand per side: cancelling
    # readouts later in the scan still lose digits
    single = worst_error("highres", (0,), 10, lambda *t: chunk_candidate(*t, scores="tf32"))
    both = worst_error("highres", (0,), 10, chunk_candidate)
    assert single[0] > 1e-2 and both[0] <= 6e-3, (single, both)
