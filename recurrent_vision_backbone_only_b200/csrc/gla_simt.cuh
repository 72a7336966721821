// gla_simt.cuh -- exact fp32 CUDA-core kernel for the key-only GLA mixer.
//
// Serves gla_fwd_f32 (float32 I/O, the tight-tolerance path) and, templated on
// the I/O type, is the plain reference schedule the tensor-core kernel is
// compared against.  All arithmetic is fp32 on CUDA cores.
//
// Math (GTR paper, arXiv 2609.26590, method section, GLA recurrence): for
// one (b, h) pair, split the scan into chunks of C tokens.  With
// lambda_t = log sigma(a_t) / 16 and the in-chunk inclusive cumulative sum
// b_t = sum_{chunk start <= j <= t} lambda_j (per key channel), the exact
// chunkwise form of S_t = Diag(gamma_t) S_{t-1} + k_t^T v_t is
//   o_t   = d_k^{-1/2} [ sum_{s<=t in chunk} (sum_c q_tc k_sc e^{b_tc-b_sc}) v_s
//                        + (q_t (.) e^{b_t}) S_in ]
//   S_out = Diag(e^{b_last}) S_in + sum_s (k_s (.) e^{b_last - b_s})^T v_s
// Every exponent above is <= 0, so nothing overflows for any gate value; the
// intra-chunk scores take one exp per (t, s, c), which is what makes this
// kernel exact and slow.
//
// Parallel schedule: a (b, h) pair's scan is cut into `segs` contiguous
// segments, one CTA each, forming one thread-block cluster.  Pass 1: every
// CTA but the last folds its segment into (G, S_agg) = (total log-decay,
// state from a zero start).  The cluster then scans those aggregates through
// distributed shared memory, each CTA owning a slice of the d_k x d_v state
// elements (the combine (G2,S2) o (G1,S1) = (G1+G2, Diag(e^{G2}) S1 + S2) is
// elementwise per state entry), and writes every segment's incoming state
// back into that segment's CTA.  Pass 2 runs the chunkwise form above from
// the incoming state and writes u.
#pragma once

#include <cooperative_groups.h>

#include "gla_common.cuh"

namespace gla {

namespace cg = cooperative_groups;

struct SimtParams {
    const void *q, *k, *v, *a, *g;
    const float *w;
    void *out;
    int B, H, gh, gw, L;
    int dir;        // 0..4
    int chunk;      // tokens per chunk (C)
    int segs;       // CTAs per (b, h) pair == cluster size
    int seg_len;    // tokens per segment (multiple of C)
    float eps;
    float scale;    // d_k^{-1/2}
};

constexpr int kSimtThreads = 256;

// q, k and b rows are padded to d_k + 4 floats: 16-byte aligned, and rows of different
// tokens fall in different shared-memory banks (the score loop reads one channel of 16 rows)
__host__ __device__ constexpr int simt_row(int dk) { return dk + 4; }

__host__ __device__ constexpr size_t simt_smem_floats(int dk, int dv, int C) {
    return (size_t)dk * dv + dk + 3 * (size_t)C * simt_row(dk) + 3 * (size_t)C * dv + (size_t)C * C + C;
}

// N consecutive floats from shared memory (N = 2, 4 or 8; p aligned to min(N, 4) floats)
template <int N>
__device__ __forceinline__ void load_run(const float *p, float *out) {
    if constexpr (N == 2) {
        const float2 v = *reinterpret_cast<const float2 *>(p);
        out[0] = v.x; out[1] = v.y;
    } else {
#pragma unroll
        for (int q = 0; q < N / 4; ++q) {
            const float4 v = *reinterpret_cast<const float4 *>(p + 4 * q);
            out[4 * q] = v.x; out[4 * q + 1] = v.y; out[4 * q + 2] = v.z; out[4 * q + 3] = v.w;
        }
    }
}

template <typename T, int DK, int DV>
__global__ void __launch_bounds__(kSimtThreads, 2)
gla_simt_kernel(const SimtParams p) {
    constexpr int NT = kSimtThreads;
    constexpr int NW = NT / 32;
    const int C = p.chunk;
    extern __shared__ float smem[];
    float *S = smem;             // [DK][DV] running state / aggregate / incoming state
    float *G = S + DK * DV;      // [DK] segment log-decay
    constexpr int KP = simt_row(DK);   // padded row of q, k, b
    float *qs = G + DK;          // [C][KP]
    float *ks = qs + C * KP;     // [C][KP]
    float *bs = ks + C * KP;     // [C][KP] in-chunk cumulative log-decay
    float *vs = bs + C * KP;     // [C][DV]
    float *Os = vs + C * DV;     // [C][DV]
    float *As = Os + C * DV;     // [C][C] decay-weighted scores
    float *gsm = As + C * C;     // [C][DV] output-gate pre-activation
    int *rows = reinterpret_cast<int *>(gsm + C * DV);  // [C] token row index (b*L+s)*H+h

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int pair = blockIdx.x / p.segs;
    const int rank = blockIdx.x - pair * p.segs;
    const int b = pair / p.H, h = pair - b * p.H;
    const int dir = p.dir == 4 ? (b & 3) : p.dir;
    const int p0 = min(p.L, rank * p.seg_len);
    const int p1 = min(p.L, p0 + p.seg_len);

    const T *q = static_cast<const T *>(p.q);
    const T *k = static_cast<const T *>(p.k);
    const T *v = static_cast<const T *>(p.v);
    const T *a = static_cast<const T *>(p.a);
    const T *g = static_cast<const T *>(p.g);
    T *out = static_cast<T *>(p.out);

    for (int e = tid; e < DK * DV; e += NT) S[e] = 0.0f;
    for (int c = tid; c < DK; c += NT) G[c] = 0.0f;

    // Gather the chunk [c0, c0+n) in scan order; b = inclusive cumsum of lambda.
    // Inputs move in 16-byte pieces: EPP elements, PK (PV) pieces per key (value) row.  Each
    // batch of pieces is loaded into registers before any is consumed, so a batch costs one
    // DRAM round trip (global loads cannot be reordered past the shared-memory stores).
    constexpr int EPP = 16 / (int)sizeof(T);
    constexpr int PK = DK / EPP, PV = DV / EPP;
    auto unpack = [&](const uint4 &r, float *o) {
        if constexpr (sizeof(T) == 2) {
            const __half2 *h2 = reinterpret_cast<const __half2 *>(&r);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __half22float2(h2[e]);
                o[2 * e] = f.x;
                o[2 * e + 1] = f.y;
            }
        } else {
            const float *f = reinterpret_cast<const float *>(&r);
#pragma unroll
            for (int e = 0; e < 4; ++e) o[e] = f[e];
        }
    };
    auto ld16 = [](const T *ptr) { return *reinterpret_cast<const uint4 *>(ptr); };
    auto load_chunk = [&](int c0, int n, bool with_q) {
        __syncthreads();
        for (int t = tid; t < n; t += NT) {
            const int r = (b * p.L + spatial_of(dir, c0 + t, p.gh, p.gw)) * p.H + h;
            rows[t] = GLA_CHECK(c0 + t < p.L && r >= 0 && r < p.B * p.L * p.H) ? r : 0;
        }
        __syncthreads();
        for (int base = 0; base < n * PK; base += NT) {
            const int pi = base + tid;
            if (pi < n * PK) {
                const int t = pi / PK, pc = pi - t * PK;
                const size_t off = (size_t)rows[t] * DK + pc * EPP;
                const uint4 kr = ld16(k + off), ar = ld16(a + off);
                const uint4 qr = with_q ? ld16(q + off) : make_uint4(0, 0, 0, 0);
                float kf[EPP], af[EPP], qf[EPP];
                unpack(kr, kf);
                unpack(ar, af);
                unpack(qr, qf);
                const int o = t * KP + pc * EPP;
#pragma unroll
                for (int e = 0; e < EPP; ++e) {
                    ks[o + e] = kf[e];
                    bs[o + e] = log_gamma(af[e]);
                    if (with_q) qs[o + e] = qf[e];
                }
            }
        }
        for (int base = 0; base < n * PV; base += NT) {
            const int pi = base + tid;
            if (pi < n * PV) {
                const int t = pi / PV, pc = pi - t * PV;
                const size_t off = (size_t)rows[t] * DV + pc * EPP;
                const uint4 vr = ld16(v + off);
                const uint4 gr = with_q ? ld16(g + off) : make_uint4(0, 0, 0, 0);
                float vf[EPP], gf[EPP];
                unpack(vr, vf);
                unpack(gr, gf);
                const int o = t * DV + pc * EPP;
#pragma unroll
                for (int e = 0; e < EPP; ++e) {
                    vs[o + e] = vf[e];
                    if (with_q) gsm[o + e] = gf[e];
                }
            }
        }
        __syncthreads();
        for (int c = tid; c < DK; c += NT) {
            float run = 0.0f;
            for (int t = 0; t < n; ++t) {
                run += bs[t * KP + c];
                bs[t * KP + c] = run;
            }
        }
        __syncthreads();
    };

    // S <- Diag(e^{b_last}) S + sum_s (k_s (.) e^{b_last - b_s})^T v_s ; G += b_last.
    // ks must already hold k_s (.) e^{b_last - b_s}.  Register-blocked: a 16 x 16 thread grid,
    // each thread a (DK/16) x (DV/16) tile of S, so every loaded k and v value feeds a row or
    // column of FMAs.  Each entry still accumulates in the order S e^{b}, s = 0, 1, ...
    auto fold_state = [&](int n) {
        constexpr int TC = DK / 16, TJ = DV / 16;
        const int c0 = (tid >> 4) * TC, j0 = (tid & 15) * TJ;
        float acc[TC][TJ];
#pragma unroll
        for (int a = 0; a < TC; ++a) {
            const float dec = expf(bs[(n - 1) * KP + c0 + a]);
#pragma unroll
            for (int b2 = 0; b2 < TJ; ++b2) acc[a][b2] = S[(c0 + a) * DV + j0 + b2] * dec;
        }
        for (int s = 0; s < n; ++s) {
            float kr[TC], vr[TJ];
            load_run<TC>(ks + s * KP + c0, kr);
            load_run<TJ>(vs + s * DV + j0, vr);
#pragma unroll
            for (int a = 0; a < TC; ++a)
#pragma unroll
                for (int b2 = 0; b2 < TJ; ++b2) acc[a][b2] = fmaf(kr[a], vr[b2], acc[a][b2]);
        }
#pragma unroll
        for (int a = 0; a < TC; ++a)
#pragma unroll
            for (int b2 = 0; b2 < TJ; ++b2) S[(c0 + a) * DV + j0 + b2] = acc[a][b2];
        for (int c = tid; c < DK; c += NT) G[c] += bs[(n - 1) * KP + c];
    };

    auto scale_keys = [&](int n) {
        for (int idx = tid; idx < n * DK; idx += NT) {
            const int t = idx / DK, c = idx - t * DK;
            ks[t * KP + c] *= expf(bs[(n - 1) * KP + c] - bs[t * KP + c]);
        }
    };

    // ---- pass 1: segment aggregates (not needed for the last segment) ----
    if (p.segs > 1) {
        if (rank < p.segs - 1) {
            for (int c0 = p0; c0 < p1; c0 += C) {
                const int n = min(C, p1 - c0);
                load_chunk(c0, n, false);
                scale_keys(n);
                __syncthreads();
                fold_state(n);
            }
        }
        // ---- cluster scan of (G, S_agg) -> incoming state per segment ----
        cg::cluster_group cluster = cg::this_cluster();
        cluster.sync();
        const int E = DK * DV;
        const int per = (E + p.segs - 1) / p.segs;
        const int e0 = rank * per, e1 = min(E, e0 + per);
        for (int e = e0 + tid; e < e1; e += NT) {
            const int c = e / DV;
            float run = 0.0f;
            for (int r = 0; r < p.segs; ++r) {
                float *Sr = cluster.map_shared_rank(S, r);
                const float *Gr = cluster.map_shared_rank(G, r);
                const float agg = Sr[e];
                const float dec = expf(Gr[c]);
                Sr[e] = run;                      // state entering segment r
                run = fmaf(dec, run, agg);
            }
        }
        cluster.sync();
    }
    __syncthreads();

    // ---- pass 2: outputs from the incoming state ----
    for (int c0 = p0; c0 < p1; c0 += C) {
        const int n = min(C, p1 - c0);
        load_chunk(c0, n, true);
        // intra-chunk decay-weighted scores, exact per (t, s, c)
        for (int idx = tid; idx < n * n; idx += NT) {
            const int t = idx / n, s = idx - t * n;
            float acc = 0.0f;
            if (s <= t) {
                const float *qt = qs + t * KP, *bt = bs + t * KP;
                const float *kk = ks + s * KP, *bb = bs + s * KP;
                for (int c = 0; c < DK; ++c) acc = fmaf(qt[c] * kk[c], expf(bt[c] - bb[c]), acc);
            }
            As[t * C + s] = acc;
        }
        __syncthreads();
        // q_t (.) e^{b_t} for the inter-chunk term; k_s (.) e^{b_last - b_s} for the state
        for (int idx = tid; idx < n * DK; idx += NT) {
            const int t = idx / DK, c = idx - t * DK;
            qs[t * KP + c] *= expf(bs[t * KP + c]);
        }
        scale_keys(n);
        __syncthreads();
        // O[t][j] = scale (sum_{s<=t} A[t][s] v_s[j] + sum_c q~_t[c] S[c][j]), 4 value columns
        // per work item; each output accumulates in the order s = 0..t, then c = 0..DK-1
        for (int w = tid; w < n * (DV / 4); w += NT) {
            const int t = w / (DV / 4), j0 = (w - t * (DV / 4)) * 4;
            float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            for (int s = 0; s <= t; ++s) {
                const float a_ts = As[t * C + s];
                const float4 vr = *reinterpret_cast<const float4 *>(vs + s * DV + j0);
                acc = make_float4(fmaf(a_ts, vr.x, acc.x), fmaf(a_ts, vr.y, acc.y),
                                  fmaf(a_ts, vr.z, acc.z), fmaf(a_ts, vr.w, acc.w));
            }
            const float *qt = qs + t * KP;
#pragma unroll 4
            for (int c = 0; c < DK; ++c) {
                const float qv = qt[c];
                const float4 sr = *reinterpret_cast<const float4 *>(S + c * DV + j0);
                acc = make_float4(fmaf(qv, sr.x, acc.x), fmaf(qv, sr.y, acc.y),
                                  fmaf(qv, sr.z, acc.z), fmaf(qv, sr.w, acc.w));
            }
            *reinterpret_cast<float4 *>(Os + t * DV + j0) =
                make_float4(acc.x * p.scale, acc.y * p.scale, acc.z * p.scale, acc.w * p.scale);
        }
        __syncthreads();
        fold_state(n);
        // epilogue: u = SiLU(g) * o / sqrt(mean(o^2) + eps) * w, one warp per token
        for (int t = warp; t < n; t += NW) {
            const float *ot = Os + t * DV;
            float ss = 0.0f;
            for (int j = lane; j < DV; j += 32) ss = fmaf(ot[j], ot[j], ss);
            for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
            const float inv = 1.0f / sqrtf(ss / DV + p.eps);
            const size_t base = (size_t)rows[t] * DV;
            for (int j = lane; j < DV; j += 32) {
                const float u = ot[j] * inv * p.w[j] * silu(gsm[t * DV + j]);
                out[base + j] = from_f32<T>(u);
            }
        }
    }
}

}  // namespace gla
