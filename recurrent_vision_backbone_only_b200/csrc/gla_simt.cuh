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

__host__ __device__ constexpr size_t simt_smem_floats(int dk, int dv, int C) {
    return (size_t)dk * dv + dk + 3 * (size_t)C * dk + 2 * (size_t)C * dv + (size_t)C * C + C;
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
    float *qs = G + DK;          // [C][DK]
    float *ks = qs + C * DK;     // [C][DK]
    float *bs = ks + C * DK;     // [C][DK] in-chunk cumulative log-decay
    float *vs = bs + C * DK;     // [C][DV]
    float *Os = vs + C * DV;     // [C][DV]
    float *As = Os + C * DV;     // [C][C] decay-weighted scores
    int *rows = reinterpret_cast<int *>(As + C * C);  // [C] token row index (b*L+s)*H+h

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
    auto load_chunk = [&](int c0, int n, bool with_q) {
        __syncthreads();
        for (int t = tid; t < n; t += NT)
            rows[t] = (b * p.L + spatial_of(dir, c0 + t, p.gh, p.gw)) * p.H + h;
        __syncthreads();
        for (int idx = tid; idx < n * DK; idx += NT) {
            const int t = idx / DK, c = idx - t * DK;
            const size_t off = (size_t)rows[t] * DK + c;
            ks[idx] = to_f32(k[off]);
            bs[idx] = log_gamma(to_f32(a[off]));
            if (with_q) qs[idx] = to_f32(q[off]);
        }
        for (int idx = tid; idx < n * DV; idx += NT) {
            const int t = idx / DV, j = idx - t * DV;
            vs[idx] = to_f32(v[(size_t)rows[t] * DV + j]);
        }
        __syncthreads();
        for (int c = tid; c < DK; c += NT) {
            float run = 0.0f;
            for (int t = 0; t < n; ++t) {
                run += bs[t * DK + c];
                bs[t * DK + c] = run;
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
            const float dec = expf(bs[(n - 1) * DK + c0 + a]);
#pragma unroll
            for (int b2 = 0; b2 < TJ; ++b2) acc[a][b2] = S[(c0 + a) * DV + j0 + b2] * dec;
        }
        for (int s = 0; s < n; ++s) {
            float kr[TC], vr[TJ];
            load_run<TC>(ks + s * DK + c0, kr);
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
        for (int c = tid; c < DK; c += NT) G[c] += bs[(n - 1) * DK + c];
    };

    auto scale_keys = [&](int n) {
        for (int idx = tid; idx < n * DK; idx += NT) {
            const int c = idx % DK;
            ks[idx] *= expf(bs[(n - 1) * DK + c] - bs[idx]);
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
                const float *qt = qs + t * DK, *bt = bs + t * DK;
                const float *kk = ks + s * DK, *bb = bs + s * DK;
                for (int c = 0; c < DK; ++c) acc = fmaf(qt[c] * kk[c], expf(bt[c] - bb[c]), acc);
            }
            As[t * C + s] = acc;
        }
        __syncthreads();
        // q_t (.) e^{b_t} for the inter-chunk term; k_s (.) e^{b_last - b_s} for the state
        for (int idx = tid; idx < n * DK; idx += NT) qs[idx] *= expf(bs[idx]);
        scale_keys(n);
        __syncthreads();
        // O[t][j] = scale (sum_{s<=t} A[t][s] v_s[j] + sum_c q~_t[c] S[c][j]); register-blocked
        // over 4 value columns and the tokens t = tg, tg + TS, ... of one thread, so each
        // loaded S row piece serves every token of the thread; each output still accumulates
        // in the order s = 0..t, then c = 0..DK-1
        {
            constexpr int JG = DV / 4, TS = NT / JG, MT = (64 + TS - 1) / TS;
            const int j0 = (tid % JG) * 4, tg = tid / JG;
            float acc[MT][4];
#pragma unroll
            for (int i = 0; i < MT; ++i)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[i][e] = 0.0f;
#pragma unroll
            for (int i = 0; i < MT; ++i) {
                const int t = tg + i * TS;
                if (t < n) {
                    for (int s = 0; s <= t; ++s) {
                        const float a_ts = As[t * C + s];
#pragma unroll
                        for (int e = 0; e < 4; ++e) acc[i][e] = fmaf(a_ts, vs[s * DV + j0 + e], acc[i][e]);
                    }
                }
            }
            for (int c = 0; c < DK; ++c) {
                const float4 sr = *reinterpret_cast<const float4 *>(S + c * DV + j0);
#pragma unroll
                for (int i = 0; i < MT; ++i) {
                    const int t = tg + i * TS;
                    if (t < n) {
                        const float qv = qs[t * DK + c];
                        acc[i][0] = fmaf(qv, sr.x, acc[i][0]);
                        acc[i][1] = fmaf(qv, sr.y, acc[i][1]);
                        acc[i][2] = fmaf(qv, sr.z, acc[i][2]);
                        acc[i][3] = fmaf(qv, sr.w, acc[i][3]);
                    }
                }
            }
#pragma unroll
            for (int i = 0; i < MT; ++i) {
                const int t = tg + i * TS;
                if (t < n) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) Os[t * DV + j0 + e] = acc[i][e] * p.scale;
                }
            }
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
                const float u = ot[j] * inv * p.w[j] * silu(to_f32(g[base + j]));
                out[base + j] = from_f32<T>(u);
            }
        }
    }
}

}  // namespace gla
