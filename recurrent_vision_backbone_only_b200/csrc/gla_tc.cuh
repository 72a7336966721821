// gla_tc.cuh -- tensor-core (tcgen05 / TMEM) kernel for the key-only GLA
// token mixer, fp16 I/O, head dims d_k = d_v = 64.
//
// Operation (GTR paper, arXiv 2609.26590, method section): per (b, h) pair,
// over the scan order of one of four directions,
//   S_t = Diag(gamma_t) S_{t-1} + k_t^T v_t, o_t = d_k^{-1/2} q_t S_t,
//   gamma_t = sigma(a_t)^(1/16), u_t = SiLU(g_t) * RMSNorm(o_t) * w,
// written back at each token's spatial position.
//
// Chunkwise form used here.  A chunk holds n <= 128 consecutive scan
// positions; b_t is the inclusive in-chunk cumulative sum of
// lambda_t = log sigma(a_t) / 16 (per key channel), B = b_{n-1}, and r is a
// per-channel reference (the chunk's middle row).  With Q~ = q (.) e^{b - r},
// K~ = k (.) e^{r - b}, Ks = k (.) e^{B - b} and the state S_in entering the
// chunk:
//   scores   A     = Q~ K~^T   split-tf32: Qh Kh^T + Qh Kl^T + Ql Kh^T, where
//                    X = Xh + Xl with Xh = tf32(X), Xl = tf32(X - Xh)
//                    (tcgen05 kind::tf32, A operands Qh/Ql in TMEM, 128x128x64)
//   masked   P     = d_k^{-1/2} A (.) [s <= t], diagonal A_tt = q_t . k_t in fp32
//   output   O     = P V + Qh (d_k^{-1/2} Diag(e^{r}) S_in)  (f16 + tf32 MMAs)
//   state    S_out = Diag(e^{B}) S_in + Ks^T V       (tcgen05 kind::f16, 64x64x128)
// Every exponent in Ks, e^{r}, e^{B} is <= 0.  Q~ and K~ carry exponents of
// either sign bounded by the chunk's decay range about r; they are kept in
// fp32-range operands (tf32: 8-bit exponent), which holds any chunk whose
// half-range is <= 60 nats.  A chunk beyond that (gates below about -100 on
// several tokens) switches to an exact CUDA-core evaluation of P with the
// chunk start as reference (exponents all <= 0).  The split score product
// keeps A to ~2^-21 relative: with single tf32 operands (2^-11), tokens whose
// readout nearly cancels -- e.g. a scan's first token with q.k ~ 0, where the
// RMSNorm epsilon makes u depend on |o| -- lose their leading digits.
//
// Schedule.  A (b, h) scan is cut into `segs` contiguous segments, one CTA
// each, one thread-block cluster per pair.  Segment aggregates
// (G = total log-decay, S from a zero start) are combined across the
// cluster through distributed shared memory, each CTA owning a slice of the
// d_k x d_v state entries (the combine is elementwise per entry), giving
// every segment its incoming state.  A segment that fits one chunk keeps its
// tiles resident and does the exchange mid-chunk; longer segments run a
// state-only pass, the exchange, then the full pass.
//
// Input gathers: 16-byte cp.async per thread, scan row t of the chunk read
// from the token's spatial position (direction remap folded into the
// address), written straight into the 128B-swizzled operand layout.
#pragma once

#include <cooperative_groups.h>

#include "gla_common.cuh"
#include "gla_ptx.cuh"

namespace gla {
namespace tc {

namespace cg = cooperative_groups;

constexpr int kThreads = 128;
constexpr int kC = 128;            // max tokens per chunk (MMA M)
constexpr int kD = 64;             // head dim handled by this kernel
constexpr float kHalfRangeSafe = 60.0f;

// ---- shared memory map (bytes from a 1024-aligned base) ----
constexpr uint32_t kKL = 0;        // K~ low part  tf32, 2 atoms x [128][128B]
constexpr uint32_t kKH = 32768;    // K~ high part tf32, 2 atoms x [128][128B] (slow path: P)
constexpr uint32_t kPB = 65536;    // b   fp32 (QT layout), then P fp16 2 atoms x [128][128B]
constexpr uint32_t kST = 98304;    // Ks fp16 [128][128B] / S~ tf32 2 x [64][128B] / exchange fp32
constexpr uint32_t kTQ = 114688;   // raw tiles, fp16 [128][128B] each
constexpr uint32_t kTK = 131072;
constexpr uint32_t kTA = 147456;
constexpr uint32_t kTV = 163840;
constexpr uint32_t kTG = 180224;
constexpr uint32_t kMISC = 196608;
constexpr uint32_t kAtom128 = 16384;   // [128 rows][128 B]
constexpr uint32_t kAtom64 = 8192;     // [64 rows][128 B]
constexpr size_t kSmemBytes = kMISC + 4096 + 1024;  // + misc + alignment slack

// TMEM columns
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColDS = 0;     // scores, 128 x 128 fp32
constexpr uint32_t kColSL = 128;   // chunk state Ks^T V, M=64 layout
constexpr uint32_t kColO = 192;    // output accumulator 128 x 64
constexpr uint32_t kColQH = 256;   // Q~ high part, tf32 A operand, 128 x 64
constexpr uint32_t kColQL = 320;   // Q~ low part

constexpr uint32_t kIdescQK = ptx::idesc_make(2, false, false, 128, 128);
constexpr uint32_t kIdescST = ptx::idesc_make(0, true, true, 64, 64);
constexpr uint32_t kIdescPV = ptx::idesc_make(0, false, true, 128, 64);
constexpr uint32_t kIdescIN = ptx::idesc_make(2, false, false, 128, 64);

struct Params {
    const __half *q, *k, *v, *a, *g;
    const float *w;
    __half *out;
    int B, H, gh, gw, L, dir;
    int segs;      // CTAs per (b, h) pair == cluster size
    int seg_len;   // scan positions per segment
    int chunk_max; // largest chunk (16..128); a segment is split into equal chunks
    float eps, scale;
};

// ------------------------------------------------------- operand addressing
// tf32 K-major operand, 64 channels = 2 atoms; float4 of channels [4*c4, 4*c4+4).
__device__ __forceinline__ uint32_t off_tf32(uint32_t atom_bytes, uint32_t row, uint32_t c4) {
    return (c4 >> 3) * atom_bytes + ptx::sw128(row, c4 & 7);
}
// fp16 row-major 64-wide tile; 16 B chunk j holds elements [8j, 8j+8).
__device__ __forceinline__ uint32_t off_f16(uint32_t row, uint32_t j) { return ptx::sw128(row, j); }
// fp16 K-major operand with K = 128 (2 atoms): chunk j of K (0..15).
__device__ __forceinline__ uint32_t off_f16k128(uint32_t row, uint32_t j) {
    return (j >> 3) * kAtom128 + ptx::sw128(row, j & 7);
}

// ------------------------------------------------------------ MMA issue (1 thread)
// scores[t][s] = sum_c Q~[t][c] K~[s][c] as Qh Kh^T + Qh Kl^T + Ql Kh^T
__device__ __forceinline__ void issue_qk(uint32_t sbase, uint32_t tmem) {
#pragma unroll
    for (int pass = 0; pass < 3; ++pass) {
        const uint32_t acol = pass == 2 ? kColQL : kColQH;
        const uint32_t bsm = pass == 1 ? kKL : kKH;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const uint32_t koff = (k >> 2) * kAtom128 + (k & 3) * 32;
            ptx::mma_tf32_ts(tmem + kColDS, tmem + acol + 8 * k,
                             ptx::desc_sw128(sbase + bsm + koff, 16, 1024), kIdescQK,
                             pass > 0 || k > 0);
        }
    }
}
// Sloc[c][j] = sum_s Ks[s][c] V[s][j]  (both operands MN-major, K = 128 rows)
__device__ __forceinline__ void issue_state(uint32_t sbase, uint32_t tmem) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        ptx::mma_f16_ss(tmem + kColSL, ptx::desc_sw128(sbase + kST + k * 2048, kAtom128, 1024),
                        ptx::desc_sw128(sbase + kTV + k * 2048, kAtom128, 1024), kIdescST, k > 0);
    }
}
// O[t][j] = sum_s P[t][s] V[s][j]
__device__ __forceinline__ void issue_pv(uint32_t sbase, uint32_t p_base, uint32_t tmem) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const uint32_t koff = (k >> 2) * kAtom128 + (k & 3) * 32;
        ptx::mma_f16_ss(tmem + kColO, ptx::desc_sw128(sbase + p_base + koff, 16, 1024),
                        ptx::desc_sw128(sbase + kTV + k * 2048, kAtom128, 1024), kIdescPV, k > 0);
    }
}
// O[t][j] += sum_c Qh[t][c] S~[j][c]
__device__ __forceinline__ void issue_inter(uint32_t sbase, uint32_t tmem, bool accumulate) {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const uint32_t soff = (k >> 2) * kAtom64 + (k & 3) * 32;
        ptx::mma_tf32_ts(tmem + kColO, tmem + kColQH + 8 * k,
                         ptx::desc_sw128(sbase + kST + soff, 16, 1024), kIdescIN,
                         accumulate || k > 0);
    }
}

// Bounded wait on an mbarrier phase; on expiry latch GLA_ERR_TIMEOUT and return false.
__device__ __forceinline__ bool wait_phase(uint64_t *bar, uint32_t parity) {
    const long long start = clock64();
    while (!ptx::mbar_try_wait(bar, parity)) {
        if (clock64() - start > (1LL << 32)) {
            raise_status(7 /* GLA_ERR_TIMEOUT */);
            return false;
        }
    }
    return true;
}

__device__ __forceinline__ float log_gamma_fast(float a) {
    return (fminf(a, 0.0f) - __logf(1.0f + __expf(-fabsf(a)))) * kInvTau;
}

__device__ __forceinline__ float silu_fast(float g) { return g / (1.0f + __expf(-g)); }

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
    const __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}

// Shared scratch scalars.
struct Misc {
    uint64_t mbar[4];
    uint32_t tmem_base;
    int slow;             // chunk uses the exact CUDA-core score path
    int range_err;        // a P entry overflowed fp16
    int abort;            // a bounded wait expired
    int rows[kC];         // token row index (b*L + s)*H + h of each chunk row
    float bref[kD];       // reference r_c (log)
    float eref[kD];       // e^{r_c}
    float Bc[kD];         // B_c = b_{n-1,c} (log)
    float eB[kD];         // e^{B_c}
    float fB[kD];         // e^{B_c - r_c}
    float Gs[kD];         // segment total log-decay (exchange)
    float tot0[kD];       // cumulative sum of the first 64 rows
    float b0[kD];         // b_{0,c}
    float w[kD];          // RMSNorm weight
};
static_assert(sizeof(Misc) <= 4096, "misc region");

template <int D>
__global__ void __launch_bounds__(kThreads, 1) gla_tc_kernel(const Params p) {
    static_assert(D == kD, "tensor-core kernel handles d_k = d_v = 64");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
    const uint32_t sbase = ptx::smem_u32(sm);
    Misc &m = *reinterpret_cast<Misc *>(sm + kMISC);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int pair = blockIdx.x / p.segs;
    const int rank = blockIdx.x - pair * p.segs;
    const int bb = pair / p.H, hh = pair - bb * p.H;
    const int dir = p.dir == 4 ? (bb & 3) : p.dir;
    const int p0 = min(p.L, rank * p.seg_len);
    const int p1 = min(p.L, p0 + p.seg_len);
    const int seg_n = p1 - p0;
    const int n_chunks = seg_n > 0 ? (seg_n + p.chunk_max - 1) / p.chunk_max : 0;
    const int chunk_len = n_chunks > 0 ? (seg_n + n_chunks - 1) / n_chunks : 0;
    const bool exchange = p.segs > 1;
    const bool resident = n_chunks <= 1;

    // ---- setup: TMEM, barriers, weight ----
    if (warp == 0) {
        ptx::tmem_alloc(&m.tmem_base, kTmemCols);
        ptx::tmem_relinquish();
    }
    if (tid == 0) {
        ptx::mbar_init(&m.mbar[0], 1);
        ptx::mbar_init(&m.mbar[1], 1);
        ptx::fence_mbarrier_init();
        m.abort = 0;
        m.range_err = 0;
    }
    if (tid < kD) {
        m.w[tid] = p.w[tid];
        m.Gs[tid] = 0.0f;
    }
    ptx::tc_fence_before_sync();
    __syncthreads();
    ptx::tc_fence_after_sync();
    const uint32_t tmem = m.tmem_base;
    const uint32_t tmem_warp = tmem + ((uint32_t)(warp * 32) << 16);
    uint32_t ph0 = 0, ph1 = 0;

    // state owned by threads with lane < 16: row c = 16*warp + lane, 64 columns
    const bool s_owner = lane < 16;
    const int s_row = warp * 16 + lane;
    float S[kD];
#pragma unroll
    for (int j = 0; j < kD; ++j) S[j] = 0.0f;

    // ------------------------------------------------------------ helpers
    auto set_rows = [&](int c0, int n) {
        if (tid < n) m.rows[tid] = (bb * p.L + spatial_of(dir, c0 + tid, p.gh, p.gw)) * p.H + hh;
    };
    // gather one fp16 [n rows][64] tile into the swizzled layout, zero rows >= n
    auto load_tile = [&](const __half *src, uint32_t dst, int n) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int idx = tid + i * kThreads;
            const int row = idx >> 3, j = idx & 7;
            const bool ok = row < n;
            const __half *g = src + (ok ? (size_t)m.rows[row] * kD + j * 8 : 0);
            ptx::cp_async16(sbase + dst + off_f16(row, j), g, ok ? 16u : 0u);
        }
    };
    // column-owner cumulative sum of lambda; writes b (fp32) and per-channel scalars
    auto gate = [&](int n) {
        const int c = tid & 63, half = tid >> 6;
        float cs[64];
        float run = 0.0f;
        const uint8_t *ta = sm + kTA;
#pragma unroll 8
        for (int i = 0; i < 64; ++i) {
            const int t = half * 64 + i;
            const __half av = *reinterpret_cast<const __half *>(ta + off_f16(t, c >> 3) + (c & 7) * 2);
            const float lam = t < n ? log_gamma_fast(__half2float(av)) : 0.0f;
            run += lam;
            cs[i] = run;
        }
        if (half == 0) {
            m.tot0[c] = run;
            m.b0[c] = cs[0];
        }
        __syncthreads();
        const float add = half ? m.tot0[c] : 0.0f;
        const int mid = (n - 1) >> 1;
        float *bp = reinterpret_cast<float *>(sm + kPB);
#pragma unroll 8
        for (int i = 0; i < 64; ++i) {
            const int t = half * 64 + i;
            const float bt = cs[i] + add;
            bp[(off_tf32(kAtom128, t, c >> 2) >> 2) + (c & 3)] = bt;
            if (t == mid) m.bref[c] = bt;
            if (t == n - 1) m.Bc[c] = bt;
        }
        __syncthreads();
        if (tid < kD) {
            const float r = m.bref[tid], Bv = m.Bc[tid];
            const bool wide = (m.b0[tid] - r > kHalfRangeSafe) || (r - Bv > kHalfRangeSafe);
            m.eB[tid] = __expf(Bv);
            m.fB[tid] = __expf(Bv - r);
            if (wide) m.slow = 1;
        }
    };
    // row-owner operand construction: Q~, K~ (fast path) and Ks; full = false builds Ks only
    auto build_operands = [&](bool full) {
        const int t = tid;
        const bool slow = m.slow != 0;
        const float *bp = reinterpret_cast<const float *>(sm + kPB);
#pragma unroll 2
        for (int j = 0; j < 8; ++j) {  // 8 channels per step
            const uint4 kraw = *reinterpret_cast<const uint4 *>(sm + kTK + off_f16(t, j));
            const uint4 qraw = *reinterpret_cast<const uint4 *>(sm + kTQ + off_f16(t, j));
            const __half2 *k2 = reinterpret_cast<const __half2 *>(&kraw);
            const __half2 *q2 = reinterpret_cast<const __half2 *>(&qraw);
            float bt[8], kv[8], qv[8];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const float4 b4 = *reinterpret_cast<const float4 *>(
                    reinterpret_cast<const uint8_t *>(bp) + off_tf32(kAtom128, t, 2 * j + h));
                bt[4 * h + 0] = b4.x; bt[4 * h + 1] = b4.y; bt[4 * h + 2] = b4.z; bt[4 * h + 3] = b4.w;
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 kf = __half22float2(k2[e]);
                const float2 qf = __half22float2(q2[e]);
                kv[2 * e] = kf.x; kv[2 * e + 1] = kf.y;
                qv[2 * e] = qf.x; qv[2 * e + 1] = qf.y;
            }
            float ks[8], qh[8], ql[8], kh[8], kl[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int c = 8 * j + e;
                if (!slow) {
                    const float e2 = __expf(m.bref[c] - bt[e]);       // e^{r - b}
                    ks[e] = kv[e] * e2 * m.fB[c];                   // k e^{B - b}
                    if (full) {
                        const float kf = kv[e] * e2;
                        const float qf = qv[e] * __expf(bt[e] - m.bref[c]);  // q e^{b - r}
                        kh[e] = ptx::to_tf32(kf);
                        kl[e] = ptx::to_tf32(kf - kh[e]);
                        qh[e] = ptx::to_tf32(qf);
                        ql[e] = ptx::to_tf32(qf - qh[e]);
                    }
                } else {
                    ks[e] = kv[e] * __expf(m.Bc[c] - bt[e]);
                    if (full) {                                      // reference = chunk start
                        qh[e] = ptx::to_tf32(qv[e] * __expf(bt[e]));
                        ql[e] = 0.0f;
                    }
                }
            }
            uint4 kso;
            kso.x = pack_half2(ks[0], ks[1]); kso.y = pack_half2(ks[2], ks[3]);
            kso.z = pack_half2(ks[4], ks[5]); kso.w = pack_half2(ks[6], ks[7]);
            *reinterpret_cast<uint4 *>(sm + kST + off_f16(t, j)) = kso;
            if (full) {
                ptx::tmem_st8(tmem_warp + kColQH + 8 * j, qh);
                ptx::tmem_st8(tmem_warp + kColQL + 8 * j, ql);
                if (!slow) {
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        *reinterpret_cast<float4 *>(sm + kKH + off_tf32(kAtom128, t, 2 * j + h)) =
                            make_float4(kh[4 * h], kh[4 * h + 1], kh[4 * h + 2], kh[4 * h + 3]);
                        *reinterpret_cast<float4 *>(sm + kKL + off_tf32(kAtom128, t, 2 * j + h)) =
                            make_float4(kl[4 * h], kl[4 * h + 1], kl[4 * h + 2], kl[4 * h + 3]);
                    }
                }
            }
        }
        if (full) ptx::tmem_st_wait();
    };
    // one-thread MMA issue + commit, everyone waits
    auto mma_round = [&](int which) {  // 0: state only, 1: QK (+state), 2: PV + inter
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before_sync();
        __syncthreads();
        if (tid == 0) {
            ptx::tc_fence_after_sync();
            if (which == 0) {
                issue_state(sbase, tmem);
                ptx::mma_commit(&m.mbar[0]);
            } else if (which == 1) {
                if (!m.slow) issue_qk(sbase, tmem);
                issue_state(sbase, tmem);
                ptx::mma_commit(&m.mbar[0]);
            } else {
                issue_pv(sbase, m.slow ? kKH : kPB, tmem);
                issue_inter(sbase, tmem, true);
                ptx::mma_commit(&m.mbar[1]);
            }
        }
        uint64_t *bar = which == 2 ? &m.mbar[1] : &m.mbar[0];
        uint32_t &ph = which == 2 ? ph1 : ph0;
        if (!wait_phase(bar, ph)) m.abort = 1;
        ph ^= 1u;
        ptx::tc_fence_after_sync();
    };
    // Sloc (TMEM, M=64 layout) -> registers of the state owners (whole warps execute the load)
    auto read_sloc = [&](float (&Sl)[kD]) {
        float r0[32], r1[32];
        ptx::tmem_ld32(tmem_warp + kColSL, r0);
        ptx::tmem_ld32(tmem_warp + kColSL + 32, r1);
        ptx::tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            Sl[j] = r0[j];
            Sl[32 + j] = r1[j];
        }
    };
    // masked, scaled scores -> P (fp16, K-major, 2 atoms) in the b region
    auto make_p_fast = [&]() {
        const int t = tid;
        int err = 0;
        // exact diagonal score q_t . k_t (decay factor 1), fp32 from the raw tiles
        float dq = 0.0f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint4 kraw = *reinterpret_cast<const uint4 *>(sm + kTK + off_f16(t, j));
            const uint4 qraw = *reinterpret_cast<const uint4 *>(sm + kTQ + off_f16(t, j));
            const __half2 *k2 = reinterpret_cast<const __half2 *>(&kraw);
            const __half2 *q2 = reinterpret_cast<const __half2 *>(&qraw);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 kf = __half22float2(k2[e]), qf = __half22float2(q2[e]);
                dq = fmaf(qf.x, kf.x, dq);
                dq = fmaf(qf.y, kf.y, dq);
            }
        }
#pragma unroll 1
        for (int blk = 0; blk < 4; ++blk) {
            float r[32];
            ptx::tmem_ld32(tmem_warp + kColDS + blk * 32, r);
            ptx::tmem_ld_wait();
#pragma unroll
            for (int j4 = 0; j4 < 4; ++j4) {  // four 16 B chunks of 8 halves
                float v8[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int s = blk * 32 + j4 * 8 + e;
                    const float x = s < t ? r[j4 * 8 + e] * p.scale : (s == t ? dq * p.scale : 0.0f);
                    err |= fabsf(x) > 65504.0f;
                    v8[e] = x;
                }
                uint4 o;
                o.x = pack_half2(v8[0], v8[1]); o.y = pack_half2(v8[2], v8[3]);
                o.z = pack_half2(v8[4], v8[5]); o.w = pack_half2(v8[6], v8[7]);
                *reinterpret_cast<uint4 *>(sm + kPB + off_f16k128(t, blk * 4 + j4)) = o;
            }
        }
        if (err) m.range_err = 1;
    };
    // exact scores on CUDA cores (reference = each pair's own decay), P into the K~ region
    auto make_p_slow = [&](int n) {
        const int t = tid;
        const float *bp = reinterpret_cast<const float *>(sm + kPB);
        auto bat = [&](int row, int c) {
            return bp[(off_tf32(kAtom128, row, c >> 2) >> 2) + (c & 3)];
        };
        auto hat = [&](uint32_t tile, int row, int c) {
            return __half2float(*reinterpret_cast<const __half *>(sm + tile + off_f16(row, c >> 3) +
                                                                   (c & 7) * 2));
        };
        int err = 0;
        for (int s0 = 0; s0 < kC; s0 += 8) {
            float v8[8];
            for (int e = 0; e < 8; ++e) {
                const int s = s0 + e;
                float acc = 0.0f;
                if (s <= t && t < n) {
                    for (int c = 0; c < kD; ++c)
                        acc = fmaf(hat(kTQ, t, c) * hat(kTK, s, c), expf(bat(t, c) - bat(s, c)), acc);
                }
                acc *= p.scale;
                err |= fabsf(acc) > 65504.0f;
                v8[e] = acc;
            }
            uint4 o;
            o.x = pack_half2(v8[0], v8[1]); o.y = pack_half2(v8[2], v8[3]);
            o.z = pack_half2(v8[4], v8[5]); o.w = pack_half2(v8[6], v8[7]);
            *reinterpret_cast<uint4 *>(sm + kKH + off_f16k128(t, s0 >> 3)) = o;
        }
        if (err) m.range_err = 1;
    };
    // S~ = scale * Diag(e^{r}) S_in, tf32 K-major [j][c] (2 atoms of 64 rows)
    auto write_stilde = [&]() {
        if (s_owner) {
            const int c = s_row;
            const float f = p.scale * m.eref[c];
            float *st = reinterpret_cast<float *>(sm + kST);
#pragma unroll 8
            for (int j = 0; j < kD; ++j)
                st[(off_tf32(kAtom64, j, c >> 2) >> 2) + (c & 3)] = ptx::to_tf32(S[j] * f);
        }
    };
    // u = SiLU(g) * o / sqrt(mean(o^2) + eps) * w for the chunk's rows
    auto epilogue = [&](int n) {
        const int t = tid;
        float o[64];
        {
            float r0[32], r1[32];
            ptx::tmem_ld32(tmem_warp + kColO, r0);
            ptx::tmem_ld32(tmem_warp + kColO + 32, r1);
            ptx::tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                o[j] = r0[j];
                o[32 + j] = r1[j];
            }
        }
        float ss = 0.0f;
#pragma unroll
        for (int j = 0; j < 64; ++j) ss = fmaf(o[j], o[j], ss);
        const float inv = rsqrtf(ss * (1.0f / 64.0f) + p.eps);
        if (t < n) {
            __half *dst = p.out + (size_t)m.rows[t] * kD;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint4 graw = *reinterpret_cast<const uint4 *>(sm + kTG + off_f16(t, j));
                const __half2 *g2 = reinterpret_cast<const __half2 *>(&graw);
                float u[8];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 gf = __half22float2(g2[e]);
                    const int c = 8 * j + 2 * e;
                    u[2 * e] = o[c] * inv * m.w[c] * silu_fast(gf.x);
                    u[2 * e + 1] = o[c + 1] * inv * m.w[c + 1] * silu_fast(gf.y);
                }
                uint4 pk;
                pk.x = pack_half2(u[0], u[1]); pk.y = pack_half2(u[2], u[3]);
                pk.z = pack_half2(u[4], u[5]); pk.w = pack_half2(u[6], u[7]);
                *reinterpret_cast<uint4 *>(dst + 8 * j) = pk;
            }
        }
    };
    auto finish_gate = [&]() {  // per-chunk reference factors after the slow decision
        __syncthreads();
        if (tid < kD) {
            if (m.slow) m.bref[tid] = 0.0f;
            m.eref[tid] = __expf(m.bref[tid]);
        }
        __syncthreads();
    };
    auto chunk_bounds = [&](int ci, int &c0, int &n) {
        c0 = p0 + ci * chunk_len;
        n = min(chunk_len, p1 - c0);
    };
    // fold the chunk's local state into S: S = e^{B} S + Sloc
    auto fold_sloc = [&](float (&Sl)[kD], bool into_g) {
        if (s_owner) {
            const float e = m.eB[s_row];
#pragma unroll
            for (int j = 0; j < kD; ++j) S[j] = fmaf(e, S[j], Sl[j]);
            if (into_g) m.Gs[s_row] += m.Bc[s_row];
        }
    };
    // cluster-wide scan of (Gs, S) -> S becomes this segment's incoming state
    auto exchange_states = [&]() {
        float *X = reinterpret_cast<float *>(sm + kST);  // [64][64] fp32, plain row-major
        __syncthreads();
        if (s_owner) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int j4 = (i + lane) & 15;
                *reinterpret_cast<float4 *>(X + s_row * kD + 4 * j4) =
                    make_float4(S[4 * j4], S[4 * j4 + 1], S[4 * j4 + 2], S[4 * j4 + 3]);
            }
        }
        cg::cluster_group cluster = cg::this_cluster();
        cluster.sync();
        const int E = kD * kD;
        const int per = (E + p.segs - 1) / p.segs;
        const int e0 = rank * per, e1 = min(E, e0 + per);
        for (int e = e0 + tid; e < e1; e += kThreads) {
            const int c = e / kD;
            float run = 0.0f;
            for (int r = 0; r < p.segs; ++r) {
                float *Xr = cluster.map_shared_rank(X, r);
                const float *Gr = cluster.map_shared_rank(m.Gs, r);
                const float agg = Xr[e];
                const float dec = __expf(Gr[c]);
                Xr[e] = run;
                run = fmaf(dec, run, agg);
            }
        }
        cluster.sync();
        if (s_owner) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int j4 = (i + lane) & 15;
                const float4 x = *reinterpret_cast<const float4 *>(X + s_row * kD + 4 * j4);
                S[4 * j4] = x.x; S[4 * j4 + 1] = x.y; S[4 * j4 + 2] = x.z; S[4 * j4 + 3] = x.w;
            }
        }
        __syncthreads();
    };
    // second half of a chunk: P, S~, PV + inter, epilogue; S advances by the chunk
    auto finish_chunk = [&](int n, float (&Sl)[kD], bool advance) {
        if (m.slow) make_p_slow(n); else make_p_fast();
        write_stilde();
        mma_round(2);
        epilogue(n);
        if (advance) fold_sloc(Sl, false);
        ptx::tc_fence_before_sync();
        __syncthreads();
    };

    float Sl[kD];
    if (resident) {
        // ---- one chunk: load all tiles, exchange mid-chunk ----
        int c0, n;
        chunk_bounds(0, c0, n);
        if (n > 0) set_rows(c0, n);
        if (tid == 0) m.slow = 0;
        __syncthreads();
        load_tile(p.k, kTK, n); load_tile(p.a, kTA, n); load_tile(p.v, kTV, n);
        load_tile(p.q, kTQ, n); load_tile(p.g, kTG, n);
        ptx::cp_async_commit();
        ptx::cp_async_wait_all();
        __syncthreads();
        gate(n);
        finish_gate();
        build_operands(true);
        mma_round(1);
        read_sloc(Sl);
        if (exchange) {
            fold_sloc(Sl, true);                      // S = 0 * e^{B} + Sloc, Gs = B
            exchange_states();
        }
        finish_chunk(n, Sl, false);
    } else {
        // ---- pass 1: state-only fold of this segment (not needed by the last one) ----
        if (exchange) {
            if (rank < p.segs - 1) {
                for (int ci = 0; ci < n_chunks; ++ci) {
                    int c0, n;
                    chunk_bounds(ci, c0, n);
                    __syncthreads();
                    set_rows(c0, n);
                    if (tid == 0) m.slow = 0;
                    __syncthreads();
                    load_tile(p.k, kTK, n); load_tile(p.a, kTA, n); load_tile(p.v, kTV, n);
                    ptx::cp_async_commit();
                    ptx::cp_async_wait_all();
                    __syncthreads();
                    gate(n);
                    finish_gate();
                    build_operands(false);
                    mma_round(0);
                    read_sloc(Sl);
                    fold_sloc(Sl, true);
                    ptx::tc_fence_before_sync();
                    __syncthreads();
                }
            }
            exchange_states();
        }
        // ---- pass 2: outputs from the incoming state ----
        for (int ci = 0; ci < n_chunks; ++ci) {
            int c0, n;
            chunk_bounds(ci, c0, n);
            __syncthreads();
            set_rows(c0, n);
            if (tid == 0) m.slow = 0;
            __syncthreads();
            load_tile(p.k, kTK, n); load_tile(p.a, kTA, n); load_tile(p.v, kTV, n);
            load_tile(p.q, kTQ, n); load_tile(p.g, kTG, n);
            ptx::cp_async_commit();
            ptx::cp_async_wait_all();
            __syncthreads();
            gate(n);
            finish_gate();
            build_operands(true);
            mma_round(1);
            read_sloc(Sl);
            finish_chunk(n, Sl, ci + 1 < n_chunks);
        }
    }

    // ---- teardown ----
    __syncthreads();
    if (tid == 0 && m.range_err) raise_status(8 /* GLA_ERR_RANGE */);
    ptx::tc_fence_after_sync();
    if (warp == 0) ptx::tmem_dealloc(tmem, kTmemCols);
}

// ---------------------------------------------------------------- self-test
// Runs one of the kernel's four MMA configurations on row-major fp32 inputs
// (converted to the operand type in the same shared-memory layouts) and
// writes D row-major: 0 = scores (split tf32, A[128][64] . B[128][64]^T -> [128][128]),
// 1 = state (f16, A[128][64]^T . B[128][64] -> [64][64]), 2 = PV (f16,
// A[128][128] . B[128][64] -> [128][64]), 3 = inter (tf32, A[128][64] .
// B[64][64]^T -> [128][64]).  One CTA of 128 threads.
__global__ void __launch_bounds__(kThreads, 1)
gla_tc_selftest_kernel(int kind, const float *A, const float *Bm, float *Dout) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
    const uint32_t sbase = ptx::smem_u32(sm);
    Misc &m = *reinterpret_cast<Misc *>(sm + kMISC);
    const int tid = threadIdx.x, warp = tid >> 5;
    if (warp == 0) {
        ptx::tmem_alloc(&m.tmem_base, kTmemCols);
        ptx::tmem_relinquish();
    }
    if (tid == 0) {
        ptx::mbar_init(&m.mbar[0], 1);
        ptx::fence_mbarrier_init();
    }
    ptx::tc_fence_before_sync();
    __syncthreads();
    ptx::tc_fence_after_sync();
    const uint32_t tmem = m.tmem_base;
    const uint32_t tmem_warp = tmem + ((uint32_t)(warp * 32) << 16);
    const int t = tid;
    auto put_tf32 = [&](uint32_t region, uint32_t atom, int row, const float *src) {
        for (int c4 = 0; c4 < 16; ++c4)
            *reinterpret_cast<float4 *>(sm + region + off_tf32(atom, row, c4)) =
                make_float4(ptx::to_tf32(src[4 * c4]), ptx::to_tf32(src[4 * c4 + 1]),
                            ptx::to_tf32(src[4 * c4 + 2]), ptx::to_tf32(src[4 * c4 + 3]));
    };
    auto put_f16 = [&](uint32_t region, int row, const float *src) {
        for (int j = 0; j < 8; ++j) {
            uint4 o;
            o.x = pack_half2(src[8 * j], src[8 * j + 1]); o.y = pack_half2(src[8 * j + 2], src[8 * j + 3]);
            o.z = pack_half2(src[8 * j + 4], src[8 * j + 5]); o.w = pack_half2(src[8 * j + 6], src[8 * j + 7]);
            *reinterpret_cast<uint4 *>(sm + region + off_f16(row, j)) = o;
        }
    };
    // split a row into tf32 high/low parts: rows of A go to TMEM, rows of B to shared memory
    auto put_split_tmem = [&](const float *src, bool with_low) {
        for (int j = 0; j < 8; ++j) {
            float h[8], l[8];
            for (int e = 0; e < 8; ++e) {
                h[e] = ptx::to_tf32(src[8 * j + e]);
                l[e] = with_low ? ptx::to_tf32(src[8 * j + e] - h[e]) : 0.0f;
            }
            ptx::tmem_st8(tmem_warp + kColQH + 8 * j, h);
            ptx::tmem_st8(tmem_warp + kColQL + 8 * j, l);
        }
        ptx::tmem_st_wait();
    };
    if (kind == 0) {
        put_split_tmem(A + t * 64, true);
        float hi[64], lo[64];
        for (int c = 0; c < 64; ++c) {
            hi[c] = ptx::to_tf32(Bm[t * 64 + c]);
            lo[c] = ptx::to_tf32(Bm[t * 64 + c] - hi[c]);
        }
        put_tf32(kKH, kAtom128, t, hi);
        put_tf32(kKL, kAtom128, t, lo);
    } else if (kind == 1) {
        put_f16(kST, t, A + t * 64);
        put_f16(kTV, t, Bm + t * 64);
    } else if (kind == 2) {
        for (int j = 0; j < 16; ++j) {
            const float *src = A + t * 128 + 8 * j;
            uint4 o;
            o.x = pack_half2(src[0], src[1]); o.y = pack_half2(src[2], src[3]);
            o.z = pack_half2(src[4], src[5]); o.w = pack_half2(src[6], src[7]);
            *reinterpret_cast<uint4 *>(sm + kPB + off_f16k128(t, j)) = o;
        }
        put_f16(kTV, t, Bm + t * 64);
    } else {
        put_split_tmem(A + t * 64, false);
        if (t < 64) put_tf32(kST, kAtom64, t, Bm + t * 64);
    }
    ptx::fence_proxy_async_smem();
    ptx::tc_fence_before_sync();
    __syncthreads();
    if (tid == 0) {
        ptx::tc_fence_after_sync();
        if (kind == 0) issue_qk(sbase, tmem);
        else if (kind == 1) issue_state(sbase, tmem);
        else if (kind == 2) issue_pv(sbase, kPB, tmem);
        else issue_inter(sbase, tmem, false);
        ptx::mma_commit(&m.mbar[0]);
    }
    wait_phase(&m.mbar[0], 0);
    ptx::tc_fence_after_sync();
    if (kind == 0) {
        for (int blk = 0; blk < 4; ++blk) {
            float r[32];
            ptx::tmem_ld32(tmem_warp + kColDS + blk * 32, r);
            ptx::tmem_ld_wait();
            for (int j = 0; j < 32; ++j) Dout[t * 128 + blk * 32 + j] = r[j];
        }
    } else if (kind == 1) {
        float r0[32], r1[32];
        ptx::tmem_ld32(tmem_warp + kColSL, r0);
        ptx::tmem_ld32(tmem_warp + kColSL + 32, r1);
        ptx::tmem_ld_wait();
        if ((tid & 31) < 16) {
            const int c = warp * 16 + (tid & 31);
            for (int j = 0; j < 32; ++j) {
                Dout[c * 64 + j] = r0[j];
                Dout[c * 64 + 32 + j] = r1[j];
            }
        }
    } else {
        float r0[32], r1[32];
        ptx::tmem_ld32(tmem_warp + kColO, r0);
        ptx::tmem_ld32(tmem_warp + kColO + 32, r1);
        ptx::tmem_ld_wait();
        for (int j = 0; j < 32; ++j) {
            Dout[t * 64 + j] = r0[j];
            Dout[t * 64 + 32 + j] = r1[j];
        }
    }
    ptx::tc_fence_before_sync();
    __syncthreads();
    ptx::tc_fence_after_sync();
    if (warp == 0) ptx::tmem_dealloc(tmem, kTmemCols);
}

}  // namespace tc
}  // namespace gla
