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
// per-channel reference (the chunk's middle row).  The kernel keeps b, B, r
// in log2 units so every factor below is one ex2.  With Q~ = q (.) e^{b - r},
// K~ = k (.) e^{r - b}, Ks = k (.) e^{B - b} and the state S_in entering the
// chunk:
//   scores   A     = Q~ K~^T   split-tf32: Qh Kh^T + Qh Kl^T + Ql Kh^T, where
//                    X = Xh + Xl with Xh = tf32(X), Xl = tf32(X - Xh)
//                    (tcgen05 kind::tf32, A operands Qh/Ql in TMEM, 128x128x64)
//   masked   P     = d_k^{-1/2} A (.) [s <= t], diagonal A_tt = q_t . k_t in fp32
//                    (d_k^{-1/2} = 2^-3 is folded into Q~'s exponent)
//   output   O     = P V + (Qh + Ql) S~,  S~ = tf32(Diag(e^{r}) S_in)  (f16 + tf32
//                    MMAs; S~ is an MN-major operand)
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
// cluster through distributed shared memory (the combine is elementwise per
// state entry with the decay of its key channel, so CTA r scans the 4-channel
// key groups g = r, r + segs, ...), giving every segment its incoming state.
// When the launch's segments fit one chunk, each keeps its tiles resident
// and does the exchange mid-chunk; otherwise the segments run a state-only
// pass, the exchange, then the full pass, gathering each next chunk under
// the current one.
//
// Input gathers: 16-byte cp.async per thread, scan row t of the chunk read
// from the token's spatial position (direction remap folded into the
// address), written straight into the 128B-swizzled operand layout.
#pragma once

#include "gla_common.cuh"
#include "gla_ptx.cuh"

namespace gla {
namespace tc {

constexpr int kThreads = 256;      // two threads per chunk row (one per channel half)
constexpr int kSelfThreads = 128;  // self-test kernel: one thread per row
constexpr int kC = 128;            // max tokens per chunk (MMA M)
constexpr int kD = 64;             // head dim handled by this kernel
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLog2Scale = -3.0f;   // log2(d_k^{-1/2}) for d_k = 64, folded into Q~
// largest |b - r| (log2 units) the tf32 operands carry: 2^86 * 65504 stays finite in fp32
constexpr float kHalfRangeSafe2 = 86.0f;

// ---- shared memory map (bytes from a 1024-aligned base) ----
constexpr uint32_t kKL = 0;        // K~ low part  tf32, 2 atoms x [128][128B]; then u staging
constexpr uint32_t kKH = 32768;    // K~ high part tf32, 2 atoms x [128][128B] (slow path: P)
constexpr uint32_t kPB = 65536;    // b   fp32 (QT layout), then P fp16 2 atoms x [128][128B]
constexpr uint32_t kST = 98304;    // Ks fp16 [128][128B]
constexpr uint32_t kTQ = 114688;   // raw tiles, fp16 [128][128B] each
constexpr uint32_t kTK = 131072;
constexpr uint32_t kTA = 147456;   // a tile; after the gate: S~ tf32 MN-major, 2 x [64 c][128B]
constexpr uint32_t kTV = 163840;
constexpr uint32_t kTG = 180224;   // g tile; before a multi-chunk pass: S_in [64 c][64 j] fp32
constexpr uint32_t kMISC = 196608;
constexpr uint32_t kMiscBytes = 8192;
constexpr uint32_t kAtom128 = 16384;   // [128 rows][128 B]
constexpr uint32_t kAtom64 = 8192;     // [64 rows][128 B]
// State exchange: the 64 key channels form 16 groups of 4; group g is scanned by CTA
// g % segs.  A scanner receives, per (own group, segment), 64 aggregate rows plus the
// segment's 2^G and 2^r entries of the group: 66 x 16 B.  A CTA owns ceil((16-r)/segs)
// groups, so the buffer bounds ceil(16/segs) * segs <= kMaxGroupSegs.
constexpr uint32_t kRECV = kMISC + kMiscBytes;
constexpr int kGroupRows = kD + 2;
constexpr int kMaxGroupSegs = 24;
constexpr uint32_t kRecvBytes = kMaxGroupSegs * kGroupRows * 16;
constexpr size_t kSmemBytes = kRECV + kRecvBytes + 1024;  // + alignment slack

// TMEM columns
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColDS = 0;     // scores, 128 x 128 fp32
constexpr uint32_t kColSL = 128;   // chunk state Ks^T V, M=64 layout
constexpr uint32_t kColO = 192;    // inter-chunk output accumulator 128 x 64
constexpr uint32_t kColQH = 256;   // Q~ high part, tf32 A operand, 128 x 64
constexpr uint32_t kColQL = 320;   // Q~ low part
constexpr uint32_t kColOP = 384;   // intra-chunk output accumulator (P V) 128 x 64
constexpr uint32_t kColSG = 448;   // SiLU(g) * w per token and channel, 128 x 64 fp32

constexpr uint32_t kIdescST = ptx::idesc_make(0, true, true, 64, 64);
constexpr uint32_t kIdescPV = ptx::idesc_make(0, false, true, 128, 64);
constexpr uint32_t kIdescIN = ptx::idesc_make(2, false, true, 128, 64);

struct Params {
    const __half *q, *k, *v, *a, *g;
    const float *w;
    __half *out;
    int B, H, gh, gw, L, dir;
    int segs;      // CTAs per (b, h) pair == cluster size
    int seg_len;   // scan positions per segment
    int chunk_max; // largest chunk (16..128); a segment is split into equal chunks
    float eps, scale;
    long long wait_limit;  // bound of every mbarrier wait, SM clocks
    int fault_chunk;       // test hook: full-pass chunk whose q/k loads never signal (-1: none)
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
// S~ (the inter product's B operand), tf32 MN-major: one 128-byte row per key channel c
// holding 32 value columns j, 32-byte granules swizzled by (c & 3) within 4-row groups of
// 512 bytes; two atoms for j < 32 and j >= 32.  Byte offset of (c, j).
__device__ __forceinline__ uint32_t off_stilde(uint32_t c, uint32_t j) {
    return (j >> 5) * kAtom64 + (c >> 2) * 512 + (c & 3) * 128 + ((((j & 31) >> 3) ^ (c & 3)) << 5) +
           (j & 7) * 4;
}
// Row slot of aggregate row j in the exchange receive buffer: a bijection within each
// 16-row block that keeps a warp's stores of 16 consecutive rows contiguous and makes the
// scanners' reads of 4 consecutive rows at one channel (8 row quads x 4 channels per warp)
// hit 32 distinct banks.
__device__ __forceinline__ uint32_t recv_slot(uint32_t j) {
    return (j & ~7u) | (j & 4u) | ((j ^ (j >> 2)) & 2u) | ((j ^ (j >> 4)) & 1u);
}

// ------------------------------------------------------------ MMA issue (1 thread)
// scores[t][s] = sum_c Q~[t][c] K~[s][c] as Qh Kh^T + Qh Kl^T + Ql Kh^T
// Only the first n_cols score columns (the chunk's rows rounded up to 16) are produced.
__device__ __forceinline__ void issue_qk(uint32_t sbase, uint32_t tmem, int n_cols) {
    const uint32_t idesc = ptx::idesc_make(2, false, false, 128, (uint32_t)n_cols);
#pragma unroll 1
    for (int pass = 0; pass < 3; ++pass) {
        const uint32_t acol = pass == 2 ? kColQL : kColQH;
        const uint32_t bsm = pass == 1 ? kKL : kKH;
#pragma unroll 1
        for (int k = 0; k < 8; ++k) {
            const uint32_t koff = (k >> 2) * kAtom128 + (k & 3) * 32;
            ptx::mma_tf32_ts(tmem + kColDS, tmem + acol + 8 * k,
                             ptx::desc_sw128(sbase + bsm + koff, 16, 1024), idesc,
                             pass > 0 || k > 0);
        }
    }
}
// Sloc^T[j][c] = sum_s V[s][j] Ks[s][c]  (both operands MN-major, K = 128 rows); the state is
// kept transposed so each thread owns one value column j and writes S~ rows contiguously.
__device__ __forceinline__ void issue_state(uint32_t sbase, uint32_t tmem) {
#pragma unroll 1
    for (int k = 0; k < 8; ++k) {
        ptx::mma_f16_ss(tmem + kColSL, ptx::desc_sw128(sbase + kTV + k * 2048, kAtom128, 1024),
                        ptx::desc_sw128(sbase + kST + k * 2048, kAtom128, 1024), kIdescST, k > 0);
    }
}
// O[t][j] = sum_s P[t][s] V[s][j]
__device__ __forceinline__ void issue_pv(uint32_t sbase, uint32_t p_base, uint32_t tmem) {
#pragma unroll 1
    for (int k = 0; k < 8; ++k) {
        const uint32_t koff = (k >> 2) * kAtom128 + (k & 3) * 32;
        ptx::mma_f16_ss(tmem + kColOP, ptx::desc_sw128(sbase + p_base + koff, 16, 1024),
                        ptx::desc_sw128(sbase + kTV + k * 2048, kAtom128, 1024), kIdescPV, k > 0);
    }
}
// O[t][j] (+)= sum_c (Qh + Ql)[t][c] S~[c][j], S~ (MN-major) in the a-tile region
__device__ __forceinline__ void issue_inter(uint32_t sbase, uint32_t tmem, bool accumulate) {
#pragma unroll 1
    for (int pass = 0; pass < 2; ++pass) {
#pragma unroll 1
        for (int k = 0; k < 8; ++k) {                  // 8 key channels = 8 S~ rows per step
            ptx::mma_tf32_ts(tmem + kColO, tmem + (pass ? kColQL : kColQH) + 8 * k,
                             ptx::desc_sw128_b32(sbase + kTA + k * 1024, kAtom64, 512), kIdescIN,
                             accumulate || pass > 0 || k > 0);
        }
    }
}

// Bounded wait on an mbarrier phase, `limit` SM clocks.  Once a wait of the CTA has expired
// (*abort set) it returns false at once; on expiry it latches GLA_ERR_TIMEOUT and sets *abort.
__device__ __forceinline__ bool wait_phase(uint64_t *bar, uint32_t parity, long long limit,
                                           volatile int *abort) {
    if (*abort) return false;
    const long long start = clock64();
    while (!ptx::mbar_try_wait(bar, parity)) {
        if (clock64() - start > limit) {
            raise_status(7 /* GLA_ERR_TIMEOUT */);
            *abort = 1;
            return false;
        }
    }
    return true;
}

// The same with cluster-scope acquire (data pushed by other CTAs of the cluster).
__device__ __forceinline__ bool wait_cluster_phase(uint64_t *bar, uint32_t parity, long long limit,
                                                   volatile int *abort) {
    if (*abort) return false;
    const long long start = clock64();
    while (!ptx::mbar_try_wait_cluster(bar, parity)) {
        if (clock64() - start > limit) {
            raise_status(7 /* GLA_ERR_TIMEOUT */);
            *abort = 1;
            return false;
        }
    }
    return true;
}

__device__ __forceinline__ float log2_gamma(float a) {
    const float x = ptx::ex2(-fabsf(a) * kLog2e);             // 2^{-|a| log2 e} = e^{-|a|}
    return (fminf(a, 0.0f) * kLog2e - ptx::lg2(1.0f + x)) * kInvTau;
}

// 1/x for a positive normal x on the FMA pipe: Newton-Raphson, y <- y + y (1 - x y), from an
// integer-subtraction seed.  Reading the float bits of x as an integer, C - bits(x) negates the
// exponent and replaces the mantissa m in [0, 1) by a linear function of it, so the seed is a
// piecewise-linear approximation of 1/x on every binade.  C = 0x7EF311C7 is the constant that
// minimises the seed's largest relative error over a binade (found by a direct search over C:
// 5.05%); each Newton step squares the error, so three steps reach fp32 rounding.  Used where
// the special-function unit is the busier pipe.
__device__ __forceinline__ float rcp_nr(float x) {
    float y = __uint_as_float(0x7EF311C7u - __float_as_uint(x));
#pragma unroll
    for (int i = 0; i < 3; ++i) y = fmaf(y, fmaf(-x, y, 1.0f), y);
    return y;
}

// SiLU(g) = g / (1 + e^{-g})
__device__ __forceinline__ float silu_fast(float g) {
    return g * ptx::rcp(1.0f + ptx::ex2(-g * kLog2e));
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
    const __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}

// Shared scratch scalars.
struct Misc {
    uint64_t mbar_mma[4];     // [0] state, [1] scores, [2] inter (+ P.V), [3] P.V (one chunk)
    uint64_t mbar_end;        // teardown after an expired wait: products still in flight
    uint64_t mbar_ld[3];      // [0] a tile, [1] q and k tiles, [2] v and g tiles
    uint64_t mbar_x[2];       // exchange: [0] aggregates received, [1] S~ / S_in received
    uint32_t tmem_base;
    int slow;                 // chunk uses the exact CUDA-core score path
    int range_err;            // a P entry overflowed fp16
    int abort;                // a bounded wait expired
    int rows[2][kC];          // token row index (b*L + s)*H + h of each chunk row (this chunk
                              // and, gathered early, the next one)
    alignas(16) float bref[kD];   // reference r_c (log2 units)
    alignas(16) float eref[kD];   // 2^{r_c}
    alignas(16) float Bc[kD];     // B_c = b_{n-1,c} (log2)
    alignas(16) float eB[kD];     // 2^{B_c}
    alignas(16) float fB[kD];     // 2^{B_c - r_c}
    alignas(16) float Gs[kD];     // segment total log2-decay (exchange)
    alignas(16) float b0[kD];     // b_{0,c}
    alignas(16) float w[kD];      // RMSNorm weight
    alignas(16) float tot[8][kD]; // per-16-row totals of the gate scan
    alignas(16) float red[2][kC]; // epilogue partial sums of squares (per channel half)
    alignas(16) float dqp[2][kC]; // diagonal score q_t . k_t, per channel half
};
static_assert(sizeof(Misc) <= kMiscBytes, "misc region");

// Exact scores on CUDA cores for a chunk whose decay range the tf32 operands
// cannot carry: P[t][s] = d_k^{-1/2} sum_c q_tc k_sc 2^{b_tc - b_sc} (s <= t),
// written as fp16 into the K~ high-part region.  Rare; kept out of line.
__device__ __noinline__ void make_p_exact(uint8_t *sm, int t, int ch, int n, float scale,
                                          int *range_err) {
    const float *bp = reinterpret_cast<const float *>(sm + kPB);
    auto bat = [&](int row, int c) { return bp[(off_tf32(kAtom128, row, c >> 2) >> 2) + (c & 3)]; };
    auto hat = [&](uint32_t tile, int row, int c) {
        return __half2float(*reinterpret_cast<const __half *>(sm + tile + off_f16(row, c >> 3) + (c & 7) * 2));
    };
    int err = 0;
    for (int s0 = ch * 64; s0 < ch * 64 + 64; s0 += 8) {
        float v8[8];
        for (int e = 0; e < 8; ++e) {
            const int s = s0 + e;
            float acc = 0.0f;
            if (s <= t && t < n) {
                for (int c = 0; c < kD; ++c)
                    acc = fmaf(hat(kTQ, t, c) * hat(kTK, s, c), exp2f(bat(t, c) - bat(s, c)), acc);
            }
            acc *= scale;
            err |= fabsf(acc) > 65504.0f;
            v8[e] = acc;
        }
        uint4 o;
        o.x = pack_half2(v8[0], v8[1]); o.y = pack_half2(v8[2], v8[3]);
        o.z = pack_half2(v8[4], v8[5]); o.w = pack_half2(v8[6], v8[7]);
        *reinterpret_cast<uint4 *>(sm + kKH + off_f16k128(t, s0 >> 3)) = o;
    }
    if (err) *range_err = 1;
}

// kMid: every segment of the launch is a single chunk and there are several segments (the
// host guarantees seg_len <= chunk_max and segs > 1): the exchange happens mid-chunk, and the
// state-only pass, the multi-chunk exchange, the next-chunk gathers and the no-exchange
// branches are compiled out of that instantiation.
// Score operands of a chunk whose decay range the fast operands cannot carry (row t, 32
// channels of half ch): Qh/Ql of d_k^{-1/2} q 2^{b} (chunk-start reference; P is then
// evaluated exactly) into TMEM, and the partial diagonal q_t . k_t.  Rare; kept out of line
// so the common path stays compact.  Called by whole warps (tcgen05.st is warp-collective).
__device__ __noinline__ void build_q_exact(uint8_t *sm, int t, int ch, uint32_t tmem_warp, float *dq_out) {
    float dqs = 0.0f;
    for (int jj = 0; jj < 4; ++jj) {
        const int j = ch * 4 + jj;
        const uint4 kraw = *reinterpret_cast<const uint4 *>(sm + kTK + off_f16(t, j));
        const uint4 qraw = *reinterpret_cast<const uint4 *>(sm + kTQ + off_f16(t, j));
        const __half2 *k2 = reinterpret_cast<const __half2 *>(&kraw);
        const __half2 *q2 = reinterpret_cast<const __half2 *>(&qraw);
        float qh[8], ql[8];
        for (int e = 0; e < 8; ++e) {
            const float kf = e & 1 ? __high2float(k2[e >> 1]) : __low2float(k2[e >> 1]);
            const float qv = e & 1 ? __high2float(q2[e >> 1]) : __low2float(q2[e >> 1]);
            const float bt = reinterpret_cast<const float *>(sm + kPB + off_tf32(kAtom128, t, 2 * j + (e >> 2)))[e & 3];
            dqs = fmaf(qv, kf, dqs);
            const float qf = qv * ptx::ex2(bt + kLog2Scale);
            qh[e] = ptx::tf32_hi(qf);
            ql[e] = qf - qh[e];
        }
        ptx::tmem_st8(tmem_warp + kColQH + 8 * j, qh);
        ptx::tmem_st8(tmem_warp + kColQL + 8 * j, ql);
    }
    *dq_out = dqs;
    ptx::tmem_st_wait();
}

template <int D, bool kMid>
__global__ void __launch_bounds__(kThreads, 1) gla_tc_kernel(const Params p) {
    static_assert(D == kD, "tensor-core kernel handles d_k = d_v = 64");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
    const uint32_t sbase = ptx::smem_u32(sm);
    Misc &m = *reinterpret_cast<Misc *>(sm + kMISC);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int w4 = warp & 3;          // TMEM lane quarter of this warp
    const int ch = warp >> 2;         // channel half handled by this thread (row-owner work)
    const int t = w4 * 32 + lane;     // chunk row owned by this thread
    const int pair = blockIdx.x / p.segs;
    const int rank = blockIdx.x - pair * p.segs;
    const int bb = pair / p.H, hh = pair - bb * p.H;
    const int dir = p.dir == 4 ? (bb & 3) : p.dir;
    const int p0 = min(p.L, rank * p.seg_len);
    const int p1 = min(p.L, p0 + p.seg_len);
    const int seg_n = p1 - p0;
    const int n_chunks = seg_n > 0 ? (seg_n + p.chunk_max - 1) / p.chunk_max : 0;
    const int chunk_len = n_chunks > 0 ? (seg_n + n_chunks - 1) / n_chunks : 0;
    const bool exchange = kMid || p.segs > 1;
    // Residency follows the launch's segment length, not this segment's: a scanner writes
    // every destination in its own layout (S~ for resident segments, S_in otherwise), so all
    // CTAs of a cluster must agree.  A shorter last segment of one chunk, in a launch whose
    // segments span several, takes the multi-chunk path with a single chunk.
    const bool resident = kMid || p.seg_len <= p.chunk_max;

    // Programmatic dependent launch: the next launch on the stream may start its prologue now;
    // this grid touches no global memory before the previous grid has completed.
    ptx::pdl_launch_dependents();
    // ---- setup: barriers and weight; TMEM is allocated once the first gathers are in flight
    if (tid == 0) {
        for (int i = 0; i < 4; ++i) ptx::mbar_init(&m.mbar_mma[i], 1);
        ptx::mbar_init(&m.mbar_end, 3);       // one commit from each MMA-issuing warp (0, 4, 7)
        for (int i = 0; i < 3; ++i) ptx::mbar_init(&m.mbar_ld[i], kThreads);
        ptx::fence_mbarrier_init();
        m.abort = 0;
        m.range_err = 0;
    }
    if (tid < kD) m.Gs[tid] = 0.0f;
    // Exchange partition: CTA r scans the channel groups g = r, r + segs, ... (< 16).
    const int my_groups = exchange ? (16 - rank + p.segs - 1) / p.segs : 0;
    if (exchange) {
        if (tid == 0) {
            ptx::mbar_init(&m.mbar_x[0], 1);
            ptx::mbar_init(&m.mbar_x[1], 1);
            ptx::fence_mbarrier_init();
            // every segment sends this CTA, per owned group, 64 aggregate rows and its 2^G and
            // 2^r entries; every 16 B of this CTA's S~ (or S_in) arrives exactly once
            ptx::mbar_arrive_expect_tx(&m.mbar_x[0], (uint32_t)(my_groups * p.segs * kGroupRows * 16));
            ptx::mbar_arrive_expect_tx(&m.mbar_x[1], (uint32_t)(kD * kD * 4));
        }
        // start-up barrier, waited on under the first gathers: its payload is the exchange
        // barriers' initialisation, published by thread 0's fence.mbarrier_init (thread 0
        // arrives after it), so the arrive itself needs no release
        ptx::cluster_arrive_relaxed();
    }
    ptx::pdl_wait_prior_grid();
    // RMSNorm weight: async copy, covered by the first chunk's v/g load group
    if (tid < kD / 4) ptx::cp_async16(ptx::smem_u32(&m.w[4 * tid]), p.w + 4 * tid, 16);
    __syncthreads();
    uint32_t tmem = 0, tmem_warp = 0;
    uint32_t it = 0;                  // chunk iterations so far (load-barrier parity)
    uint32_t ph_mma[4] = {0, 0, 0, 0};

    // State rows owned by lanes < 16: state column j = 16*w4 + lane (a row of the transposed
    // state), channels c in [32*ch, 32*ch + 32).
    const bool s_owner = lane < 16;
    const int s_row = w4 * 16 + lane;
    float S[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) S[j] = 0.0f;
    float Sl[32];

    volatile int *abort_flag = &m.abort;
    auto wait_bar = [&](uint64_t *bar, uint32_t parity) { wait_phase(bar, parity, p.wait_limit, abort_flag); };
    // ------------------------------------------------------------ loads
    auto set_rows = [&](int c0, int n, int rb) {
        if (tid < n) {
            const int r = (bb * p.L + spatial_of(dir, c0 + tid, p.gh, p.gw)) * p.H + hh;
            // a gathered or stored token row lies inside the arrays (row 0 stands in otherwise)
            m.rows[rb][tid] = GLA_CHECK(c0 + tid < p.L && r >= 0 && r < p.B * p.L * p.H) ? r : 0;
        }
    };
    // issue the chunk's gathers (fp16 [n rows][64] tiles, rows >= n zero-filled) into the
    // swizzled layout; completion is tracked per group on mbar_ld[0..2]
    // `withhold`: test hook, the q/k group never signals its barrier (its wait then expires)
    auto issue_loads = [&](int n, bool full, int rb, bool withhold) {
        size_t goff[4];
        uint32_t soff[4], bytes[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int row = (tid >> 3) + 32 * i, j = tid & 7;
            const bool ok = row < n;
            goff[i] = ok ? (size_t)m.rows[rb][row] * kD + j * 8 : 0;
            soff[i] = sbase + off_f16(row, j);
            bytes[i] = ok ? 16u : 0u;
        }
        auto tile = [&](const __half *src, uint32_t dst) {
#pragma unroll
            for (int i = 0; i < 4; ++i) ptx::cp_async16(soff[i] + dst, src + goff[i], bytes[i]);
        };
        tile(p.a, kTA);
        ptx::cp_async_mbar_arrive_noinc(&m.mbar_ld[0]);
        tile(p.k, kTK);
        if (full) tile(p.q, kTQ);
        if (!withhold) ptx::cp_async_mbar_arrive_noinc(&m.mbar_ld[1]);
        tile(p.v, kTV);
        if (full) tile(p.g, kTG);
        ptx::cp_async_mbar_arrive_noinc(&m.mbar_ld[2]);
    };
    // ------------------------------------------------------------ gate
    // 16 rows x 2 channels per thread: b = inclusive cumsum of log2(gamma) down the chunk
    auto gate = [&](int n) {
        const int cp = tid & 31, tq = tid >> 5;   // channels 2cp, 2cp+1; rows 16tq..16tq+15
        wait_bar(&m.mbar_ld[0], it & 1);
        float c0s[16], c1s[16];
        float r0 = 0.0f, r1 = 0.0f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int row = tq * 16 + i;
            const __half2 av = *reinterpret_cast<const __half2 *>(sm + kTA + off_f16(row, cp >> 2) +
                                                                  (cp & 3) * 4);
            const float2 af = __half22float2(av);
            const bool ok = row < n;
            r0 += ok ? log2_gamma(af.x) : 0.0f;
            r1 += ok ? log2_gamma(af.y) : 0.0f;
            c0s[i] = r0;
            c1s[i] = r1;
        }
        *reinterpret_cast<float2 *>(&m.tot[tq][2 * cp]) = make_float2(r0, r1);
        __syncthreads();
        float a0 = 0.0f, a1 = 0.0f;
        for (int q = 0; q < tq; ++q) {
            const float2 x = *reinterpret_cast<const float2 *>(&m.tot[q][2 * cp]);
            a0 += x.x;
            a1 += x.y;
        }
        const int c = 2 * cp;
#pragma unroll
        for (int i = 0; i < 16; ++i)
            *reinterpret_cast<float2 *>(sm + kPB + off_tf32(kAtom128, tq * 16 + i, c >> 2) + (c & 3) * 4) =
                make_float2(c0s[i] + a0, c1s[i] + a1);
        __syncthreads();
        if (tid < kD) {
            const float *bp = reinterpret_cast<const float *>(sm + kPB);
            auto bat = [&](int row) { return bp[(off_tf32(kAtom128, row, tid >> 2) >> 2) + (tid & 3)]; };
            const float r = bat((n - 1) >> 1), Bv = bat(n - 1);
            m.bref[tid] = r;
            m.Bc[tid] = Bv;
            if ((bat(0) - r > kHalfRangeSafe2) || (r - Bv > kHalfRangeSafe2)) m.slow = 1;
        }
        __syncthreads();
        if (tid < kD) {
            if (m.slow) m.bref[tid] = 0.0f;           // slow path: chunk-start reference
            const float r = m.bref[tid], Bv = m.Bc[tid];
            m.eB[tid] = ptx::ex2(Bv);
            m.fB[tid] = ptx::ex2(Bv - r);
            m.eref[tid] = ptx::ex2(r);
        }
        __syncthreads();
    };
    // ------------------------------------------------------------ operands (row t, 32 channels)
    // Decayed keys Ks = k 2^{B - b} (fp16, the state product's A operand).  Built first so
    // the segment aggregate can be published before the score operands exist.
    auto build_ks = [&]() {
        wait_bar(&m.mbar_ld[1], it & 1);
#pragma unroll 1
        for (int jj = 0; jj < 4; ++jj) {
            const int j = ch * 4 + jj;             // 16 B chunk of 8 channels
            const uint4 kraw = *reinterpret_cast<const uint4 *>(sm + kTK + off_f16(t, j));
            const __half2 *k2 = reinterpret_cast<const __half2 *>(&kraw);
            float ks[8];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const float4 b4 = *reinterpret_cast<const float4 *>(sm + kPB + off_tf32(kAtom128, t, 2 * j + h));
                const float4 B4 = *reinterpret_cast<const float4 *>(&m.Bc[8 * j + 4 * h]);
                const float2 k01 = __half22float2(k2[2 * h]), k23 = __half22float2(k2[2 * h + 1]);
                ks[4 * h + 0] = k01.x * ptx::ex2(B4.x - b4.x);
                ks[4 * h + 1] = k01.y * ptx::ex2(B4.y - b4.y);
                ks[4 * h + 2] = k23.x * ptx::ex2(B4.z - b4.z);
                ks[4 * h + 3] = k23.y * ptx::ex2(B4.w - b4.w);
            }
            uint4 kso;
            kso.x = pack_half2(ks[0], ks[1]); kso.y = pack_half2(ks[2], ks[3]);
            kso.z = pack_half2(ks[4], ks[5]); kso.w = pack_half2(ks[6], ks[7]);
            *reinterpret_cast<uint4 *>(sm + kST + off_f16(t, j)) = kso;
        }
    };
    // Score operands.  With x = 2^{r - b} (one ex2), Kh/Kl (smem tf32) of K~ = k x and Qh/Ql
    // (TMEM) of Q~ = q / (8 x) (Newton reciprocal; the rounding of x cancels in each product
    // q_tc x^-1 k_sc x), and the exact diagonal q_t . k_t; a chunk beyond the fast operands'
    // range takes build_q_exact.
    auto build_qk = [&]() {
        if (m.slow) {                              // CTA-uniform
            build_q_exact(sm, t, ch, tmem_warp, &m.dqp[ch][t]);
            return;
        }
        float dqs = 0.0f;                          // partial q_t . k_t over this half's channels
#pragma unroll 1
        for (int jj = 0; jj < 4; ++jj) {
            const int j = ch * 4 + jj;
            const uint4 kraw = *reinterpret_cast<const uint4 *>(sm + kTK + off_f16(t, j));
            const uint4 qraw = *reinterpret_cast<const uint4 *>(sm + kTQ + off_f16(t, j));
            const __half2 *k2 = reinterpret_cast<const __half2 *>(&kraw);
            const __half2 *q2 = reinterpret_cast<const __half2 *>(&qraw);
            float bt[8], rr[8], kv[8], qv[8];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const float4 b4 = *reinterpret_cast<const float4 *>(sm + kPB + off_tf32(kAtom128, t, 2 * j + h));
                const float4 r4 = *reinterpret_cast<const float4 *>(&m.bref[8 * j + 4 * h]);
                bt[4 * h] = b4.x; bt[4 * h + 1] = b4.y; bt[4 * h + 2] = b4.z; bt[4 * h + 3] = b4.w;
                rr[4 * h] = r4.x; rr[4 * h + 1] = r4.y; rr[4 * h + 2] = r4.z; rr[4 * h + 3] = r4.w;
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 kf = __half22float2(k2[e]);
                const float2 qf = __half22float2(q2[e]);
                kv[2 * e] = kf.x; kv[2 * e + 1] = kf.y;
                qv[2 * e] = qf.x; qv[2 * e + 1] = qf.y;
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) dqs = fmaf(qv[e], kv[e], dqs);
            // tf32 splits: high = low 13 bits cleared, low = exact remainder (the tensor core
            // drops the low part's own low bits: error <= 2^-20 of the value)
            float qh[8], ql[8], kh[8], kl[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float x = ptx::ex2(rr[e] - bt[e]);
                const float kf = kv[e] * x;                                  // k 2^{r - b}
                const float qf = qv[e] * rcp_nr(x) * 0.125f;                 // q 2^{b - r} / 8
                kh[e] = ptx::tf32_hi(kf);
                kl[e] = kf - kh[e];
                qh[e] = ptx::tf32_hi(qf);
                ql[e] = qf - qh[e];
            }
            ptx::tmem_st8(tmem_warp + kColQH + 8 * j, qh);
            ptx::tmem_st8(tmem_warp + kColQL + 8 * j, ql);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                *reinterpret_cast<float4 *>(sm + kKH + off_tf32(kAtom128, t, 2 * j + h)) =
                    make_float4(kh[4 * h], kh[4 * h + 1], kh[4 * h + 2], kh[4 * h + 3]);
                *reinterpret_cast<float4 *>(sm + kKL + off_tf32(kAtom128, t, 2 * j + h)) =
                    make_float4(kl[4 * h], kl[4 * h + 1], kl[4 * h + 2], kl[4 * h + 3]);
            }
        }
        m.dqp[ch][t] = dqs;
        ptx::tmem_st_wait();
    };
    // ------------------------------------------------------------ MMA issue (one thread)
    // Make every thread's shared-memory operand writes visible to the tensor core, then
    // let thread 0 issue.
    auto operands_ready = [&]() {
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before_sync();
        __syncthreads();
    };
    auto wait_mma = [&](int i) {
        wait_bar(&m.mbar_mma[i], ph_mma[i]);
        ph_mma[i] ^= 1u;
        ptx::tc_fence_after_sync();
    };
    // transposed chunk state (TMEM, M=64 layout) -> registers of the state owners (warp-wide)
    auto read_sloc = [&]() {
        ptx::tmem_ld32(tmem_warp + kColSL + 32 * ch, Sl);
        ptx::tmem_ld_wait();
    };
    // ------------------------------------------------------------ P (row t, 64 columns)
    // P block: columns [s0, s0 + 32) of row t, fp16 into the b region.  The TMEM load is
    // warp-collective (.sync.aligned): it is skipped only when the whole warp's rows lie above
    // the block (a warp-uniform test); pad rows t >= n and entries s > t are zeroed per lane.
    auto p_block = [&](int s0, int n, float dq, float &amax) {
        uint8_t *dst = sm + kPB;
        const int jb = s0 >> 3;
        const bool warp_above = s0 > 32 * w4 + 31;
        float r[32];
        if (!warp_above) {
            ptx::tmem_ld32(tmem_warp + kColDS + s0, r);
            ptx::tmem_ld_wait();
        }
        if (warp_above || s0 > t || t >= n) {
            const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int j4 = 0; j4 < 4; ++j4) *reinterpret_cast<uint4 *>(dst + off_f16k128(t, jb + j4)) = z;
            return;
        }
        if (s0 + 31 >= t) {                            // block holding the diagonal
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const int s = s0 + e;
                r[e] = s < t ? r[e] : (s == t ? dq : 0.0f);
            }
        }
#pragma unroll
        for (int e = 0; e < 32; ++e) amax = fmaxf(amax, fabsf(r[e]));
#pragma unroll
        for (int j4 = 0; j4 < 4; ++j4) {
            uint4 o;
            o.x = pack_half2(r[8 * j4], r[8 * j4 + 1]); o.y = pack_half2(r[8 * j4 + 2], r[8 * j4 + 3]);
            o.z = pack_half2(r[8 * j4 + 4], r[8 * j4 + 5]); o.w = pack_half2(r[8 * j4 + 6], r[8 * j4 + 7]);
            *reinterpret_cast<uint4 *>(dst + off_f16k128(t, jb + j4)) = o;
        }
    };
    // all warps: row t, the 64 columns of this thread's half
    auto make_p_fast = [&](int n) {
        const float dq = (m.dqp[0][t] + m.dqp[1][t]) * p.scale;   // exact diagonal score
        float amax = 0.0f;
#pragma unroll 1
        for (int blk = 0; blk < 2; ++blk) p_block(ch * 64 + 32 * blk, n, dq, amax);
        if (amax > 65504.0f) m.range_err = 1;
    };
    // S~[c][j] = tf32(2^{r_c} S[c][j]) from the state owners' registers (value column j, key
    // channels 32ch..32ch+31); 16 consecutive j per warp fill 64 contiguous bytes of a row
    auto write_stilde = [&]() {
        if (s_owner) {
#pragma unroll
            for (int k = 0; k < 32; ++k) {
                const int c = 32 * ch + k;
                *reinterpret_cast<float *>(sm + kTA + off_stilde(c, s_row)) = ptx::to_tf32(S[k] * m.eref[c]);
            }
        }
    };
    // SiLU(g) * w for row t, channel chunks [j0, j1) of 8, into TMEM (read by the epilogue).
    // Run while the score products execute, by warps of this row's TMEM lane quarter.
    auto prep_sg = [&](int j0, int j1) {
        wait_bar(&m.mbar_ld[2], it & 1);               // g tile
#pragma unroll 2
        for (int j = j0; j < j1; ++j) {
            const uint4 graw = *reinterpret_cast<const uint4 *>(sm + kTG + off_f16(t, j));
            const __half2 *g2 = reinterpret_cast<const __half2 *>(&graw);
            const float4 wa = *reinterpret_cast<const float4 *>(&m.w[8 * j]);
            const float4 wb = *reinterpret_cast<const float4 *>(&m.w[8 * j + 4]);
            const float wv[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
            float sg[8];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 gf = __half22float2(g2[e]);
                sg[2 * e] = wv[2 * e] * silu_fast(gf.x);
                sg[2 * e + 1] = wv[2 * e + 1] * silu_fast(gf.y);
            }
            ptx::tmem_st8(tmem_warp + kColSG + 8 * j, sg);
        }
        ptx::tmem_st_wait();
    };
    // u = (O_inter + O_intra) / rms * SiLU(g) * w.  Row t, 32 channels per thread, staged as
    // fp16 rows in the K~ low-part region (free once the score products completed), then
    // stored with each group of 8 threads writing one whole 128-byte token row.  A row's two
    // halves live in warps w4 and w4 + 4, which synchronise on named barrier 1 + w4 only.
    auto epilogue = [&](int n, int rb) {
        float o[32], op[32];
        ptx::tmem_ld32(tmem_warp + kColO + 32 * ch, o);
        ptx::tmem_ld32(tmem_warp + kColOP + 32 * ch, op);
        ptx::tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 32; ++j) o[j] += op[j];
        float ss = 0.0f;
#pragma unroll
        for (int j = 0; j < 32; ++j) ss = fmaf(o[j], o[j], ss);
        m.red[ch][t] = ss;
        ptx::tmem_ld32(tmem_warp + kColSG + 32 * ch, op);
        ptx::tmem_ld_wait();
        ptx::named_bar_sync(1 + w4, 64);
        const float inv = rsqrtf((m.red[0][t] + m.red[1][t]) * (1.0f / 64.0f) + p.eps);
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            float u[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) u[e] = o[8 * jj + e] * inv * op[8 * jj + e];
            uint4 pk;
            pk.x = pack_half2(u[0], u[1]); pk.y = pack_half2(u[2], u[3]);
            pk.z = pack_half2(u[4], u[5]); pk.w = pack_half2(u[6], u[7]);
            *reinterpret_cast<uint4 *>(sm + kKL + off_f16(t, 4 * ch + jj)) = pk;
        }
        ptx::named_bar_sync(1 + w4, 64);
        const int pt = (ch << 5) | lane;                // 0..63 within the warp pair
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int row = 32 * w4 + (pt >> 3) + 8 * i, j = pt & 7;
            if (row < n)
                *reinterpret_cast<uint4 *>(p.out + (size_t)m.rows[rb][row] * kD + 8 * j) =
                    *reinterpret_cast<const uint4 *>(sm + kKL + off_f16(row, j));
        }
    };
    // fold the chunk's local state into S: S = S Diag(2^{B}) + Sloc (transposed form)
    auto fold_sloc = [&](bool into_g) {
        if (s_owner) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float4 e4 = *reinterpret_cast<const float4 *>(&m.eB[32 * ch + 4 * i]);
                S[4 * i] = fmaf(e4.x, S[4 * i], Sl[4 * i]);
                S[4 * i + 1] = fmaf(e4.y, S[4 * i + 1], Sl[4 * i + 1]);
                S[4 * i + 2] = fmaf(e4.z, S[4 * i + 2], Sl[4 * i + 2]);
                S[4 * i + 3] = fmaf(e4.w, S[4 * i + 3], Sl[4 * i + 3]);
            }
        }
        if (into_g && tid < kD) m.Gs[tid] += m.Bc[tid];
    };
    // Cluster-wide scan of the segment aggregates (Gs, S): every segment receives its
    // incoming state.  The scan is elementwise per state entry (j, c) with the decay of key
    // channel c, so it is split by channel groups: scanner r owns groups g = r + lg*segs.
    // Forward: the state owners store each 4-channel piece of their row straight from
    // registers into the group's scanner, and 32 threads store the 2^{G} and 2^{r} pieces
    // (st.async, bytes counted on the receiver's mbar_x[0]); receive layout
    // [lg][segment][66 rows][4] fp32, aggregate row j in slot recv_slot(j), then the 2^{G} and
    // 2^{r} rows.  Return: a scanner combines the segments in order and stores each segment's
    // result, as soon as it is produced, into that segment's operand region (S~, MN-major, in
    // the a tile, direct) or channel-major into the g tile (S_in, before a multi-chunk pass),
    // counted on the receiver's mbar_x[1].  Every remote region written is
    // idle at its owner by then: a CTA's a and g tiles are consumed before it publishes its
    // aggregate, and results follow the aggregates.
    bool cluster_ready = false;
    auto cluster_ready_once = [&]() {                 // every CTA's exchange barriers exist
        if (!cluster_ready) ptx::cluster_wait();
        cluster_ready = true;
    };
    auto recv_off = [&](int lg, int seg, int row) {
        const uint32_t o = (uint32_t)(((lg * p.segs + seg) * kGroupRows + row) * 16);
        // a receive slot lies inside the receive region (its first slot stands in otherwise)
        return kRECV + (GLA_CHECK(row < kGroupRows && o + 16 <= kRecvBytes) ? o : 0u);
    };
    auto xchg_begin = [&]() {
        cluster_ready_once();
        // each state row is held by lanes 0..15 (32 channels per warp); lanes 16..31 take the
        // upper 16 channels of lane - 16's row so every store instruction uses the whole warp
        float hi[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) hi[k] = __shfl_sync(0xffffffffu, S[16 + k], lane & 15);
        const int row = w4 * 16 + (lane & 15), i0 = lane < 16 ? 0 : 4;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int g = 8 * ch + i0 + i, dst = g % p.segs;
            const float4 v = lane < 16 ? make_float4(S[4 * i], S[4 * i + 1], S[4 * i + 2], S[4 * i + 3])
                                       : make_float4(hi[4 * i], hi[4 * i + 1], hi[4 * i + 2], hi[4 * i + 3]);
            ptx::st_async_v4(ptx::mapa(sbase + recv_off(g / p.segs, rank, recv_slot(row)), dst), v,
                             ptx::mapa(ptx::smem_u32(&m.mbar_x[0]), dst));
        }
        // the group pieces of 2^{G} and 2^{r}.  G of a one-chunk segment is its B (the gate's
        // row, barrier-separated from here); of a longer segment the sum over its state-only
        // pass, complete since that pass's last barrier
        if (tid < 32) {
            const int g = tid & 15, dst = g % p.segs;
            float4 v;
            if (tid < 16) {
                const float *gs = resident ? m.Bc : m.Gs;
                v = make_float4(ptx::ex2(gs[4 * g]), ptx::ex2(gs[4 * g + 1]), ptx::ex2(gs[4 * g + 2]),
                                ptx::ex2(gs[4 * g + 3]));
            } else {
                v = *reinterpret_cast<const float4 *>(m.eref + 4 * g);
            }
            ptx::st_async_v4(ptx::mapa(sbase + recv_off(g / p.segs, rank, kD + (tid >> 4)), dst), v,
                             ptx::mapa(ptx::smem_u32(&m.mbar_x[0]), dst));
        }
    };
    // Scan of the received aggregates by warps 0..3.  An item is (owned group, key channel c,
    // quad of value columns j0..j0+3); its chain runs over the segments in order and the state
    // entering each segment is stored, as one 16-byte piece of that segment's S~ row c (or
    // S_in row c), as soon as it is produced.  A warp covers 8 quads x 4 channels, i.e. four
    // whole 128-byte destination rows per store.
    auto xchg_scan = [&](bool direct) {
        if (warp >= 4) return;                        // warp-uniform
        wait_cluster_phase(&m.mbar_x[0], 0, p.wait_limit, abort_flag);
        const int segs = p.segs;
        const uint32_t lbar = ptx::smem_u32(&m.mbar_x[1]);
        for (int idx = tid; idx < my_groups * kD; idx += 128) {
            const int lg = idx >> 6, jq = (idx >> 2) & 15, cl = idx & 3;
            const int c = 4 * (lg * segs + rank) + cl, j0 = 4 * jq;
            const uint32_t laddr = sbase + (direct ? kTA + off_stilde(c, j0) : kTG + c * 256 + j0 * 4);
            uint32_t rs[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) rs[i] = recv_slot(j0 + i) * 16 + cl * 4;
            float4 run = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll 2
            for (int q = 0; q < segs; ++q) {
                const uint8_t *blk = sm + recv_off(lg, q, 0);
                const float4 agg = make_float4(*reinterpret_cast<const float *>(blk + rs[0]),
                                               *reinterpret_cast<const float *>(blk + rs[1]),
                                               *reinterpret_cast<const float *>(blk + rs[2]),
                                               *reinterpret_cast<const float *>(blk + rs[3]));
                const float g = *reinterpret_cast<const float *>(blk + kD * 16 + cl * 4);
                float4 out = run;                      // state entering segment q
                if (direct) {
                    const float f = *reinterpret_cast<const float *>(blk + (kD + 1) * 16 + cl * 4);
                    out = make_float4(ptx::to_tf32(f * run.x), ptx::to_tf32(f * run.y),
                                      ptx::to_tf32(f * run.z), ptx::to_tf32(f * run.w));
                }
                ptx::st_async_v4(ptx::mapa(laddr, q), out, ptx::mapa(lbar, q));
                run = make_float4(fmaf(g, run.x, agg.x), fmaf(g, run.y, agg.y),
                                  fmaf(g, run.z, agg.z), fmaf(g, run.w, agg.w));
            }
        }
    };
    // wait for this CTA's incoming state S_in (channel-major, g tile) before a multi-chunk pass
    // and read it back into the state owners' registers
    auto xchg_wait_sin = [&]() {
        wait_cluster_phase(&m.mbar_x[1], 0, p.wait_limit, abort_flag);
        if (s_owner) {
            const float *Sin = reinterpret_cast<const float *>(sm + kTG);
#pragma unroll
            for (int k = 0; k < 32; ++k) S[k] = Sin[(32 * ch + k) * kD + s_row];
        }
        __syncthreads();
    };

    // ------------------------------------------------------------ schedule
    // Non-resident segments run a state-only pass first (all ranks but the last), then the
    // exchange, then the full pass; a resident segment (one chunk) runs the full pass once
    // and exchanges mid-chunk.  Every CTA exchanges exactly once.
    const int n_pass1 = (!kMid && !resident && exchange && rank < p.segs - 1) ? n_chunks : 0;
    // Within a pass, the next chunk's gathers are issued as soon as this chunk's tiles are
    // free (after the state product in the state-only pass, after the last products in the
    // full pass), into the other row-index buffer; never across the exchange, which writes
    // S_in into the g tile.
    int rb = 0;                        // row-index buffer of the current chunk
    bool preloaded = false;            // its gathers were issued during the previous chunk
    auto preload_next = [&](int ci, bool full) {
        if (ci + 1 >= n_chunks) return;
        const int c1 = p0 + (ci + 1) * chunk_len;
        const int n1 = min(chunk_len, p1 - c1);
        set_rows(c1, n1, rb ^ 1);
        __syncthreads();
        issue_loads(n1, full, rb ^ 1, full && ci + 1 == p.fault_chunk);
        preloaded = true;
    };
    for (int step = 0; step < n_pass1 + n_chunks; ++step) {
        const bool pass1 = step < n_pass1;
        const int ci = pass1 ? step : step - n_pass1;
        if (!kMid && !pass1 && ci == 0 && !resident && exchange) {
            xchg_begin();
            xchg_scan(false);
            xchg_wait_sin();
        }
        int n;
        {
            const int c0 = p0 + ci * chunk_len;
            n = min(chunk_len, p1 - c0);
            if (!preloaded) {
                __syncthreads();
                set_rows(c0, n, rb);
                __syncthreads();
                issue_loads(n, !pass1, rb, !pass1 && ci == p.fault_chunk);
            }
            preloaded = false;
            if (tid == 0) m.slow = 0;               // read only after the gate's barriers
        }
        if (step == 0 && warp == 0) {                // overlaps the first gathers' latency
            ptx::tmem_alloc(&m.tmem_base, kTmemCols);
            ptx::tmem_relinquish();
            ptx::tc_fence_before_sync();
        }
        if (step == 0 && exchange) cluster_ready_once();   // under the first gathers' latency
        gate(n);                                     // contains block barriers
        if (step == 0) {
            ptx::tc_fence_after_sync();
            tmem = m.tmem_base;
            tmem_warp = tmem + ((uint32_t)(w4 * 32) << 16);
        }
        build_ks();
        wait_bar(&m.mbar_ld[2], it & 1);             // V, an operand of the state product
        operands_ready();
        // The state product goes first: the segment aggregate is published while the score
        // products run.  The issuing thread stalls while its products drain, so the score
        // products are issued only after this CTA has arrived on the cluster barrier.
        if (warp == 0 && ptx::elect_one()) {
            ptx::tc_fence_after_sync();
            if (!*abort_flag) issue_state(sbase, tmem);
            ptx::mma_commit(&m.mbar_mma[0]);
        }
        wait_mma(0);
        const bool mid_xchg = kMid || (!pass1 && resident && exchange);
        if (!kMid && pass1) preload_next(ci, false);   // a, k, v consumed
        read_sloc();
        if (pass1 || mid_xchg) fold_sloc(true);     // S = S 2^{B} + Sloc, Gs += B
        if (pass1) {
            ptx::tc_fence_before_sync();
            __syncthreads();
            ++it;
            rb ^= preloaded ? 1 : 0;
            continue;
        }
        // publish the segment aggregate now: the exchange runs under the score operands and
        // the score products
        if (mid_xchg) xchg_begin();
        build_qk();
        operands_ready();
        // score products, issued by warp 7; meanwhile the scanning warps store the segment
        // states and the other warps compute SiLU(g) * w for their TMEM lane quarters
        if (warp == 7 && ptx::elect_one()) {
            ptx::tc_fence_after_sync();
            if (!m.slow && !*abort_flag) issue_qk(sbase, tmem, min(kC, (n + 15) & ~15));
            ptx::mma_commit(&m.mbar_mma[1]);
        }
        if (mid_xchg) {
            xchg_scan(true);
            if (warp == 3 || (warp >= 4 && warp < 7)) prep_sg(0, 8);
        } else {
            if (warp == 3) prep_sg(0, 8);            // no scan: each warp its own channel half,
            else if (warp != 7) prep_sg(4 * ch, 4 * ch + 4);   // warp 3 also the issuer's
            write_stilde();                          // S~ from the state entering this chunk,
            if (!kMid && ci + 1 < n_chunks)          // then S = S 2^{B} + Sloc for the next
                fold_sloc(false);
            ptx::fence_proxy_async_smem();
        }
        wait_mma(1);
        if (!mid_xchg) {
            // the inter product by warp 4 while the others build P (warp 4's rows 0..31 need
            // no column of P past 31: its share is zero fill)
            ptx::tc_fence_before_sync();
            __syncthreads();                         // S~ complete
            if (warp == 4 && ptx::elect_one()) {
                ptx::tc_fence_after_sync();
                if (!*abort_flag) issue_inter(sbase, tmem, false);
                ptx::mma_commit(&m.mbar_mma[2]);
            }
        }
        if (m.slow) make_p_exact(sm, t, ch, n, p.scale, &m.range_err);
        else make_p_fast(n);
        operands_ready();
        if (mid_xchg) {
            // P.V by warp 0; the inter product by warp 4 as soon as S~ has arrived (its bytes
            // are counted on mbar_x[1]; the proxy fence orders them before the tensor core reads)
            if (warp == 0 && ptx::elect_one()) {
                ptx::tc_fence_after_sync();
                if (!*abort_flag) issue_pv(sbase, m.slow ? kKH : kPB, tmem);
                ptx::mma_commit(&m.mbar_mma[3]);
            } else if (warp == 4 && ptx::elect_one()) {
                wait_cluster_phase(&m.mbar_x[1], 0, p.wait_limit, abort_flag);
                ptx::fence_proxy_async_smem();
                ptx::tc_fence_after_sync();
                if (!*abort_flag) issue_inter(sbase, tmem, false);
                ptx::mma_commit(&m.mbar_mma[2]);
            }
            wait_mma(3);
        } else {
            if (warp == 0 && ptx::elect_one()) {
                ptx::tc_fence_after_sync();
                if (!*abort_flag) issue_pv(sbase, m.slow ? kKH : kPB, tmem);
                ptx::mma_commit(&m.mbar_mma[3]);
            }
            wait_mma(3);
        }
        wait_mma(2);
        if (!kMid) preload_next(ci, true);           // every tile consumed (all products done)
        epilogue(n, rb);
        ptx::tc_fence_before_sync();
        __syncthreads();
        ++it;
        rb ^= preloaded ? 1 : 0;
    }

    // ---- teardown ----
    __syncthreads();
    if (*abort_flag) {
        // a wait expired: copies, remote stores and products already in flight land before the
        // shared memory and TMEM are released (bounded again; the status is already latched)
        volatile int no_abort = 0;
        asm volatile("cp.async.wait_all;" ::: "memory");
        if ((warp == 0 || warp == 4 || warp == 7) && ptx::elect_one()) ptx::mma_commit(&m.mbar_end);
        if (tid == 0) {
            wait_phase(&m.mbar_end, 0, p.wait_limit, &no_abort);
            if (exchange) {
                wait_cluster_phase(&m.mbar_x[0], 0, p.wait_limit, &no_abort);
                wait_cluster_phase(&m.mbar_x[1], 0, p.wait_limit, &no_abort);
            }
        }
        __syncthreads();
    }
    // every CTA of the cluster reaches this barrier, so none leaves while another may still
    // store into its shared memory
    if (exchange) {
        ptx::cluster_arrive_release();
        ptx::cluster_wait();
    }
    if (tid == 0 && m.range_err) raise_status(8 /* GLA_ERR_RANGE */);
    ptx::tc_fence_after_sync();
    if (warp == 0 && n_pass1 + n_chunks > 0) ptx::tmem_dealloc(tmem, kTmemCols);
}

// ------------------------------------------------------------- launch floor
// Does nothing but the programmatic-dependent-launch handshake of gla_tc_kernel; launched
// with that kernel's exact shape it measures the per-launch cost no work can remove.
__global__ void __launch_bounds__(kThreads, 1) gla_empty_kernel() {
    ptx::pdl_launch_dependents();
    ptx::pdl_wait_prior_grid();
}

// ------------------------------------------------------------- timeout self-test
// One thread waits, with the kernel's bounded-wait loop but a caller-given bound, on an
// mbarrier that nothing ever arrives on: the wait must expire, latch GLA_ERR_TIMEOUT in
// the device status word and return, leaving the context usable.
__global__ void gla_timeout_selftest_kernel(long long limit_cycles) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        ptx::mbar_init(&bar, 1);
        ptx::fence_mbarrier_init();
        const long long start = clock64();
        while (!ptx::mbar_try_wait(&bar, 0)) {
            if (clock64() - start > limit_cycles) {
                raise_status(7 /* GLA_ERR_TIMEOUT */);
                break;
            }
        }
    }
}

// ------------------------------------------------------- reciprocal self-test
// y[i] = rcp_nr(x[i]): the kernel's Newton reciprocal, for an error-bound test against 1/x.
__global__ void gla_rcp_selftest_kernel(const float *x, float *y, int n) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) y[i] = rcp_nr(x[i]);
}

// ---------------------------------------------------------------- self-test
// Runs one of the kernel's four MMA configurations on row-major fp32 inputs
// (converted to the operand type in the same shared-memory layouts) and
// writes D row-major: 0 = scores (split tf32, A[128][64] . B[128][64]^T -> [128][128]),
// 1 = state (f16, B[128][64]^T . A[128][64] -> [64][64]), 2 = PV (f16,
// A[128][128] . B[128][64] -> [128][64]), 3 = inter (tf32, A[128][64] .
// B[64][64]^T -> [128][64]).  One CTA of kSelfThreads = 128 threads.
__global__ void __launch_bounds__(kSelfThreads, 1)
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
        ptx::mbar_init(&m.mbar_mma[0], 1);
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
                make_float4(src[4 * c4], src[4 * c4 + 1], src[4 * c4 + 2], src[4 * c4 + 3]);
    };
    auto put_f16 = [&](uint32_t region, int row, const float *src) {
        for (int j = 0; j < 8; ++j) {
            uint4 o;
            o.x = pack_half2(src[8 * j], src[8 * j + 1]); o.y = pack_half2(src[8 * j + 2], src[8 * j + 3]);
            o.z = pack_half2(src[8 * j + 4], src[8 * j + 5]); o.w = pack_half2(src[8 * j + 6], src[8 * j + 7]);
            *reinterpret_cast<uint4 *>(sm + region + off_f16(row, j)) = o;
        }
    };
    // split a row into tf32 high/low parts exactly as the kernel's score operands are built:
    // high = the value with its low 13 mantissa bits cleared, low = the exact remainder (the
    // tensor core drops the remainder's own low bits).  Kind 3 (no low part) rounds to tf32.
    auto put_split_tmem = [&](const float *src, bool with_low) {
        for (int j = 0; j < 8; ++j) {
            float h[8], l[8];
            for (int e = 0; e < 8; ++e) {
                const float x = src[8 * j + e];
                h[e] = with_low ? ptx::tf32_hi(x) : ptx::to_tf32(x);
                l[e] = with_low ? x - h[e] : 0.0f;
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
            hi[c] = ptx::tf32_hi(Bm[t * 64 + c]);
            lo[c] = Bm[t * 64 + c] - hi[c];
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
        if (t < 64) {                                  // B row j = t, MN-major (S~ layout)
            for (int c = 0; c < 64; ++c)
                *reinterpret_cast<float *>(sm + kTA + off_stilde(c, t)) = ptx::to_tf32(Bm[t * 64 + c]);
        }
    }
    ptx::fence_proxy_async_smem();
    ptx::tc_fence_before_sync();
    __syncthreads();
    if (tid == 0) {
        ptx::tc_fence_after_sync();
        if (kind == 0) issue_qk(sbase, tmem, kC);
        else if (kind == 1) issue_state(sbase, tmem);
        else if (kind == 2) issue_pv(sbase, kPB, tmem);
        else issue_inter(sbase, tmem, false);
        ptx::mma_commit(&m.mbar_mma[0]);
    }
    volatile int no_abort = 0;
    wait_phase(&m.mbar_mma[0], 0, 1LL << 32, &no_abort);
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
        const uint32_t col = kind == 2 ? kColOP : kColO;
        ptx::tmem_ld32(tmem_warp + col, r0);
        ptx::tmem_ld32(tmem_warp + col + 32, r1);
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
