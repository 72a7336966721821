// gla_gate.cuh -- the retention gate's low-rank projection a = x W1 W2 + b on tcgen05 tensor
// cores (fp16 I/O, fp32 accumulation).
//
// Operation (GTR paper, arXiv 2609.26590, method section, GLA recurrence paragraph): the key-wise
// retention gate is gamma_t = sigma(x_t W_alpha^(1) W_alpha^(2) + b_alpha)^(1/tau), a low-rank
// projection of rank r = 16 built as GLA builds it: one first factor W1 [d][16] shared by the heads, a
// second factor W2 [16][n] onto every head's key channels (n = H d_k), a bias per key channel.
// The output a [T][n] is the operator's gate_preact input, [B][L][H][d_k].
//
// Per 128-token tile (one M = 128 tcgen05 tile):
//   T  = X W1          d / 16 MMAs (K = 16, N = 16), X streamed through a TMA ring of 64-channel
//                      K-blocks, W1 resident (K-major)                    -> TMEM, fp32, 2 buffers
//   T  = Th + Tl       split to fp16 high / low on CUDA cores, back into TMEM as the A operand
//   D  = Th W2 + Tl W2 two MMAs per 128-column chunk of n (W2 resident, MN-major), into one of
//                      two TMEM buffers, so a chunk's epilogue overlaps the next chunk's products
//   a  = fp16(D + b)   epilogue (thread = token row) into a 128-byte swizzled staging tile,
//                      written out by TMA stores (rows past the last token are clipped by TMA)
// The split keeps the second product exact to ~2^-22 relative; only the output rounding remains.
//
// Work split: the (tile, output chunk) units in order, cut into equal contiguous ranges, one per
// CTA, so every CTA has the same number of output chunks to within one whatever the tile count
// (no partial last wave).  A CTA computes X W1 once for each tile its range touches; a tile
// shared by two ranges is read twice, the second time mostly from L2.
//
// Roles (352 threads, one CTA per SM): warps 0-7 epilogue and the one-time staging of W1 / W2 /
// b (warp w reads TMEM lanes 32 (w % 4) .. +31 = tile rows, output columns 64 (w / 4) .. +63 of
// each chunk, i.e. one TMA box; two warps per sub-partition keep the TMEM-load -> convert ->
// store chains overlapped), warp 8 TMA producer, warp 9 issues X W1, warp 10 issues the W2
// products.  The X stream and X W1 run up to two tiles ahead of the epilogue (T is double
// buffered), so loads never wait for the output side; the producer starts before the weights
// are staged.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>

#include "gla_common.cuh"
#include "gla_ptx.cuh"

namespace gla {
namespace gp {

constexpr int kRank = 16;
constexpr int kTileM = 128;
constexpr int kThreads = 352;
constexpr int kEpi = 256;                       // epilogue threads (warps 0-7)
constexpr int kMaxStages = 8;                   // X ring: [128 rows][64 channels] fp16 K-blocks
constexpr uint32_t kBlk = kTileM * 128;         // 16 KB
constexpr uint32_t kOBuf = 2 * kBlk;            // output staging: [2 boxes][128 rows][128 B]
constexpr int kMaxD = 1024, kMaxN = 1024;
// TMEM columns: T[b] at 16 b, Th[b] / Tl[b] at 32 + 16 b (+ 8), D[db] at 256 + 128 db
constexpr uint32_t kColT = 0, kColTs = 32, kColD = 256, kChunkN = 128;
constexpr uint32_t kTmemCols = 512;

struct GateMisc {
    uint64_t xfull[kMaxStages], xempty[kMaxStages];
    uint64_t tdone[2], tfree[2], t16[2], dfull[2], dempty[2], end_t, end_d;
    uint32_t tmem_base;
    int abort, range_err;
    alignas(16) float bias[kMaxN];
};

// Shared-memory layout for widths d, n: resident W1 (d / 64 blocks of 2 KB, K-major) and W2
// (n / 64 blocks, MN-major), two output staging buffers, then as many ring stages as fit
// (at least 3).  Offsets are from the 1024-aligned base; `bytes` includes the alignment slack.
struct GateLayout {
    uint32_t w1, w2, o, x, misc, bytes;
    int stages;
};

__host__ __device__ inline GateLayout gate_layout(int d, int n, size_t smem_cap) {
    GateLayout L;
    L.w1 = 0;
    L.w2 = L.w1 + (uint32_t)(d / 64) * 2048u;
    L.o = L.w2 + (uint32_t)(n / 64) * 2048u;
    L.x = L.o + 2 * kOBuf;
    const size_t fixed = (size_t)L.x + sizeof(GateMisc) + 1024;
    const long long fit = smem_cap > fixed ? (long long)((smem_cap - fixed) / kBlk) : 0;
    L.stages = (int)(fit < kMaxStages ? fit : kMaxStages);
    L.misc = L.x + (uint32_t)(L.stages > 0 ? L.stages : 0) * kBlk;
    L.bytes = L.misc + (uint32_t)sizeof(GateMisc) + 1024u;
    return L;
}

struct GateParams {
    const __half *w1, *w2;
    const float *b;                             // the output a goes through its tensor map
    int T, d, n;
    GateLayout lay;
    long long wait_limit;
};

__device__ __forceinline__ bool gate_wait(uint64_t *bar, uint32_t parity, long long limit,
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

__global__ void __launch_bounds__(kThreads, 1)
    gla_gate_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap amap,
                    const GateParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
    const uint32_t sbase = ptx::smem_u32(sm);
    const GateLayout &L = p.lay;
    const int S = L.stages;
    GateMisc &m = *reinterpret_cast<GateMisc *>(sm + L.misc);
    volatile int *abort_flag = &m.abort;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int kb_n = p.d / 64, nchunks = p.n / kChunkN;
    const int tiles = (p.T + kTileM - 1) / kTileM;
    auto wait = [&](uint64_t *bar, int use) { return gate_wait(bar, (uint32_t)(use & 1), p.wait_limit, abort_flag); };
    // this CTA's units [u0, u1) of the tiles x nchunks (tile, chunk) sequence; tiles
    // [tile_lo, tile_hi] and, per tile, output chunks [c0, c1)
    const long long units = (long long)tiles * nchunks;
    const int u0 = (int)(units * blockIdx.x / gridDim.x), u1 = (int)(units * (blockIdx.x + 1) / gridDim.x);
    const int tile_lo = u0 / nchunks, tile_hi = u1 > u0 ? (u1 - 1) / nchunks : tile_lo - 1;
    auto chunk_range = [&](int tile, int &c0, int &c1) {
        c0 = max(u0, tile * nchunks) - tile * nchunks;
        c1 = min(u1, (tile + 1) * nchunks) - tile * nchunks;
    };

    ptx::pdl_launch_dependents();
    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            ptx::mbar_init(&m.xfull[s], 1);
            ptx::mbar_init(&m.xempty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(&m.tdone[i], 1);
            ptx::mbar_init(&m.tfree[i], 1);
            ptx::mbar_init(&m.t16[i], 1);
            ptx::mbar_init(&m.dfull[i], 1);
            ptx::mbar_init(&m.dempty[i], 1);
        }
        ptx::mbar_init(&m.end_t, 1);
        ptx::mbar_init(&m.end_d, 1);
        ptx::fence_mbarrier_init();
        m.abort = 0;
        m.range_err = 0;
    }
    if (warp == 0) {
        ptx::tmem_alloc(&m.tmem_base, kTmemCols);
        ptx::tmem_relinquish();
    }
    if (warp == 8 && lane == 0) {
        ptx::prefetch_tmap(&xmap);
        ptx::prefetch_tmap(&amap);
    }
    ptx::tc_fence_before_sync();
    __syncthreads();
    ptx::tc_fence_after_sync();
    const uint32_t tmem = m.tmem_base;
    ptx::pdl_wait_prior_grid();

    if (warp < 8) {
        // resident operands: W1 transposed to K-major [16 rows (r)][d (k)], W2 as MN-major
        // [16 rows (r)][n (c)], both in 128-byte swizzled 2 KB blocks of 64 columns.  Every
        // global read is one 16-byte cp.async issued up front (W1 lands raw in the output
        // staging buffers, free until the first chunk, and is transposed from there), so
        // staging costs one memory latency, under the first X loads.
        for (int e = tid; e < p.d * kRank / 8; e += kEpi)
            if (GLA_CHECK(16u * e + 16u <= 2 * kOBuf)) ptx::cp_async16(sbase + L.o + 16 * e, p.w1 + 8 * (size_t)e, 16);
        for (int e = tid; e < kRank * p.n / 8; e += kEpi) {     // 8 consecutive c of one row r
            const int r = e / (p.n / 8), c0 = 8 * (e % (p.n / 8));
            ptx::cp_async16(sbase + L.w2 + (c0 / 64) * 2048 + ptx::sw128(r, (c0 % 64) / 8),
                            p.w2 + (size_t)r * p.n + c0, 16);
        }
        for (int e = tid; e < p.n / 4; e += kEpi) ptx::cp_async16(ptx::smem_u32(&m.bias[4 * e]), p.b + 4 * e, 16);
        ptx::cp_async_wait_all();
        ptx::named_bar_sync(1, kEpi);
        const __half *raw = reinterpret_cast<const __half *>(sm + L.o);   // [d][16]
        for (int e = tid; e < p.d * kRank / 8; e += kEpi) {     // 8 consecutive k of one row r
            const int r = e % kRank, k0 = 8 * (e / kRank);
            __align__(16) __half v[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] = raw[(k0 + i) * kRank + r];
            *reinterpret_cast<uint4 *>(sm + L.w1 + (k0 / 64) * 2048 + ptx::sw128(r, (k0 % 64) / 8)) =
                *reinterpret_cast<const uint4 *>(v);
        }
        ptx::fence_proxy_async_smem();
        ptx::named_bar_sync(1, kEpi);                           // raw W1 read before staging reuse
        ptx::named_bar_sync(2, kEpi + 64);                      // weights staged (with warps 9, 10)

        // ===================================================================== epilogue
        const int quarter = warp & 3, half = warp >> 2;
        const int row = 32 * quarter + lane;                    // tile row = TMEM lane
        const uint32_t lanes = (uint32_t)(32 * quarter) << 16;
        int t = 0, q = 0;
        for (int tile = tile_lo; tile <= tile_hi; ++tile, ++t) {
            const int b = t & 1;
            int c0, c1;
            chunk_range(tile, c0, c1);
            if (half == 0) {                                    // warps 0-3 split T
                wait(&m.tdone[b], t >> 1);
                ptx::tc_fence_after_sync();
                float tv[16];
                ptx::tmem_ld16(tmem + lanes + kColT + 16 * b, tv);
                ptx::tmem_ld_wait();
                float hi[8], lo[8];
                float amax = 0.0f;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const __half2 h = __floats2half2_rn(tv[2 * i], tv[2 * i + 1]);
                    const float2 hf = __half22float2(h);
                    const __half2 l = __floats2half2_rn(tv[2 * i] - hf.x, tv[2 * i + 1] - hf.y);
                    hi[i] = __uint_as_float(*reinterpret_cast<const uint32_t *>(&h));
                    lo[i] = __uint_as_float(*reinterpret_cast<const uint32_t *>(&l));
                    amax = fmaxf(amax, fmaxf(fabsf(tv[2 * i]), fabsf(tv[2 * i + 1])));
                }
                if (amax > 65504.0f) m.range_err = 1;
                ptx::tmem_st8(tmem + lanes + kColTs + 16 * b, hi);
                ptx::tmem_st8(tmem + lanes + kColTs + 16 * b + 8, lo);
                ptx::tmem_st_wait();
            }
            ptx::tc_fence_before_sync();
            ptx::named_bar_sync(1, kEpi);
            if (tid == 0) {
                ptx::mbar_arrive(&m.t16[b]);                    // Th, Tl ready for the W2 products
                ptx::mbar_arrive(&m.tfree[b]);                  // T[b] read: X W1 may reuse it
            }
            for (int c = c0; c < c1; ++c, ++q) {
                const int db = q & 1;                           // TMEM buffer = staging buffer
                const uint32_t obuf = sbase + L.o + db * kOBuf;
                wait(&m.dfull[db], q >> 1);
                ptx::tc_fence_after_sync();
                // this warp's 64 columns of the chunk: both TMEM loads in flight, one wait
                float v0[32], v1[32];
                const uint32_t taddr = tmem + lanes + kColD + db * kChunkN + 64 * half;
                ptx::tmem_ld32(taddr, v0);
                ptx::tmem_ld32(taddr + 32, v1);
                ptx::tmem_ld_wait();
                const float4 *bias4 = reinterpret_cast<const float4 *>(&m.bias[c * (int)kChunkN + 64 * half]);
                // staging box `half`, row `row`, 16-byte pieces j = 0..7 (8 columns each)
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float *v = j < 4 ? &v0[8 * j] : &v1[8 * (j - 4)];
                    const float4 ba = bias4[2 * j], bb = bias4[2 * j + 1];
                    const __half2 o0 = __floats2half2_rn(v[0] + ba.x, v[1] + ba.y);
                    const __half2 o1 = __floats2half2_rn(v[2] + ba.z, v[3] + ba.w);
                    const __half2 o2 = __floats2half2_rn(v[4] + bb.x, v[5] + bb.y);
                    const __half2 o3 = __floats2half2_rn(v[6] + bb.z, v[7] + bb.w);
                    const uint32_t off = half * kBlk + ptx::sw128(row, j);
                    if (GLA_CHECK(off + 16 <= kOBuf))
                        *reinterpret_cast<uint4 *>(sm + (obuf - sbase) + off) =
                            make_uint4(*reinterpret_cast<const uint32_t *>(&o0), *reinterpret_cast<const uint32_t *>(&o1),
                                       *reinterpret_cast<const uint32_t *>(&o2), *reinterpret_cast<const uint32_t *>(&o3));
                }
                ptx::tc_fence_before_sync();
                ptx::fence_proxy_async_smem();
                // the previous chunk's TMA store has read the other staging buffer, which the
                // next chunk writes
                if (tid == 0) ptx::bulk_wait_group_read<0>();
                ptx::named_bar_sync(1, kEpi);
                if (tid == 0) {
                    ptx::mbar_arrive(&m.dempty[db]);
                    if (!*abort_flag && GLA_CHECK(tile >= 0 && tile < tiles && c < nchunks)) {
                        ptx::tma_store_3d(&amap, obuf, c * (int)kChunkN, 0, tile * kTileM);
                        ptx::tma_store_3d(&amap, obuf + kBlk, c * (int)kChunkN + 64, 0, tile * kTileM);
                    }
                    ptx::bulk_commit_group();
                }
            }
        }
        if (tid == 0) ptx::bulk_wait_group_all();               // stores done before smem is freed
        __syncthreads();
    } else if (warp == 8) {
        // ================================================================ TMA producer
        int g = 0;                                              // K-blocks of the schedule so far
        int last[kMaxStages];                                   // last block issued into each slot
        for (int s = 0; s < kMaxStages; ++s) last[s] = -1;
        for (int tile = tile_lo; tile <= tile_hi; ++tile)
            for (int kb = 0; kb < kb_n; ++kb, ++g) {
                const int s = g % S;
                if (g >= S) wait(&m.xempty[s], g / S - 1);
                if (lane == 0 && !*abort_flag) {
                    ptx::mbar_arrive_expect_tx(&m.xfull[s], kBlk);
                    ptx::tma_load_3d(sbase + L.x + s * kBlk, &xmap, 64 * kb, 0, tile * kTileM,
                                     ptx::smem_u32(&m.xfull[s]));
                    last[s] = g;
                }
                __syncwarp();
            }
        // teardown: after an expired wait, the blocks in flight land before smem is freed
        __syncthreads();
        if (*abort_flag && lane == 0) {
            volatile int no_abort = 0;
            for (int s = 0; s < S; ++s)
                if (last[s] >= 0)
                    gate_wait(&m.xfull[s], (uint32_t)((last[s] / S) & 1), p.wait_limit, &no_abort);
        }
    } else if (warp == 9) {
        // ============================================================== T = X W1 issuer
        constexpr uint32_t kId1 = ptx::idesc_ab(0, 0, false, false, kTileM, kRank);
        ptx::named_bar_sync(2, kEpi + 64);
        int g = 0, t = 0;
        for (int tile = tile_lo; tile <= tile_hi; ++tile, ++t) {
            const int b = t & 1;
            if (t >= 2) wait(&m.tfree[b], (t >> 1) - 1);       // the epilogue has read T[b]
            for (int kb = 0; kb < kb_n; ++kb, ++g) {
                const int s = g % S;
                wait(&m.xfull[s], g / S);
                if (lane == 0) {
                    ptx::tc_fence_after_sync();
                    if (!*abort_flag) {
                        const uint64_t ad = ptx::desc_sw128(sbase + L.x + s * kBlk, 16, 1024);
                        const uint64_t bd = ptx::desc_sw128(sbase + L.w1 + kb * 2048, 16, 1024);
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            ptx::mma_f16_ss(tmem + kColT + 16 * b, ad + 2 * k, bd + 2 * k, kId1, kb > 0 || k > 0);
                    }
                    ptx::mma_commit(&m.xempty[s]);              // the block may be reloaded
                }
                __syncwarp();
            }
            if (lane == 0) ptx::mma_commit(&m.tdone[b]);
            __syncwarp();
        }
        __syncthreads();
        if (*abort_flag && lane == 0) {
            volatile int no_abort = 0;
            ptx::mma_commit(&m.end_t);
            gate_wait(&m.end_t, 0, p.wait_limit, &no_abort);
        }
    } else {
        // ========================================================= D = (Th + Tl) W2 issuer
        constexpr uint32_t kId2 = ptx::idesc_ab(0, 0, false, true, kTileM, kChunkN);
        ptx::named_bar_sync(2, kEpi + 64);
        int t = 0, q = 0;
        for (int tile = tile_lo; tile <= tile_hi; ++tile, ++t) {
            const int b = t & 1;
            int c0, c1;
            chunk_range(tile, c0, c1);
            wait(&m.t16[b], t >> 1);                            // Th, Tl written by the epilogue
            for (int c = c0; c < c1; ++c, ++q) {
                const int db = q & 1;
                if (q >= 2) wait(&m.dempty[db], (q >> 1) - 1);
                if (lane == 0) {
                    ptx::tc_fence_after_sync();
                    if (!*abort_flag) {
                        const uint64_t bd = ptx::desc_sw128(sbase + L.w2 + c * 2 * 2048, 2048, 1024);
                        const uint32_t d = tmem + kColD + db * kChunkN;
                        ptx::mma_f16_ts(d, tmem + kColTs + 16 * b, bd, kId2, false);
                        ptx::mma_f16_ts(d, tmem + kColTs + 16 * b + 8, bd, kId2, true);
                    }
                    ptx::mma_commit(&m.dfull[db]);
                }
                __syncwarp();
            }
        }
        __syncthreads();
        if (*abort_flag && lane == 0) {
            volatile int no_abort = 0;
            ptx::mma_commit(&m.end_d);
            gate_wait(&m.end_d, 0, p.wait_limit, &no_abort);
        }
    }
    // ---- teardown
    __syncthreads();
    if (tid == 0 && m.range_err) raise_status(8 /* GLA_ERR_RANGE */);
    ptx::tc_fence_after_sync();
    if (warp == 0) ptx::tmem_dealloc(tmem, kTmemCols);
}

}  // namespace gp
}  // namespace gla
