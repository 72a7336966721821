// gla_gate.cuh -- the retention gate's low-rank projection a = x W1 W2 + b on tcgen05 tensor
// cores (fp16 I/O, fp32 accumulation).
//
// Operation (GTR paper, arXiv 2609.26590, method section, GLA recurrence paragraph): the key-wise
// retention gate is gamma_t = sigma(x_t W_alpha^(1) W_alpha^(2) + b_alpha)^(1/tau), a low-rank
// projection of rank r = 16 "following GLA": one first factor W1 [d][16] shared by the heads, a
// second factor W2 [16][n] onto every head's key channels (n = H d_k), a bias per key channel.
// The output a [T][n] is the operator's gate_preact input, [B][L][H][d_k].
//
// Per 128-token tile (one M = 128 tcgen05 tile):
//   T  = X W1          d / 16 MMAs (K = 16, N = 16), X streamed through a TMA ring of 64-channel
//                      K-blocks, W1 resident (K-major)                         -> TMEM, fp32
//   T  = Th + Tl       split to fp16 high / low on CUDA cores, back into TMEM as the A operand
//   D  = Th W2 + Tl W2 two MMAs per 128-column chunk of n (W2 resident, MN-major), into one of
//                      two TMEM buffers, so a chunk's epilogue overlaps the next chunk's products
//   a  = fp16(D + b)   epilogue (thread = token row) into a 128-byte swizzled staging tile,
//                      written out by TMA stores (rows past the last token are clipped by TMA)
// The split keeps the second product exact to ~2^-22 relative; only the output rounding remains.
//
// Work items: (tile, column group).  With fewer tiles than SMs the host splits each tile's output
// chunks into `groups` column groups, one item each (every item recomputes its tile's rank-16
// X W1, which the re-read X tile mostly serves from L2), so short inputs still use the device.
//
// Roles (192 threads, persistent over items): warps 0-3 epilogue (TMEM lanes = tile rows) and
// the one-time staging of W1 / W2 / b, warp 4 TMA producer, warp 5 MMA issuer.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>

#include "gla_common.cuh"
#include "gla_ptx.cuh"

namespace gla {
namespace gp {

constexpr int kRank = 16;
constexpr int kTileM = 128;
constexpr int kThreads = 192;
constexpr int kStages = 4;                      // X ring: [128 rows][64 channels] fp16 K-blocks
constexpr uint32_t kBlk = kTileM * 128;         // 16 KB
constexpr int kMaxD = 1024, kMaxN = 1024;
constexpr uint32_t kW1 = 0;                                   // [d/64][16 rows][128 B], K-major
constexpr uint32_t kW2 = kW1 + (kMaxD / 64) * 2048;           // [n/64][16 rows][128 B], MN-major
constexpr uint32_t kX = kW2 + (kMaxN / 64) * 2048;            // ring
constexpr uint32_t kO = kX + kStages * kBlk;                 // 2 x [2 boxes][128 rows][128 B]
constexpr uint32_t kOBuf = 2 * kBlk;
constexpr uint32_t kMisc = kO + 2 * kOBuf;
// TMEM columns
constexpr uint32_t kColT = 0, kColTh = 16, kColTl = 24, kColD = 256, kChunkN = 128;
constexpr uint32_t kTmemCols = 512;

struct GateParams {
    const __half *w1, *w2;
    const float *b;                             // the output a goes through its tensor map
    int T, d, n;
    int groups;                                 // column groups per tile (1 .. n / 128)
    long long wait_limit;
};

struct GateMisc {
    uint64_t xfull[kStages], xempty[kStages];
    uint64_t tdone, t16, dfull[2], dempty[2], end;
    uint32_t tmem_base;
    int abort, range_err;
    alignas(16) float bias[kMaxN];
};

constexpr size_t gate_smem_bytes() { return kMisc + sizeof(GateMisc) + 1024; }

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
    GateMisc &m = *reinterpret_cast<GateMisc *>(sm + kMisc);
    volatile int *abort_flag = &m.abort;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int kb_n = p.d / 64, nchunks = p.n / kChunkN;
    const int tiles = (p.T + kTileM - 1) / kTileM;
    const int per_group = (nchunks + p.groups - 1) / p.groups;
    const int items = tiles * p.groups;
    // output chunks [c0, c1) of item w
    auto chunk_range = [&](int w, int &c0, int &c1) {
        c0 = (w % p.groups) * per_group;
        c1 = min(nchunks, c0 + per_group);
    };
    auto wait = [&](uint64_t *bar, int use) { return gate_wait(bar, (uint32_t)(use & 1), p.wait_limit, abort_flag); };

    ptx::pdl_launch_dependents();
    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            ptx::mbar_init(&m.xfull[s], 1);
            ptx::mbar_init(&m.xempty[s], 1);
        }
        ptx::mbar_init(&m.tdone, 1);
        ptx::mbar_init(&m.t16, 1);
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(&m.dfull[i], 1);
            ptx::mbar_init(&m.dempty[i], 1);
        }
        ptx::mbar_init(&m.end, 1);
        ptx::fence_mbarrier_init();
        m.abort = 0;
        m.range_err = 0;
    }
    if (warp == 0) {
        ptx::tmem_alloc(&m.tmem_base, kTmemCols);
        ptx::tmem_relinquish();
    }
    if (warp == 4 && lane == 0) {
        ptx::prefetch_tmap(&xmap);
        ptx::prefetch_tmap(&amap);
    }
    ptx::tc_fence_before_sync();
    __syncthreads();
    ptx::tc_fence_after_sync();
    const uint32_t tmem = m.tmem_base;
    ptx::pdl_wait_prior_grid();
    // resident operands: W1 transposed to K-major [16 rows (r)][d (k)], W2 as MN-major
    // [16 rows (r)][n (c)], both in 128-byte swizzled 2 KB blocks of 64 columns.  Every global
    // read is one 16-byte cp.async issued up front (W1 lands raw in the X ring, free until the
    // producer starts, and is transposed from there), so staging costs one memory latency.
    if (warp < 4) {
        for (int e = tid; e < p.d * kRank / 8; e += 128)
            ptx::cp_async16(sbase + kX + 16 * e, p.w1 + 8 * (size_t)e, 16);
        for (int e = tid; e < kRank * p.n / 8; e += 128) {      // 8 consecutive c of one row r
            const int r = e / (p.n / 8), c0 = 8 * (e % (p.n / 8));
            ptx::cp_async16(sbase + kW2 + (c0 / 64) * 2048 + ptx::sw128(r, (c0 % 64) / 8),
                            p.w2 + (size_t)r * p.n + c0, 16);
        }
        for (int e = tid; e < p.n / 4; e += 128) ptx::cp_async16(ptx::smem_u32(&m.bias[4 * e]), p.b + 4 * e, 16);
        ptx::cp_async_wait_all();
        ptx::named_bar_sync(1, 128);
        const __half *raw = reinterpret_cast<const __half *>(sm + kX);   // [d][16]
        for (int e = tid; e < p.d * kRank / 8; e += 128) {      // 8 consecutive k of one row r
            const int r = e % kRank, k0 = 8 * (e / kRank);
            __align__(16) __half v[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] = raw[(k0 + i) * kRank + r];
            *reinterpret_cast<uint4 *>(sm + kW1 + (k0 / 64) * 2048 + ptx::sw128(r, (k0 % 64) / 8)) =
                *reinterpret_cast<const uint4 *>(v);
        }
        ptx::fence_proxy_async_smem();
    }
    __syncthreads();

    if (warp == 4) {
        // ================================================================ TMA producer
        int g = 0;                                              // K-blocks of the schedule so far
        int last[kStages];                                      // last block issued into each slot
        for (int s = 0; s < kStages; ++s) last[s] = -1;
        for (int w = blockIdx.x; w < items; w += gridDim.x)
            for (int kb = 0; kb < kb_n; ++kb, ++g) {
                const int tile = w / p.groups;
                const int s = g % kStages;
                if (g >= kStages) wait(&m.xempty[s], g / kStages - 1);
                if (lane == 0 && !*abort_flag) {
                    ptx::mbar_arrive_expect_tx(&m.xfull[s], kBlk);
                    ptx::tma_load_3d(sbase + kX + s * kBlk, &xmap, 64 * kb, 0, tile * kTileM,
                                     ptx::smem_u32(&m.xfull[s]));
                    last[s] = g;
                }
                __syncwarp();
            }
        // teardown: after an expired wait, the blocks in flight land before smem is freed
        __syncthreads();
        if (*abort_flag && lane == 0) {
            volatile int no_abort = 0;
            for (int s = 0; s < kStages; ++s)
                if (last[s] >= 0)
                    gate_wait(&m.xfull[s], (uint32_t)((last[s] / kStages) & 1), p.wait_limit, &no_abort);
        }
    } else if (warp == 5) {
        // ================================================================== MMA issuer
        constexpr uint32_t kId1 = ptx::idesc_ab(0, 0, false, false, kTileM, kRank);
        constexpr uint32_t kId2 = ptx::idesc_ab(0, 0, false, true, kTileM, kChunkN);
        int g = 0, t = 0, q = 0;                                // K-blocks, tiles, output chunks
        for (int w = blockIdx.x; w < items; w += gridDim.x, ++t) {
            int c0, c1;
            chunk_range(w, c0, c1);
            // T = X W1; the epilogue has read the previous tile's T before this tile's t16
            // signal, and each tile's MMAs wait for their own t16, so T is free here
            for (int kb = 0; kb < kb_n; ++kb, ++g) {
                const int s = g % kStages;
                wait(&m.xfull[s], g / kStages);
                if (lane == 0) {
                    ptx::tc_fence_after_sync();
                    if (!*abort_flag) {
                        const uint64_t ad = ptx::desc_sw128(sbase + kX + s * kBlk, 16, 1024);
                        const uint64_t bd = ptx::desc_sw128(sbase + kW1 + kb * 2048, 16, 1024);
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            ptx::mma_f16_ss(tmem + kColT, ad + 2 * k, bd + 2 * k, kId1, kb > 0 || k > 0);
                    }
                    ptx::mma_commit(&m.xempty[s]);              // the block may be reloaded
                }
                __syncwarp();
            }
            if (lane == 0) ptx::mma_commit(&m.tdone);
            __syncwarp();
            wait(&m.t16, t);                                    // Th, Tl written by the epilogue
            for (int c = c0; c < c1; ++c, ++q) {
                const int db = q & 1;
                if (q >= 2) wait(&m.dempty[db], q / 2 - 1);
                if (lane == 0) {
                    ptx::tc_fence_after_sync();
                    if (!*abort_flag) {
                        const uint64_t bd = ptx::desc_sw128(sbase + kW2 + c * 2 * 2048, 2048, 1024);
                        const uint32_t d = tmem + kColD + db * kChunkN;
                        ptx::mma_f16_ts(d, tmem + kColTh, bd, kId2, false);
                        ptx::mma_f16_ts(d, tmem + kColTl, bd, kId2, true);
                    }
                    ptx::mma_commit(&m.dfull[db]);
                }
                __syncwarp();
            }
        }
        __syncthreads();
        if (*abort_flag && lane == 0) {
            volatile int no_abort = 0;
            ptx::mma_commit(&m.end);
            gate_wait(&m.end, 0, p.wait_limit, &no_abort);
        }
    } else {
        // ===================================================================== epilogue
        // thread tid = tile row = TMEM lane
        const uint32_t lanes = (uint32_t)(32 * warp) << 16;
        int t = 0, q = 0;
        for (int w = blockIdx.x; w < items; w += gridDim.x, ++t) {
            const int tile = w / p.groups;
            int c0, c1;
            chunk_range(w, c0, c1);
            wait(&m.tdone, t);
            ptx::tc_fence_after_sync();
            {
                float tv[32];
                ptx::tmem_ld32(tmem + lanes + kColT, tv);
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
                ptx::tmem_st8(tmem + lanes + kColTh, hi);
                ptx::tmem_st8(tmem + lanes + kColTl, lo);
                ptx::tmem_st_wait();
            }
            ptx::tc_fence_before_sync();
            ptx::named_bar_sync(1, 128);
            if (tid == 0) ptx::mbar_arrive(&m.t16);
            for (int c = c0; c < c1; ++c, ++q) {
                const int db = q & 1;                           // TMEM buffer = staging buffer
                const uint32_t obuf = sbase + kO + db * kOBuf;
                wait(&m.dfull[db], q / 2);
                // the TMA store that last read this staging buffer (two chunks ago) is done
                if (tid == 0) ptx::bulk_wait_group_read<1>();
                ptx::named_bar_sync(1, 128);
                ptx::tc_fence_after_sync();
#pragma unroll 1
                for (int h = 0; h < (int)kChunkN / 32; ++h) {
                    float v[32];
                    ptx::tmem_ld32(tmem + lanes + kColD + db * kChunkN + 32 * h, v);
                    ptx::tmem_ld_wait();
                    const int cb = c * (int)kChunkN + 32 * h;   // first output column
                    // columns 32h .. 32h+31 of the chunk: box h / 2, 16-byte pieces 4 (h % 2) + u
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        uint32_t pk[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int i = 8 * u + 2 * e;
                            const __half2 o = __floats2half2_rn(v[i] + m.bias[cb + i], v[i + 1] + m.bias[cb + i + 1]);
                            pk[e] = *reinterpret_cast<const uint32_t *>(&o);
                        }
                        const uint32_t off = (h / 2) * kBlk + ptx::sw128(tid, 4 * (h % 2) + u);
                        if (GLA_CHECK(off + 16 <= kOBuf))
                            *reinterpret_cast<uint4 *>(sm + (obuf - sbase) + off) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    }
                }
                ptx::tc_fence_before_sync();
                ptx::fence_proxy_async_smem();
                ptx::named_bar_sync(1, 128);
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
    }
    // ---- teardown
    __syncthreads();
    if (tid == 0 && m.range_err) raise_status(8 /* GLA_ERR_RANGE */);
    ptx::tc_fence_after_sync();
    if (warp == 0) ptx::tmem_dealloc(tmem, kTmemCols);
}

}  // namespace gp
}  // namespace gla
