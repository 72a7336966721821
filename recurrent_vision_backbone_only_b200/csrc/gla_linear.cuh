// gla_linear.cuh -- the block's dense projections y = x W (+ bias) on tcgen05 tensor cores
// (fp16 I/O, fp32 accumulation).
//
// Operation (GTR paper, arXiv 2609.26590, method section): the input projections
// Q = X W_Q, K = X W_K, V = X W_V and the output gate's x W_r (GLA recurrence and output-gate
// paragraphs), and the output projection that maps the concatenated heads back to the model
// dimension (output-gate paragraph).  x [M][K] row-major, W [K][N] row-major, optional bias [N].
// The output is written as parts of n_part columns each, [N / n_part][M][n_part]: with
// n_part = N that is a plain [M][N] matrix; with W = [W_Q | W_K | W_V | W_r] and n_part = H d
// it is q, k, v and the output-gate pre-activation as four separate [B][L][H][d] tensors, the
// operator's input layout, from one pass over x.
//
// Per output tile of 128 rows x nt columns (nt = 128, 192 or 256):
//   K loop in 64-wide blocks through a TMA ring: the x block [128][64] (K-major, 128-byte
//   swizzle) and nt / 64 boxes of W [64 K rows][64 columns] (MN-major, 128-byte swizzle);
//   4 tcgen05.mma of K = 16 per block into a TMEM accumulator (two accumulators, so one
//   tile's epilogue overlaps the next tile's products);
//   epilogue: TMEM -> registers (+ bias) -> fp16 -> two 128-byte swizzled staging boxes of
//   [128 rows][64 columns], two boxes per round -> TMA stores (rows past M are clipped by TMA).
//   Staging two boxes rather than the whole tile leaves room for one more ring stage.
// Tiles are numbered column tile fastest, and CTAs stride over them, so the CTAs working at the
// same time share x tiles through L2.
//
// Roles (320 threads, one CTA per SM): warps 0-7 epilogue (warp w reads TMEM lanes
// 32 (w % 4) .. +31 = tile rows), warp 8 TMA
// producer, warp 9 MMA issuer.  In round r the warps with w / 4 = h convert box 2 r + h.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>

#include "gla_common.cuh"
#include "gla_ptx.cuh"

namespace gla {
namespace ln {

constexpr int kTileM = 128, kBK = 64;
constexpr int kThreads = 320;
constexpr int kEpi = 256;                       // epilogue threads (warps 0-7)
constexpr int kMaxStages = 8;
constexpr uint32_t kABytes = kTileM * 128;      // x block: [128 rows][64 K] fp16 = 16 KB
constexpr uint32_t kBBox = kBK * 128;           // W box: [64 K rows][64 columns] fp16 = 8 KB
constexpr uint32_t kOBox = kTileM * 128;        // staging box: [128 rows][64 columns] = 16 KB
constexpr uint32_t kTmemCols = 512;             // two accumulators of up to 256 columns

struct LinMisc {
    uint64_t full[kMaxStages], empty[kMaxStages];
    uint64_t accfull[2], accempty[2], end;
    uint32_t tmem_base;
    int abort;
};

// Shared-memory layout for an nt-column tile: the ring (stages of one x block and nt / 64 W
// boxes), two staging boxes, then the barriers.  Offsets are from the 1024-aligned
// base; `bytes` includes the alignment slack.
struct LinLayout {
    uint32_t stage_bytes, ring, o, misc, bytes;
    int stages;
};

__host__ __device__ inline LinLayout lin_layout(int nt, size_t smem_cap) {
    LinLayout L;
    L.stage_bytes = kABytes + (uint32_t)(nt / 64) * kBBox;
    L.ring = 0;
    const uint32_t staging = 2 * kOBox;
    const size_t fixed = (size_t)staging + sizeof(LinMisc) + 1024;
    const long long fit = smem_cap > fixed ? (long long)((smem_cap - fixed) / L.stage_bytes) : 0;
    L.stages = (int)(fit < kMaxStages ? fit : kMaxStages);
    L.o = L.ring + (uint32_t)(L.stages > 0 ? L.stages : 0) * L.stage_bytes;
    L.misc = L.o + staging;
    L.bytes = L.misc + (uint32_t)sizeof(LinMisc) + 1024u;
    return L;
}

struct LinParams {
    const float *bias;                          // [N] or nullptr
    int M, K, N, n_part;
    int nt;                                     // columns per tile: 128, 192 or 256
    LinLayout lay;
    long long wait_limit;
};

__device__ __forceinline__ bool lin_wait(uint64_t *bar, uint32_t parity, long long limit, volatile int *abort) {
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

// nt-column MMA instruction descriptors (fp16 x fp16 -> fp32, A K-major, B MN-major)
__device__ __forceinline__ uint32_t lin_idesc(int nt) {
    return nt == 256 ? ptx::idesc_ab(0, 0, false, true, kTileM, 256)
                     : nt == 192 ? ptx::idesc_ab(0, 0, false, true, kTileM, 192)
                                 : ptx::idesc_ab(0, 0, false, true, kTileM, 128);
}

__global__ void __launch_bounds__(kThreads, 1)
    gla_linear_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap wmap,
                      const __grid_constant__ CUtensorMap ymap, const LinParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
    const uint32_t sbase = ptx::smem_u32(sm);
    const LinLayout &L = p.lay;
    const int S = L.stages;
    LinMisc &m = *reinterpret_cast<LinMisc *>(sm + L.misc);
    volatile int *abort_flag = &m.abort;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int kb_n = p.K / kBK, nbox = p.nt / 64;
    const int mtiles = (p.M + kTileM - 1) / kTileM, ntiles = p.N / p.nt;
    const long long tiles = (long long)mtiles * ntiles;
    auto wait = [&](uint64_t *bar, int use) { return lin_wait(bar, (uint32_t)(use & 1), p.wait_limit, abort_flag); };

    ptx::pdl_launch_dependents();
    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            ptx::mbar_init(&m.full[s], 1);
            ptx::mbar_init(&m.empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(&m.accfull[i], 1);
            ptx::mbar_init(&m.accempty[i], 1);
        }
        ptx::mbar_init(&m.end, 1);
        ptx::fence_mbarrier_init();
        m.abort = 0;
    }
    if (warp == 0) {
        ptx::tmem_alloc(&m.tmem_base, kTmemCols);
        ptx::tmem_relinquish();
    }
    if (warp == 8 && lane == 0) {
        ptx::prefetch_tmap(&xmap);
        ptx::prefetch_tmap(&wmap);
        ptx::prefetch_tmap(&ymap);
    }
    ptx::tc_fence_before_sync();
    __syncthreads();
    ptx::tc_fence_after_sync();
    const uint32_t tmem = m.tmem_base;
    ptx::pdl_wait_prior_grid();

    if (warp < 8) {
        // ===================================================================== epilogue
        const int quarter = warp & 3, half = warp >> 2;
        const int row = 32 * quarter + lane;                    // tile row = TMEM lane
        const uint32_t lanes = (uint32_t)(32 * quarter) << 16;
        int tc = 0;
        for (long long t = blockIdx.x; t < tiles; t += gridDim.x, ++tc) {
            const int mt = (int)(t / ntiles), n0 = (int)(t % ntiles) * p.nt;
            const int ab = tc & 1;
            wait(&m.accfull[ab], tc >> 1);
            ptx::tc_fence_after_sync();
            for (int r0 = 0; r0 < nbox; r0 += 2) {
                const int j = r0 + half;
                // the previous round's TMA stores have read the two staging boxes
                if (tid == 0) ptx::bulk_wait_group_read<0>();
                ptx::named_bar_sync(1, kEpi);
                if (j < nbox) {
                    float v0[32], v1[32];
                    const uint32_t taddr = tmem + lanes + (uint32_t)(ab * 256 + 64 * j);
                    ptx::tmem_ld32(taddr, v0);
                    ptx::tmem_ld32(taddr + 32, v1);
                    ptx::tmem_ld_wait();
                    const int cb = n0 + 64 * j;                     // first output column of box j
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const float *v = u < 4 ? &v0[8 * u] : &v1[8 * (u - 4)];
                        float4 ba = make_float4(0.f, 0.f, 0.f, 0.f), bb = ba;
                        if (p.bias) {
                            ba = __ldg(reinterpret_cast<const float4 *>(p.bias + cb + 8 * u));
                            bb = __ldg(reinterpret_cast<const float4 *>(p.bias + cb + 8 * u + 4));
                        }
                        const __half2 o0 = __floats2half2_rn(v[0] + ba.x, v[1] + ba.y);
                        const __half2 o1 = __floats2half2_rn(v[2] + ba.z, v[3] + ba.w);
                        const __half2 o2 = __floats2half2_rn(v[4] + bb.x, v[5] + bb.y);
                        const __half2 o3 = __floats2half2_rn(v[6] + bb.z, v[7] + bb.w);
                        const uint32_t off = L.o + (uint32_t)half * kOBox + ptx::sw128(row, u);
                        if (GLA_CHECK(off + 16 <= L.misc))
                            *reinterpret_cast<uint4 *>(sm + off) =
                                make_uint4(*reinterpret_cast<const uint32_t *>(&o0), *reinterpret_cast<const uint32_t *>(&o1),
                                           *reinterpret_cast<const uint32_t *>(&o2), *reinterpret_cast<const uint32_t *>(&o3));
                    }
                }
                ptx::tc_fence_before_sync();
                ptx::fence_proxy_async_smem();
                ptx::named_bar_sync(1, kEpi);
                if (tid == 0) {
                    if (r0 + 2 >= nbox) ptx::mbar_arrive(&m.accempty[ab]);   // accumulator ab read
                    if (!*abort_flag) {
                        for (int jj = r0; jj < r0 + 2 && jj < nbox; ++jj) {
                            const int c = n0 + 64 * jj, part = c / p.n_part, col = c % p.n_part;
                            if (GLA_CHECK(c < p.N && mt < mtiles))
                                ptx::tma_store_3d(&ymap, sbase + L.o + (uint32_t)(jj - r0) * kOBox, col, mt * kTileM,
                                                  part);
                        }
                    }
                    ptx::bulk_commit_group();
                }
            }
        }
        if (tid == 0) ptx::bulk_wait_group_all();               // stores done before smem is freed
        __syncthreads();
    } else if (warp == 8) {
        // ================================================================ TMA producer
        int g = 0;
        int last[kMaxStages];
        for (int s = 0; s < kMaxStages; ++s) last[s] = -1;
        for (long long t = blockIdx.x; t < tiles; t += gridDim.x) {
            const int mt = (int)(t / ntiles), n0 = (int)(t % ntiles) * p.nt;
            for (int kb = 0; kb < kb_n; ++kb, ++g) {
                const int s = g % S;
                if (g >= S) wait(&m.empty[s], g / S - 1);
                if (lane == 0 && !*abort_flag) {
                    const uint32_t st = sbase + L.ring + (uint32_t)s * L.stage_bytes;
                    ptx::mbar_arrive_expect_tx(&m.full[s], L.stage_bytes);
                    ptx::tma_load_3d(st, &xmap, kBK * kb, 0, mt * kTileM, ptx::smem_u32(&m.full[s]));
                    for (int j = 0; j < nbox; ++j)
                        ptx::tma_load_3d(st + kABytes + (uint32_t)j * kBBox, &wmap, n0 + 64 * j, 0, kBK * kb,
                                         ptx::smem_u32(&m.full[s]));
                    last[s] = g;
                }
                __syncwarp();
            }
        }
        __syncthreads();
        if (*abort_flag && lane == 0) {
            volatile int no_abort = 0;
            for (int s = 0; s < S; ++s)
                if (last[s] >= 0) lin_wait(&m.full[s], (uint32_t)((last[s] / S) & 1), p.wait_limit, &no_abort);
        }
    } else {
        // ================================================================== MMA issuer
        const uint32_t idesc = lin_idesc(p.nt);
        int g = 0, tc = 0;
        for (long long t = blockIdx.x; t < tiles; t += gridDim.x, ++tc) {
            const int ab = tc & 1;
            if (tc >= 2) wait(&m.accempty[ab], (tc >> 1) - 1);  // the epilogue has read it
            for (int kb = 0; kb < kb_n; ++kb, ++g) {
                const int s = g % S;
                wait(&m.full[s], g / S);
                if (lane == 0) {
                    ptx::tc_fence_after_sync();
                    if (!*abort_flag) {
                        const uint32_t st = sbase + L.ring + (uint32_t)s * L.stage_bytes;
                        const uint64_t ad = ptx::desc_sw128(st, 16, 1024);
                        // W boxes: 64-column blocks kBBox apart (LBO), 8-row K groups 1024 apart
                        const uint64_t bd = ptx::desc_sw128(st + kABytes, kBBox, 1024);
#pragma unroll
                        for (int k = 0; k < 4; ++k)           // K = 16: 32 B along x, 16 rows of W
                            ptx::mma_f16_ss(tmem + (uint32_t)(ab * 256), ad + 2 * k, bd + (uint64_t)(k * 2048 >> 4),
                                            idesc, kb > 0 || k > 0);
                    }
                    ptx::mma_commit(&m.empty[s]);
                }
                __syncwarp();
            }
            if (lane == 0) ptx::mma_commit(&m.accfull[ab]);
            __syncwarp();
        }
        __syncthreads();
        if (*abort_flag && lane == 0) {
            volatile int no_abort = 0;
            ptx::mma_commit(&m.end);
            lin_wait(&m.end, 0, p.wait_limit, &no_abort);
        }
    }
    // ---- teardown
    __syncthreads();
    ptx::tc_fence_after_sync();
    if (warp == 0) ptx::tmem_dealloc(tmem, kTmemCols);
}

}  // namespace ln
}  // namespace gla
