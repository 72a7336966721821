// gla_sswiglu.cuh -- Spatial SwiGLU's token mixing step, fused: h = SiLU(gate) * (DWConv3x3(value) + b)
// (fp16 I/O, fp32 arithmetic, CUDA cores; HBM-bound).
//
// Operation (GTR paper, arXiv 2609.26590, method section, Spatial SwiGLU paragraph): the value
// branch of the SwiGLU block is reshaped to the 2-D patch grid, passed through a 3x3 depthwise
// convolution and restored to sequence order; the gating branch stays tokenwise.  Read as a
// framework depthwise Conv2d (per-channel 3x3 cross-correlation, zero padding of one token, a
// bias per channel) on the value branch, multiplied by SiLU of the gating branch:
//     h[b][y][x][c] = SiLU(gate[b][y][x][c]) * (bias[c] + sum_{i,j in 0..2} w[c][i][j] value[b][y+i-1][x+j-1][c])
// value, gate, h are token-major [B][grid_h * grid_w][C] (C contiguous); w [C][3][3], bias [C].
//
// Tiling: a CTA tile is R <= 8 grid rows x Wt <= 16 grid columns x 64 channels.  Two TMA boxes
// of 4-D views {C, W, H, B} bring the tile's values with a one-token halo ((R + 2) x (Wt + 2) x
// 128 B) and its gates (R x Wt x 128 B) into shared memory; halo positions outside the grid
// (the zero padding) come back as zeros from the TMA bounds check, so no thread special-cases
// the border.  Two stages: the next tile's boxes load while this tile computes (with two CTAs
// per SM, about 80 KB of loads in flight per SM).  The grid is a multiple of the channel-slab
// count, so a CTA keeps one slab and loads its taps once.  Thread (xl, q) owns grid column
// x0 + xl and channels 4q .. 4q+3 of the slab and walks down the R rows with a 3 x 3 window of
// fp32 values in registers (rows taken three at a time, so the window is renamed rather than
// copied): each output reads one new value row segment (3 x 8 B) and its gate (8 B) from shared
// memory and stores 8 B of h.  The taps, the window and the SiLU arithmetic use packed
// fp32 pairs (f32x2 FMA / multiply / add), two channels per instruction.  A warp's 32 threads cover two grid
// columns x 128 B, so shared loads, gate loads and stores are all contiguous 256-byte runs.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>

#include "gla_common.cuh"
#include "gla_ptx.cuh"

namespace gla {
namespace sw {

constexpr int kSlab = 64;                       // channels per tile: one 128-byte row per token
constexpr int kQ = kSlab / 4;                   // 4-channel groups per slab (threads per column)
constexpr int kMaxR = 8, kMaxWt = 16;           // tile extent limits
constexpr int kThreads = kQ * kMaxWt;           // 256

struct SwParams {
    const float *w, *b;                         // value and gate come through their tensor maps
    __half *out;
    int B, H, W, C;
    int R, Wt;                                  // tile extent: grid rows, grid columns
    int nyb, nxb, nslab;                        // tile counts per dimension
    long long tiles;
    long long wait_limit;
};

// Packed fp32 pairs (Blackwell's f32x2 arithmetic): two channels per instruction.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ float2 f2_unpack(uint64_t v) {
    float2 r;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
    return r;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
// two fp16 (low half first) -> a packed fp32 pair
__device__ __forceinline__ uint64_t f2_from_h2(uint32_t h2) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&h2));
    return f2_pack(f.x, f.y);
}

// one stage: the value box with its halo, then the gate box
__host__ __device__ constexpr uint32_t sw_val_bytes(int R, int Wt) {
    return (uint32_t)(R + 2) * (uint32_t)(Wt + 2) * 128u;
}
__host__ __device__ constexpr uint32_t sw_buf_bytes(int R, int Wt) {
    return sw_val_bytes(R, Wt) + (uint32_t)R * (uint32_t)Wt * 128u;
}

__global__ void __launch_bounds__(kThreads, 2)
    gla_sswiglu_kernel(const __grid_constant__ CUtensorMap vmap, const __grid_constant__ CUtensorMap gmap,
                       const SwParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    __shared__ uint64_t full[2];
    __shared__ int abort_sh;
    volatile int &abort_flag = abort_sh;
    const uint32_t sbase = ptx::smem_u32(sm);
    const uint32_t buf_bytes = sw_buf_bytes(p.R, p.Wt), val_bytes = sw_val_bytes(p.R, p.Wt);
    const int tid = threadIdx.x;
    const int xl = tid / kQ, q = tid % kQ;
    const bool active = xl < p.Wt;

    if (tid == 0) {
        ptx::mbar_init(&full[0], 1);
        ptx::mbar_init(&full[1], 1);
        ptx::fence_mbarrier_init();
        abort_sh = 0;
        ptx::prefetch_tmap(&vmap);
        ptx::prefetch_tmap(&gmap);
    }
    __syncthreads();
    ptx::pdl_launch_dependents();
    ptx::pdl_wait_prior_grid();

    // tile t -> (b, y block, x block, slab), slab fastest
    auto coords = [&](long long t, int &b, int &yb, int &xb, int &slab) {
        slab = (int)(t % p.nslab);
        long long r = t / p.nslab;
        xb = (int)(r % p.nxb);
        r /= p.nxb;
        yb = (int)(r % p.nyb);
        b = (int)(r / p.nyb);
    };
    int issued[2] = {0, 0};                                     // loads armed per buffer (thread 0)
    auto issue = [&](long long t, int buf) {
        ++issued[buf];
        int b, yb, xb, slab;
        coords(t, b, yb, xb, slab);
        if (GLA_CHECK(b >= 0 && b < p.B && slab * kSlab < p.C)) {
            ptx::mbar_arrive_expect_tx(&full[buf], buf_bytes);
            ptx::tma_load_4d(sbase + buf * buf_bytes, &vmap, slab * kSlab, xb * p.Wt - 1, yb * p.R - 1, b,
                             ptx::smem_u32(&full[buf]));
            ptx::tma_load_4d(sbase + buf * buf_bytes + val_bytes, &gmap, slab * kSlab, xb * p.Wt, yb * p.R, b,
                             ptx::smem_u32(&full[buf]));
        } else {
            ptx::mbar_arrive(&full[buf]);
        }
    };

    float amax = 0.0f;
    uint64_t wt[9][2], bias[2];
    int cur_slab = -1;
    if (tid == 0 && (long long)blockIdx.x < p.tiles) issue(blockIdx.x, 0);
    int it = 0;
    for (long long t = blockIdx.x; t < p.tiles; t += gridDim.x, ++it) {
        const int buf = it & 1;
        // the other buffer was last read in the previous iteration, which ended at a barrier
        if (tid == 0 && !abort_flag && t + gridDim.x < p.tiles) issue(t + gridDim.x, buf ^ 1);
        int b, yb, xb, slab;
        coords(t, b, yb, xb, slab);
        const int c = slab * kSlab + 4 * q;
        const int x = xb * p.Wt + xl;
        const int y0 = yb * p.R;
        const int rows = min(p.R, p.H - y0);
        const bool live = active && x < p.W;
        // this thread's taps and bias (4 channels as two packed fp32 pairs), reloaded only
        // when the slab changes
        if (slab != cur_slab) {
            cur_slab = slab;
#pragma unroll
            for (int pr = 0; pr < 2; ++pr) {
                const int ca = c + 2 * pr;
                bias[pr] = active ? f2_pack(p.b[ca], p.b[ca + 1]) : 0ull;
#pragma unroll
                for (int k = 0; k < 9; ++k)
                    wt[k][pr] = active ? f2_pack(p.w[(size_t)ca * 9 + k], p.w[(size_t)(ca + 1) * 9 + k]) : 0ull;
            }
        }
        const size_t row_stride = (size_t)p.W * p.C;
        __half *obase = p.out + ((size_t)b * p.H + y0) * row_stride + (size_t)x * p.C + c;

        // wait for the tile's values (bounded)
        if (!abort_flag) {
            const long long start = clock64();
            while (!ptx::mbar_try_wait(&full[buf], (uint32_t)((it >> 1) & 1))) {
                if (clock64() - start > p.wait_limit) {
                    raise_status(7 /* GLA_ERR_TIMEOUT */);
                    abort_flag = 1;
                    break;
                }
            }
        }
        const bool go = active && !abort_flag;
        const uint8_t *tb = sm + buf * buf_bytes + 8 * q;
        const uint8_t *gtb = tb + val_bytes;
        const uint32_t row_bytes = (uint32_t)(p.Wt + 2) * 128u;
        // tile row tr, columns xl .. xl+2 -> [column][channel pair]
        auto load3 = [&](int tr, uint64_t (&dst)[3][2]) {
#pragma unroll
            for (int j = 0; j < 3; ++j) {
                const uint32_t off = (uint32_t)tr * row_bytes + (uint32_t)(xl + j) * 128u;
                uint2 u = make_uint2(0, 0);
                if (GLA_CHECK(off + 8 * q + 8 <= buf_bytes)) u = *reinterpret_cast<const uint2 *>(tb + off);
                dst[j][0] = f2_from_h2(u.x);
                dst[j][1] = f2_from_h2(u.y);
            }
        };
        // one output row: window rows (A, B, C) = tile rows (r, r+1, r+2), C loaded here
        auto step = [&](int r, uint64_t (&A)[3][2], uint64_t (&Bw)[3][2], uint64_t (&Cw)[3][2]) {
            load3(r + 2, Cw);
            const uint32_t goff = ((uint32_t)r * (uint32_t)p.Wt + (uint32_t)xl) * 128u;
            uint2 GA = make_uint2(0, 0);
            if (GLA_CHECK(val_bytes + goff + 8 * q + 8 <= buf_bytes)) GA = *reinterpret_cast<const uint2 *>(gtb + goff);
            uint64_t acc[2];
#pragma unroll
            for (int pr = 0; pr < 2; ++pr) {
                uint64_t s2 = bias[pr];
#pragma unroll
                for (int j = 0; j < 3; ++j) {
                    s2 = f2_fma(wt[j][pr], A[j][pr], s2);
                    s2 = f2_fma(wt[3 + j][pr], Bw[j][pr], s2);
                    s2 = f2_fma(wt[6 + j][pr], Cw[j][pr], s2);
                }
                acc[pr] = s2;
            }
            // SiLU(g) = g / (1 + 2^(-g log2 e)), times the convolution
            const uint64_t g2[2] = {f2_from_h2(GA.x), f2_from_h2(GA.y)};
            uint32_t packed[2];
#pragma unroll
            for (int pr = 0; pr < 2; ++pr) {
                const float2 t = f2_unpack(f2_mul(g2[pr], f2_pack(-1.4426950408889634f, -1.4426950408889634f)));
                const uint64_t den = f2_add(f2_pack(ptx::ex2(t.x), ptx::ex2(t.y)), f2_pack(1.0f, 1.0f));
                const float2 dv = f2_unpack(den);
                const uint64_t sg = f2_mul(g2[pr], f2_pack(ptx::rcp(dv.x), ptx::rcp(dv.y)));
                const float2 h = f2_unpack(f2_mul(sg, acc[pr]));
                amax = fmaxf(amax, fmaxf(fabsf(h.x), fabsf(h.y)));
                const __half2 o = __floats2half2_rn(h.x, h.y);
                packed[pr] = *reinterpret_cast<const uint32_t *>(&o);
            }
            if (live) __stcs(reinterpret_cast<uint2 *>(obase + (size_t)r * row_stride), make_uint2(packed[0], packed[1]));
        };
        uint64_t W0[3][2], W1[3][2], W2[3][2];
        if (go) {
            load3(0, W0);
            load3(1, W1);
            // rows in threes with the window and gate registers renamed, not copied
            int r = 0;
#pragma unroll 1
            for (; r + 3 <= rows; r += 3) {
                step(r, W0, W1, W2);
                step(r + 1, W1, W2, W0);
                step(r + 2, W2, W0, W1);
            }
            if (r < rows) step(r, W0, W1, W2);
            if (r + 1 < rows) step(r + 1, W1, W2, W0);
        }
        __syncthreads();                                        // buffer `buf` free for reuse
    }
    // NaN or above the fp16 range: the output cannot hold it
    if (!(amax <= 65504.0f)) raise_status(8 /* GLA_ERR_RANGE */);
    // a box still in flight after an expired wait lands before the CTA exits: the k-th load
    // armed on a buffer completes its phase k
    if (tid == 0 && abort_flag) {
        for (int buf = 0; buf < 2; ++buf) {
            if (issued[buf] == 0) continue;
            const long long start = clock64();
            while (!ptx::mbar_try_wait(&full[buf], (uint32_t)((issued[buf] - 1) & 1)))
                if (clock64() - start > p.wait_limit) break;
        }
    }
}

}  // namespace sw
}  // namespace gla
