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
// Tiling: a CTA tile is R grid rows x Wt grid columns x 64 channels.  One TMA box of a 4-D view
// {C, W, H, B} brings the tile's values with a one-token halo, (R + 2) x (Wt + 2) x 128 B, into
// shared memory; halo positions outside the grid (the zero padding) come back as zeros from the
// TMA bounds check, so no thread special-cases the border.  Two buffers: the next tile's box
// loads while this tile computes.  Thread (xl, q) owns grid column x0 + xl and channels
// 4q .. 4q+3 of the slab and walks down the R rows with a 3 x 3 window of fp32 values in
// registers: each output reads one new smem row segment (3 x 8 B), loads its gate directly from
// global memory two rows ahead, and stores 8 B of h.  A warp's 32 threads cover two grid
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
constexpr int kMaxTile = 16;                    // R, Wt <= 16
constexpr int kThreads = kQ * kMaxTile;         // 256

struct SwParams {
    const __half *gate;
    const float *w, *b;
    __half *out;
    int B, H, W, C;
    int R, Wt;                                  // tile extent: grid rows, grid columns
    int nyb, nxb, nslab;                        // tile counts per dimension
    long long tiles;
    long long wait_limit;
};

__host__ __device__ constexpr uint32_t sw_buf_bytes(int R, int Wt) {
    return (uint32_t)(R + 2) * (uint32_t)(Wt + 2) * 128u;
}

__global__ void __launch_bounds__(kThreads, 2)
    gla_sswiglu_kernel(const __grid_constant__ CUtensorMap vmap, const SwParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    __shared__ uint64_t full[2];
    __shared__ int abort_sh;
    volatile int &abort_flag = abort_sh;
    const uint32_t sbase = ptx::smem_u32(sm);
    const uint32_t buf_bytes = sw_buf_bytes(p.R, p.Wt);
    const int tid = threadIdx.x;
    const int xl = tid / kQ, q = tid % kQ;
    const bool active = xl < p.Wt;

    if (tid == 0) {
        ptx::mbar_init(&full[0], 1);
        ptx::mbar_init(&full[1], 1);
        ptx::fence_mbarrier_init();
        abort_sh = 0;
        ptx::prefetch_tmap(&vmap);
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
        } else {
            ptx::mbar_arrive(&full[buf]);
        }
    };

    float amax = 0.0f;
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
        // this thread's taps and bias (4 channels)
        float wt[9][4], bias[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            bias[i] = live ? p.b[c + i] : 0.0f;
#pragma unroll
            for (int k = 0; k < 9; ++k) wt[k][i] = live ? p.w[(size_t)(c + i) * 9 + k] : 0.0f;
        }
        // gate of output rows 0 and 1, two rows ahead of use
        const size_t row_stride = (size_t)p.W * p.C;
        const __half *gbase = p.gate + ((size_t)b * p.H + y0) * row_stride + (size_t)x * p.C + c;
        __half *obase = p.out + ((size_t)b * p.H + y0) * row_stride + (size_t)x * p.C + c;
        uint2 g0 = make_uint2(0, 0), g1 = make_uint2(0, 0);
        if (live) g0 = __ldcs(reinterpret_cast<const uint2 *>(gbase));
        if (live && rows > 1) g1 = __ldcs(reinterpret_cast<const uint2 *>(gbase + row_stride));

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
        const uint8_t *tb = sm + buf * buf_bytes + 8 * q;
        const uint32_t row_bytes = (uint32_t)(p.Wt + 2) * 128u;
        auto load3 = [&](int tr, float (&dst)[3][4]) {          // tile row tr, columns xl .. xl+2
#pragma unroll
            for (int j = 0; j < 3; ++j) {
                const uint32_t off = (uint32_t)tr * row_bytes + (uint32_t)(xl + j) * 128u;
                uint2 u = make_uint2(0, 0);
                if (GLA_CHECK(off + 8 * q + 8 <= buf_bytes)) u = *reinterpret_cast<const uint2 *>(tb + off);
                const float2 lo = __half22float2(*reinterpret_cast<const __half2 *>(&u.x));
                const float2 hi = __half22float2(*reinterpret_cast<const __half2 *>(&u.y));
                dst[j][0] = lo.x;
                dst[j][1] = lo.y;
                dst[j][2] = hi.x;
                dst[j][3] = hi.y;
            }
        };
        float win[3][3][4];                                     // [window row][column][channel]
        if (active && !abort_flag) {
            load3(0, win[0]);
            load3(1, win[1]);
        }
#pragma unroll 1
        for (int r = 0; r < rows; ++r) {
            uint2 g2 = make_uint2(0, 0);
            if (live && r + 2 < rows) g2 = __ldcs(reinterpret_cast<const uint2 *>(gbase + (size_t)(r + 2) * row_stride));
            if (active && !abort_flag) {
                load3(r + 2, win[2]);
                float acc[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    float s = bias[i];
#pragma unroll
                    for (int a = 0; a < 3; ++a)
#pragma unroll
                        for (int j = 0; j < 3; ++j) s = fmaf(wt[3 * a + j][i], win[a][j][i], s);
                    acc[i] = s;
                }
                const float2 ga = __half22float2(*reinterpret_cast<const __half2 *>(&g0.x));
                const float2 gb = __half22float2(*reinterpret_cast<const __half2 *>(&g0.y));
                const float gv[4] = {ga.x, ga.y, gb.x, gb.y};
                float h[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    h[i] = __fdividef(gv[i], 1.0f + __expf(-gv[i])) * acc[i];
                    amax = fmaxf(amax, fabsf(h[i]));
                }
                if (live) {
                    const __half2 o0 = __floats2half2_rn(h[0], h[1]);
                    const __half2 o1 = __floats2half2_rn(h[2], h[3]);
                    __stcs(reinterpret_cast<uint2 *>(obase + (size_t)r * row_stride),
                           make_uint2(*reinterpret_cast<const uint32_t *>(&o0), *reinterpret_cast<const uint32_t *>(&o1)));
                }
#pragma unroll
                for (int j = 0; j < 3; ++j)
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        win[0][j][i] = win[1][j][i];
                        win[1][j][i] = win[2][j][i];
                    }
            }
            g0 = g1;
            g1 = g2;
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
