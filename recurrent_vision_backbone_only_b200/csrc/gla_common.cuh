// gla_common.cuh -- device helpers shared by the GLA kernels of libgla.so.
//
// Operation: key-only gated linear attention of the GTR paper (arXiv
// 2609.26590, method section): gamma_t = sigma(a_t)^(1/16),
// S_t = Diag(gamma_t) S_{t-1} + k_t^T v_t, o_t = d_k^{-1/2} q_t S_t,
// u_t = SiLU(g_t) * RMSNorm(o_t), over a patch grid in one of four scan
// directions, written back in spatial order.
#pragma once

#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace gla {

// Retention-gate temperature tau = 16 (method section, GLA recurrence paragraph).
constexpr float kTau = 16.0f;
constexpr float kInvTau = 1.0f / kTau;

// Per-device latched status word (first nonzero code wins); read and cleared
// by gla_get_status().  Lives in the library image, so no allocation.
__device__ int g_status;

__device__ __forceinline__ void raise_status(int code) {
    atomicCAS(&g_status, 0, code);
}

// Index checks of the checked build (compiled with -DGLA_CHECKED into libgla_checked.so): a
// computed index outside its buffer latches GLA_ERR_CHECK (10) and the caller skips the access
// instead of making it.  The release build compiles every check to `true`.
#ifdef GLA_CHECKED
__device__ __forceinline__ bool gla_check(bool ok) {
    if (!ok) raise_status(10 /* GLA_ERR_CHECK */);
    return ok;
}
#define GLA_CHECK(cond) ::gla::gla_check(cond)
#else
#define GLA_CHECK(cond) true
#endif

// Scan position p -> row-major spatial index y*gw + x.
//   0 L->R: row y = p / gw, x = p % gw
//   1 R->L: row y = p / gw, x = gw-1 - p % gw
//   2 T->B: column x = p / gh, y = p % gh
//   3 B->T: column x = p / gh, y = gh-1 - p % gh
__device__ __forceinline__ int spatial_of(int dir, int p, int gh, int gw) {
    int x, y;
    if (dir <= 1) {
        y = p / gw;
        x = p - y * gw;
        if (dir == 1) x = gw - 1 - x;
    } else {
        x = p / gh;
        y = p - x * gh;
        if (dir == 3) y = gh - 1 - y;
    }
    return y * gw + x;
}

// log(gamma) = log(sigma(a)) / tau, stable for either sign of a:
// log sigma(a) = min(a, 0) - log(1 + exp(-|a|)).
__device__ __forceinline__ float log_gamma(float a) {
    return (fminf(a, 0.0f) - log1pf(expf(-fabsf(a)))) * kInvTau;
}

__device__ __forceinline__ float silu(float g) {
    return g / (1.0f + expf(-g));
}

template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__half>(__half x) { return __half2float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __half from_f32<__half>(float x) { return __float2half_rn(x); }

}  // namespace gla
