// gla_api.cu -- the C ABI of libgla.so (declared in include/gla.h).
//
// Argument validation, schedule selection and kernel launches for the
// key-only GLA token mixer of the GTR paper (arXiv 2609.26590, method
// section).  Every step of the operation runs in the kernels included here;
// this file only checks arguments, picks launch shapes and launches.
#include <cstddef>
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cuda_runtime.h>

#include "gla.h"
#include "gla_common.cuh"
#include "gla_simt.cuh"

#define GLA_VERSION_CODE 100  // 0.1.0

namespace gla {
namespace {

struct Args {
    const void *q, *k, *v, *a, *g;
    const float *w;
    void *out;
    int B, H, gh, gw, dk, dv, dir;
    int elem;  // bytes per I/O element
};

bool is_supported_dim(int d) { return d == 32 || d == 64 || d == 128; }

bool ranges_overlap(const void *p, size_t pn, const void *o, size_t on) {
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(p), a1 = a0 + pn;
    const uintptr_t b0 = reinterpret_cast<uintptr_t>(o), b1 = b0 + on;
    return a0 < b1 && b0 < a1;
}

// Host-side checks, no CUDA call: returns a gla_status.
int validate(const Args &x) {
    if (!x.q || !x.k || !x.v || !x.a || !x.g || !x.w || !x.out) return GLA_ERR_NULL;
    if (x.B <= 0 || x.H <= 0 || x.gh <= 0 || x.gw <= 0) return GLA_ERR_SHAPE;
    if (x.dir < 0 || x.dir > 4) return GLA_ERR_DIRECTION;
    if (!is_supported_dim(x.dk) || !is_supported_dim(x.dv)) return GLA_ERR_UNSUPPORTED;
    // token-row indices (b*L + s)*H + h are kept in int32
    const long long rowsN = (long long)x.B * x.gh * x.gw * x.H;
    if ((long long)x.gh * x.gw > (1LL << 30) || rowsN >= (1LL << 31)) return GLA_ERR_SHAPE;
    const void *ptrs[7] = {x.q, x.k, x.v, x.a, x.g, x.w, x.out};
    for (const void *ptr : ptrs)
        if (reinterpret_cast<uintptr_t>(ptr) & 15u) return GLA_ERR_UNSUPPORTED;
    const size_t nk = (size_t)rowsN * x.dk * x.elem, nv = (size_t)rowsN * x.dv * x.elem;
    if (ranges_overlap(x.q, nk, x.out, nv) || ranges_overlap(x.k, nk, x.out, nv) ||
        ranges_overlap(x.a, nk, x.out, nv) || ranges_overlap(x.v, nv, x.out, nv) ||
        ranges_overlap(x.g, nv, x.out, nv) ||
        ranges_overlap(x.w, (size_t)x.dv * sizeof(float), x.out, nv))
        return GLA_ERR_ALIAS;
    return GLA_OK;
}

struct DeviceInfo {
    int sms = 0;
    int major = 0;
    int max_smem_optin = 0;
    bool ok = false;
};

DeviceInfo device_info(int dev) {
    static std::mutex mu;
    static DeviceInfo cache[64];
    static bool have[64] = {};
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 0 || dev >= 64) return DeviceInfo{};
    if (!have[dev]) {
        DeviceInfo d;
        if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess &&
            cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev) == cudaSuccess &&
            cudaDeviceGetAttribute(&d.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) ==
                cudaSuccess)
            d.ok = (d.major == 10);
        cache[dev] = d;
        have[dev] = true;
    }
    return cache[dev];
}

int current_device_info(DeviceInfo *info) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return GLA_ERR_NO_DEVICE;
    }
    *info = device_info(dev);
    return info->ok ? GLA_OK : GLA_ERR_NO_DEVICE;
}

int ceil_div(long long a, long long b) { return (int)((a + b - 1) / b); }

// True when at least one cluster of this launch shape can be resident.
template <typename K>
bool cluster_fits(K kern, const cudaLaunchConfig_t &cfg) {
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return n > 0;
}

// ---------------------------------------------------------------- SIMT path
template <typename T, int DK, int DV>
int launch_simt_t(const Args &x, int chunk, int segs, float eps, cudaStream_t st,
                  const DeviceInfo &di) {
    auto kern = gla_simt_kernel<T, DK, DV>;
    const int L = x.gh * x.gw;
    const int n_pairs = x.B * x.H;
    if (chunk <= 0) chunk = 16;
    if (chunk % 16 != 0 || chunk > 64) return GLA_ERR_UNSUPPORTED;
    const size_t smem = simt_smem_floats(DK, DV, chunk) * sizeof(float);
    if (smem > (size_t)di.max_smem_optin) return GLA_ERR_UNSUPPORTED;
    const bool auto_segs = segs <= 0;
    if (auto_segs) {
        segs = ceil_div(di.sms, n_pairs);
        segs = segs < 1 ? 1 : (segs > 16 ? 16 : segs);
    }
    if (segs > 16) return GLA_ERR_UNSUPPORTED;
    const int n_chunks = ceil_div(L, chunk);
    int seg_len = 0;
    auto plan = [&](int s) {  // whole chunks per segment, no empty segment
        if (s > n_chunks) s = n_chunks;
        seg_len = ceil_div(n_chunks, s) * chunk;
        return ceil_div(L, seg_len);
    };
    segs = plan(segs);

    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess ||
        cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
        cudaGetLastError();
        return GLA_ERR_CUDA;
    }

    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    auto configure = [&](int s) {
        cfg = cudaLaunchConfig_t{};
        cfg.gridDim = dim3((unsigned)(n_pairs * s), 1, 1);
        cfg.blockDim = dim3(kSimtThreads, 1, 1);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = st;
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)s;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    };
    configure(segs);
    while (!cluster_fits(kern, cfg)) {
        if (!auto_segs || segs == 1) return GLA_ERR_UNSUPPORTED;
        segs = plan((segs + 1) / 2);
        configure(segs);
    }
    SimtParams p;
    p.q = x.q; p.k = x.k; p.v = x.v; p.a = x.a; p.g = x.g; p.w = x.w; p.out = x.out;
    p.B = x.B; p.H = x.H; p.gh = x.gh; p.gw = x.gw; p.L = L;
    p.dir = x.dir; p.chunk = chunk; p.segs = segs; p.seg_len = seg_len;
    p.eps = eps; p.scale = 1.0f / sqrtf((float)DK);
    if (cudaLaunchKernelEx(&cfg, kern, p) != cudaSuccess) {
        cudaGetLastError();
        return GLA_ERR_CUDA;
    }
    return GLA_OK;
}

template <typename T, int DK>
int launch_simt_dv(const Args &x, int chunk, int segs, float eps, cudaStream_t st, const DeviceInfo &di) {
    switch (x.dv) {
    case 32: return launch_simt_t<T, DK, 32>(x, chunk, segs, eps, st, di);
    case 64: return launch_simt_t<T, DK, 64>(x, chunk, segs, eps, st, di);
    default: return launch_simt_t<T, DK, 128>(x, chunk, segs, eps, st, di);
    }
}

template <typename T>
int launch_simt(const Args &x, int chunk, int segs, float eps, cudaStream_t st, const DeviceInfo &di) {
    switch (x.dk) {
    case 32: return launch_simt_dv<T, 32>(x, chunk, segs, eps, st, di);
    case 64: return launch_simt_dv<T, 64>(x, chunk, segs, eps, st, di);
    default: return launch_simt_dv<T, 128>(x, chunk, segs, eps, st, di);
    }
}

// ------------------------------------------------------------- dispatch
constexpr float kEps = 1e-6f;

int run(const Args &x, int dtype, int chunk, int segs, float eps, cudaStream_t st) {
    int rc = validate(x);
    if (rc != GLA_OK) return rc;
    if (segs < 0 || segs > 16 || chunk < 0 || !(eps >= 0.0f)) return GLA_ERR_UNSUPPORTED;
    DeviceInfo di;
    rc = current_device_info(&di);
    if (rc != GLA_OK) return rc;
    if (dtype == 1) return launch_simt<float>(x, chunk, segs, eps, st, di);
    return launch_simt<__half>(x, chunk, segs, eps, st, di);
}

Args make_args(const void *q, const void *k, const void *v, const void *a, const void *g,
               const float *w, void *out, int B, int H, int gh, int gw, int dk, int dv, int dir,
               int elem) {
    Args x;
    x.q = q; x.k = k; x.v = v; x.a = a; x.g = g; x.w = w; x.out = out;
    x.B = B; x.H = H; x.gh = gh; x.gw = gw; x.dk = dk; x.dv = dv; x.dir = dir; x.elem = elem;
    return x;
}

// Library-owned device buffers behind gla_fwd_host, one set per device.
struct HostStaging {
    void *buf = nullptr;
    size_t cap = 0;
};

}  // namespace
}  // namespace gla

using namespace gla;

extern "C" {

int gla_fwd(const void *q, const void *k, const void *v, const void *gate_preact,
            const void *out_gate_preact, const float *rms_weight, void *out, int B, int H,
            int grid_h, int grid_w, int d_k, int d_v, int direction, void *stream) {
    const Args x = make_args(q, k, v, gate_preact, out_gate_preact, rms_weight, out, B, H, grid_h,
                             grid_w, d_k, d_v, direction, 2);
    return run(x, 0, 0, 0, kEps, static_cast<cudaStream_t>(stream));
}

int gla_fwd_f32(const float *q, const float *k, const float *v, const float *gate_preact,
                const float *out_gate_preact, const float *rms_weight, float *out, int B, int H,
                int grid_h, int grid_w, int d_k, int d_v, int direction, void *stream) {
    const Args x = make_args(q, k, v, gate_preact, out_gate_preact, rms_weight, out, B, H, grid_h,
                             grid_w, d_k, d_v, direction, 4);
    return run(x, 1, 0, 0, kEps, static_cast<cudaStream_t>(stream));
}

int gla_fwd_ex(const void *q, const void *k, const void *v, const void *gate_preact,
               const void *out_gate_preact, const float *rms_weight, void *out, int B, int H,
               int grid_h, int grid_w, int d_k, int d_v, int direction, int dtype, int chunk,
               int segments, float eps, void *stream) {
    if (dtype != 0 && dtype != 1) return GLA_ERR_UNSUPPORTED;
    const Args x = make_args(q, k, v, gate_preact, out_gate_preact, rms_weight, out, B, H, grid_h,
                             grid_w, d_k, d_v, direction, dtype == 0 ? 2 : 4);
    return run(x, dtype, chunk, segments, eps, static_cast<cudaStream_t>(stream));
}

int gla_fwd_host(const void *q, const void *k, const void *v, const void *gate_preact,
                 const void *out_gate_preact, const float *rms_weight, void *out, int B, int H,
                 int grid_h, int grid_w, int d_k, int d_v, int direction, int dtype, void *stream) {
    if (dtype != 0 && dtype != 1) return GLA_ERR_UNSUPPORTED;
    const int elem = dtype == 0 ? 2 : 4;
    Args hx = make_args(q, k, v, gate_preact, out_gate_preact, rms_weight, out, B, H, grid_h,
                        grid_w, d_k, d_v, direction, elem);
    int rc = validate(hx);
    if (rc != GLA_OK) return rc;
    DeviceInfo di;
    rc = current_device_info(&di);
    if (rc != GLA_OK) return rc;
    int dev = 0;
    cudaGetDevice(&dev);

    static std::mutex mu;
    static HostStaging staging[64];
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 0 || dev >= 64) return GLA_ERR_NO_DEVICE;
    HostStaging &hs = staging[dev];

    const size_t rowsN = (size_t)B * grid_h * grid_w * H;
    auto up16 = [](size_t n) { return (n + 255) & ~(size_t)255; };
    const size_t nk = rowsN * d_k * elem, nv = rowsN * d_v * elem, nw = (size_t)d_v * sizeof(float);
    const size_t total = 3 * up16(nk) + 3 * up16(nv) + up16(nw);
    if (hs.cap < total) {
        if (hs.buf) cudaFree(hs.buf);
        hs.buf = nullptr;
        hs.cap = 0;
        if (cudaMalloc(&hs.buf, total) != cudaSuccess) {
            cudaGetLastError();
            return GLA_ERR_CUDA;
        }
        hs.cap = total;
    }
    char *base = static_cast<char *>(hs.buf);
    char *dq = base, *dk_ = dq + up16(nk), *da = dk_ + up16(nk), *dv_ = da + up16(nk);
    char *dg = dv_ + up16(nv), *dout = dg + up16(nv), *dw = dout + up16(nv);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const struct { void *dst; const void *src; size_t n; } up[6] = {
        {dq, q, nk}, {dk_, k, nk}, {da, gate_preact, nk}, {dv_, v, nv}, {dg, out_gate_preact, nv},
        {dw, rms_weight, nw}};
    for (const auto &c : up) {
        if (cudaMemcpyAsync(c.dst, c.src, c.n, cudaMemcpyHostToDevice, st) != cudaSuccess) {
            cudaGetLastError();
            return GLA_ERR_CUDA;
        }
    }
    const Args dx = make_args(dq, dk_, dv_, da, dg, reinterpret_cast<const float *>(dw), dout, B, H,
                              grid_h, grid_w, d_k, d_v, direction, elem);
    rc = run(dx, dtype, 0, 0, kEps, st);
    if (rc != GLA_OK) return rc;
    if (cudaMemcpyAsync(out, dout, nv, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess) {
        cudaGetLastError();
        return GLA_ERR_CUDA;
    }
    return GLA_OK;
}

int gla_get_status(void *stream, int *device_status) {
    if (!device_status) return GLA_ERR_NULL;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int value = 0, zero = 0;
    if (cudaStreamSynchronize(st) != cudaSuccess ||
        cudaMemcpyFromSymbol(&value, g_status, sizeof(int)) != cudaSuccess ||
        cudaMemcpyToSymbol(g_status, &zero, sizeof(int)) != cudaSuccess) {
        cudaGetLastError();
        return GLA_ERR_CUDA;
    }
    *device_status = value;
    return GLA_OK;
}

const char *gla_status_string(int code) {
    switch (code) {
    case GLA_OK: return "GLA_OK";
    case GLA_ERR_NULL: return "GLA_ERR_NULL: a required pointer is NULL";
    case GLA_ERR_SHAPE: return "GLA_ERR_SHAPE: non-positive or too large shape";
    case GLA_ERR_UNSUPPORTED: return "GLA_ERR_UNSUPPORTED: head dim, alignment or schedule not supported";
    case GLA_ERR_DIRECTION: return "GLA_ERR_DIRECTION: direction must be 0..4";
    case GLA_ERR_ALIAS: return "GLA_ERR_ALIAS: out overlaps an input";
    case GLA_ERR_CUDA: return "GLA_ERR_CUDA: CUDA runtime or launch error";
    case GLA_ERR_TIMEOUT: return "GLA_ERR_TIMEOUT: a bounded device wait ran out";
    case GLA_ERR_RANGE: return "GLA_ERR_RANGE: an intermediate left the supported operand range";
    case GLA_ERR_NO_DEVICE: return "GLA_ERR_NO_DEVICE: no usable sm_100 device is current";
    default: return "unknown gla status";
    }
}

int gla_version(void) { return GLA_VERSION_CODE; }

}  // extern "C"
