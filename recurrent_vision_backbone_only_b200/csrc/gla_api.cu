// gla_api.cu -- the C ABI of libgla.so (declared in include/gla.h).
//
// Argument validation, schedule selection and kernel launches for the
// key-only GLA token mixer of the GTR paper (arXiv 2609.26590, method
// section).  Every step of the operation runs in the kernels included here;
// this file only checks arguments, picks launch shapes and launches.
#include <cmath>
#include <cstddef>
#include <cstdint>
#include <algorithm>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "gla.h"
#include "gla_chunk.cuh"
#include "gla_pipe.cuh"
#include "gla_gate.cuh"
#include "gla_sswiglu.cuh"
#include "gla_linear.cuh"
#include "gla_common.cuh"
#include "gla_simt.cuh"
#include "gla_tc.cuh"

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

// Kernels: 1 = 128-row tensor-core kernel (fp16, d_k = d_v = 64), 2 = CUDA-core kernel (any
// supported shape, fp16 or fp32), 3 = 64-row tensor-core kernel (fp16, d_k = d_v in {64, 128}),
// 4 = the 64-row kernel with two chunks in flight (fp16, d_k = d_v = 64).
enum { kAuto = 0, kTc128 = 1, kSimt = 2, kTc64 = 3, kPipe64 = 4 };

// Launch schedule: `segs` CTAs (one thread-block cluster) per (b, h) pair,
// each owning `seg_len` consecutive scan positions.
struct Plan {
    int kernel = 0;            // 1 = tensor-core kernel, 2 = CUDA-core kernel
    int segs = 1;
    int seg_len = 0;
    int chunk = 0;             // tokens per chunk (CUDA-core) / largest chunk (tensor-core)
    size_t smem = 0;
    int max_active_clusters = 0;
    int ctas = 0;              // CTAs of all launches
    int tail_pairs = 0;        // pipelined kernel: pairs of a second launch (0: none) ...
    int tail_segs = 0;         // ... with this many segments per pair
    cudaLaunchConfig_t cfg{};
    cudaLaunchAttribute attr[2];
    bool pdl = false;          // programmatic dependent launch (tensor-core kernel)
};

void configure_launch(Plan &pl, int n_pairs, int threads, cudaStream_t st) {
    pl.cfg = cudaLaunchConfig_t{};
    pl.cfg.gridDim = dim3((unsigned)(n_pairs * pl.segs), 1, 1);
    pl.cfg.blockDim = dim3((unsigned)threads, 1, 1);
    pl.cfg.dynamicSmemBytes = pl.smem;
    pl.cfg.stream = st;
    pl.attr[0].id = cudaLaunchAttributeClusterDimension;
    pl.attr[0].val.clusterDim.x = (unsigned)pl.segs;
    pl.attr[0].val.clusterDim.y = 1;
    pl.attr[0].val.clusterDim.z = 1;
    pl.cfg.attrs = pl.attr;
    pl.cfg.numAttrs = 1;
    if (pl.pdl) {
        pl.attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        pl.attr[1].val.programmaticStreamSerializationAllowed = 1;
        pl.cfg.numAttrs = 2;
    }
}

// Clusters of `size` CTAs of this launch shape the device holds at once (0 = none).
template <typename K>
int active_clusters(K kern, Plan &pl, int n_pairs, int size, int threads, cudaStream_t st) {
    Plan probe = pl;
    probe.segs = size;
    configure_launch(probe, n_pairs, threads, st);
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &probe.cfg) != cudaSuccess) {
        cudaGetLastError();
        n = 0;
    }
    return n;
}

// Tensor-core schedule cost model, relative units (a full 128-token chunk ~ 1): a chunk of
// n tokens costs 0.45 + 0.55 n/128 (fixed latency chain + per-token work); a segment of
// one chunk runs resident and adds 0.15 for the exchange; a longer segment that exchanges
// first runs a state-only pass (~0.4 per chunk) and the exchange (0.2); a launch takes
// ceil(pairs / resident clusters) waves.
double tc_cost(int L, int n_pairs, int segs, int active) {
    if (active <= 0) return 1e30;
    const int seg_len = ceil_div(L, segs);
    const int s_eff = ceil_div(L, seg_len);
    const int chunks = ceil_div(seg_len, 128);
    const double chunk_len = (double)seg_len / chunks;
    const double per_chunk = 0.45 + 0.55 * chunk_len / 128.0;
    double per_cta = chunks * per_chunk;
    if (s_eff > 1) per_cta += chunks <= 1 ? 0.15 : chunks * 0.4 + 0.2;
    const int waves = ceil_div(n_pairs, active);
    return waves * per_cta;
}

// The tensor-core kernel's state exchange deals the 16 four-channel key groups out to the
// segments; a scanner's receive buffer holds ceil(16/segs) groups from every segment, so
// ceil(16/segs) * segs must not exceed tc::kMaxGroupSegs (24).
bool tc_segs_ok(int segs) { return segs == 1 || ceil_div(16, segs) * segs <= tc::kMaxGroupSegs; }

// Pick the segment count (auto when segs <= 0), shrinking it until a cluster
// fits on the device.  `unit` is the granularity of a segment's length.  With a
// cost model (tensor-core kernel) every cluster size 1..16 is scored instead.
template <typename K>
int make_plan(K kern, Plan &pl, int L, int n_pairs, int segs, int unit, int threads,
              cudaStream_t st, const DeviceInfo &di, bool cost_model = false) {
    if (pl.smem > (size_t)di.max_smem_optin) return GLA_ERR_UNSUPPORTED;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pl.smem) !=
            cudaSuccess ||
        cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
        cudaGetLastError();
        return GLA_ERR_CUDA;
    }
    const bool auto_segs = segs <= 0;
    if (auto_segs && cost_model) {
        static std::mutex mu;
        static int cache[64][17];
        static bool have[64][17] = {};
        int dev = 0;
        cudaGetDevice(&dev);
        double best = 1e30;
        int best_s = 1;
        for (int cand = 1; cand <= 16 && cand <= L; ++cand) {
            const int s_eff = ceil_div(L, ceil_div(L, cand));
            if (s_eff != cand) continue;           // equal-length segments only
            if (!tc_segs_ok(cand)) continue;        // channel groups must fit the buffer
            int act;
            {
                std::lock_guard<std::mutex> lock(mu);
                if (dev >= 0 && dev < 64 && have[dev][cand]) {
                    act = cache[dev][cand];
                } else {
                    act = active_clusters(kern, pl, n_pairs, cand, threads, st);
                    if (dev >= 0 && dev < 64) {
                        cache[dev][cand] = act;
                        have[dev][cand] = true;
                    }
                }
            }
            const double c = tc_cost(L, n_pairs, cand, act);
            if (c < best - 1e-9) {
                best = c;
                best_s = cand;
            }
        }
        segs = best_s;
    } else if (auto_segs) {
        segs = di.sms / n_pairs;
        segs = segs < 1 ? 1 : (segs > 16 ? 16 : segs);
    }
    if (segs > 16) return GLA_ERR_UNSUPPORTED;
    const int n_units = ceil_div(L, unit);
    auto plan_segs = [&](int s) {  // whole units per segment, none empty
        if (s > n_units) s = n_units;
        pl.seg_len = ceil_div(n_units, s) * unit;
        pl.segs = ceil_div(L, pl.seg_len);
    };
    plan_segs(segs);
    configure_launch(pl, n_pairs, threads, st);
    for (;;) {
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, kern, &pl.cfg) != cudaSuccess) {
            cudaGetLastError();
            n = 0;
        }
        pl.max_active_clusters = n;
        if (n > 0) return GLA_OK;
        if (!auto_segs || pl.segs == 1) return GLA_ERR_UNSUPPORTED;
        int next = (pl.segs + 1) / 2;
        if (cost_model)
            while (next > 1 && !tc_segs_ok(next)) --next;
        plan_segs(next);
        configure_launch(pl, n_pairs, threads, st);
    }
}

// ---------------------------------------------------------------- SIMT path
template <typename T, int DK, int DV>
int run_simt_t(const Args &x, int chunk, int segs, float eps, cudaStream_t st,
               const DeviceInfo &di, Plan *query) {
    auto kern = gla_simt_kernel<T, DK, DV>;
    const int L = x.gh * x.gw;
    const int n_pairs = x.B * x.H;
    if (chunk <= 0) chunk = 16;
    if (chunk % 16 != 0 || chunk > 64) return GLA_ERR_UNSUPPORTED;
    Plan pl;
    pl.kernel = kSimt;
    pl.chunk = chunk;
    pl.smem = simt_smem_floats(DK, DV, chunk) * sizeof(float);
    int rc = make_plan(kern, pl, L, n_pairs, segs, chunk, kSimtThreads, st, di);
    if (rc != GLA_OK) return rc;
    if (query) {
        *query = pl;
        return GLA_OK;
    }
    SimtParams p;
    p.q = x.q; p.k = x.k; p.v = x.v; p.a = x.a; p.g = x.g; p.w = x.w; p.out = x.out;
    p.B = x.B; p.H = x.H; p.gh = x.gh; p.gw = x.gw; p.L = L;
    p.dir = x.dir; p.chunk = chunk; p.segs = pl.segs; p.seg_len = pl.seg_len;
    p.eps = eps; p.scale = 1.0f / sqrtf((float)DK);
    if (cudaLaunchKernelEx(&pl.cfg, kern, p) != cudaSuccess) {
        cudaGetLastError();
        return GLA_ERR_CUDA;
    }
    return GLA_OK;
}

template <typename T, int DK>
int run_simt_dv(const Args &x, int chunk, int segs, float eps, cudaStream_t st, const DeviceInfo &di,
                Plan *query) {
    switch (x.dv) {
    case 32: return run_simt_t<T, DK, 32>(x, chunk, segs, eps, st, di, query);
    case 64: return run_simt_t<T, DK, 64>(x, chunk, segs, eps, st, di, query);
    default: return run_simt_t<T, DK, 128>(x, chunk, segs, eps, st, di, query);
    }
}

template <typename T>
int run_simt(const Args &x, int chunk, int segs, float eps, cudaStream_t st, const DeviceInfo &di,
             Plan *query) {
    switch (x.dk) {
    case 32: return run_simt_dv<T, 32>(x, chunk, segs, eps, st, di, query);
    case 64: return run_simt_dv<T, 64>(x, chunk, segs, eps, st, di, query);
    default: return run_simt_dv<T, 128>(x, chunk, segs, eps, st, di, query);
    }
}

// ---------------------------------------------------------- tensor-core path
// fp16 I/O with d_k = d_v = 64.  One cluster of `segs` CTAs per (b, h) pair.
int run_tc(const Args &x, int chunk, int segs, float eps, cudaStream_t st, const DeviceInfo &di,
           Plan *query, long long wait_limit = 1LL << 32, int fault_chunk = -1) {
    auto kern = tc::gla_tc_kernel<64, false>;
    const int L = x.gh * x.gw;
    const int n_pairs = x.B * x.H;
    if (chunk <= 0) chunk = tc::kC;
    if (chunk % 16 != 0 || chunk > tc::kC) return GLA_ERR_UNSUPPORTED;
    if (segs > 0) {                              // explicit: must fit the exchange slices
        int s_eff = segs > L ? L : segs;
        s_eff = ceil_div(L, ceil_div(L, s_eff));
        if (!tc_segs_ok(s_eff)) return GLA_ERR_UNSUPPORTED;
    }
    Plan pl;
    pl.kernel = kTc128;
    pl.chunk = chunk;
    pl.smem = tc::kSmemBytes;
    pl.pdl = true;
    int rc = make_plan(kern, pl, L, n_pairs, segs, 1, tc::kThreads, st, di, true);
    if (rc != GLA_OK) return rc;
    if (query) {
        *query = pl;
        return GLA_OK;
    }
    tc::Params p;
    p.q = static_cast<const __half *>(x.q); p.k = static_cast<const __half *>(x.k);
    p.v = static_cast<const __half *>(x.v); p.a = static_cast<const __half *>(x.a);
    p.g = static_cast<const __half *>(x.g); p.w = x.w; p.out = static_cast<__half *>(x.out);
    p.B = x.B; p.H = x.H; p.gh = x.gh; p.gw = x.gw; p.L = L; p.dir = x.dir;
    p.segs = pl.segs; p.seg_len = pl.seg_len; p.chunk_max = chunk;
    p.eps = eps; p.scale = 0.125f;  // 64^{-1/2}
    p.wait_limit = wait_limit;
    p.fault_chunk = fault_chunk;
    // every segment one chunk and several segments: the instantiation with only the
    // mid-chunk exchange path (same resources and launch shape as the planned one)
    auto launch = kern;
    if (pl.seg_len <= chunk && pl.segs > 1) {
        launch = tc::gla_tc_kernel<64, true>;
        if (cudaFuncSetAttribute(launch, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pl.smem) !=
                cudaSuccess ||
            cudaFuncSetAttribute(launch, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
            cudaGetLastError();
            return GLA_ERR_CUDA;
        }
    }
    if (cudaLaunchKernelEx(&pl.cfg, launch, p) != cudaSuccess) {
        cudaGetLastError();
        return GLA_ERR_CUDA;
    }
    return GLA_OK;
}

// ---------------------------------------------------------- chunk kernel path
// fp16 I/O with d_k = d_v = D in {64, 128}: gla_chunk_kernel<D>, one cluster of `segs` CTAs per
// (b, h) pair, inputs gathered by TMA through one tensor map per input.

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static std::once_flag once;
    static EncodeTiledFn fn = nullptr;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
        else
            cudaGetLastError();
    });
    return fn;
}

// 3-D views of a token-major fp16 array [B][gh][gw][H][D] whose boxes (64 channels x 1 x 64
// positions, 128B-swizzled) are 64 consecutive positions of one grid row (row family: view
// [B gh gw][H][D]) or of one grid column (column family: view [B gh][gw H][D]) of one head.
bool make_line_map(CUtensorMap *map, const void *base, int fam, int B, int H, int gh, int gw, int D,
                   int rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t mid = fam ? (cuuint64_t)gw * H : (cuuint64_t)H;
    const cuuint64_t outer = fam ? (cuuint64_t)B * gh : (cuuint64_t)B * gh * gw;
    const cuuint64_t dims[3] = {(cuuint64_t)D, mid, outer};
    const cuuint64_t strides[2] = {(cuuint64_t)D * 2, mid * D * 2};
    const cuuint32_t box[3] = {64, 1, (cuuint32_t)rows};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tensor maps of the five inputs for the line families the directions of a launch use; boxes
// of rows[fam] positions (64, or the group height of packed chunks).
bool make_maps(ck::Maps *maps, const void *const src[5], int dir, int B, int H, int gh, int gw, int D,
               const int rows[2]) {
    for (int fam = 0; fam < 2; ++fam) {
        const bool used = dir == 4 || (dir >> 1) == fam;
        if (!used) continue;
        CUtensorMap *dst = fam ? maps->col : maps->row;
        for (int i = 0; i < 5; ++i)
            if (!make_line_map(&dst[i], src[i], fam, B, H, gh, gw, D, rows[fam])) return false;
    }
    return true;
}

// Shared memory requested per CTA: the kernel's own need, or (spread) enough that one CTA fills
// an SM's shared memory, so a launch whose CTAs fit on the device gets one SM per CTA.
template <int D>
size_t chunk_smem(bool spread) {
    const size_t need = ck::smem_bytes<D>();
    return spread && need < 120 * 1024 ? 120 * 1024 : need;
}

// Schedule cost of `segs` segments per pair (a scan of `q` chunks), in units of one full-pass
// chunk on an SM of its own: every full chunk 1, a state-only chunk 0.35, the exchange
// 0.5 + 0.04 segs; CTAs beyond one per SM share SMs (x 1.4 each when two share), and a launch
// takes ceil(pairs / resident clusters) waves.
double chunk_cost(int q, int n_pairs, int segs, int sms, int active1, int active2) {
    const int chunks = ceil_div(q, segs);
    double per_cta = chunks;
    if (segs > 1) per_cta += chunks * 0.35 + 0.5 + 0.04 * segs;
    const long long ctas = (long long)n_pairs * segs;
    if (ctas <= sms && active1 > 0) return per_cta * ceil_div(n_pairs, active1);
    if (active2 <= 0) return 1e30;
    return per_cta * 1.4 * ceil_div(n_pairs, active2);
}

template <int D, bool kPipe = false>
int run_chunk(const Args &x, int chunk, int segs, float eps, cudaStream_t st, const DeviceInfo &di,
              Plan *query, long long wait_limit = 1LL << 32, int fault_chunk = -1) {
    static_assert(!kPipe || D == 64, "the pipelined kernel handles d = 64");
    auto kern = kPipe ? ck::gla_pipe_kernel : ck::gla_chunk_kernel<D>;
    using C = ck::Cfg<D>;
    constexpr int kThreads = kPipe ? ck::PipeCfg::kThreads : C::kThreads;
    const int L = x.gh * x.gw;
    const int n_pairs = x.B * x.H;
    if (chunk <= 0) chunk = ck::kC;
    if (chunk % 16 != 0 || chunk > ck::kC) return GLA_ERR_UNSUPPORTED;
    // chunks per scan: the pipelined kernel packs chunks across lines where the line length
    // allows (hb > 0), the other cuts lines into pieces of at most `chunk` positions; a cycling
    // launch mixes both line families
    int hb[2] = {0, 0};
    if (kPipe) {
        hb[0] = ck::box_rows(x.dir, 0, x.gh, x.gw, chunk);
        hb[1] = ck::box_rows(x.dir, 1, x.gh, x.gw, chunk);
    }
    int q = 0, clen = 0;
    for (int dir = 0; dir < 4; ++dir)
        if (x.dir == 4 || x.dir == dir) {
            const ck::Scan sc(dir, x.gh, x.gw, chunk, hb[dir >> 1]);
            q = std::max(q, sc.chunks);
            clen = std::max(clen, sc.cl);
        }
    const size_t smem_max = kPipe ? ck::pipe_smem_bytes() : chunk_smem<D>(true);
    if (smem_max > (size_t)di.max_smem_optin) return GLA_ERR_UNSUPPORTED;
    // all of the unified L1 / shared memory as shared memory, so two d = 64 CTAs fit on an SM
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_max) != cudaSuccess ||
        cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared) != cudaSuccess ||
        cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
        cudaGetLastError();
        return GLA_ERR_CUDA;
    }
    Plan pl;
    pl.kernel = kPipe ? kPipe64 : kTc64;
    pl.chunk = chunk;
    pl.pdl = true;
    auto smem_of = [&](bool spread) { return kPipe ? ck::pipe_smem_bytes() : chunk_smem<D>(spread); };
    auto clusters = [&](int size, bool spread) {
        Plan probe = pl;
        probe.segs = size;
        probe.smem = smem_of(spread);
        configure_launch(probe, n_pairs, kThreads, st);
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, kern, &probe.cfg) != cudaSuccess) {
            cudaGetLastError();
            n = 0;
        }
        return n;
    };
    const bool auto_segs = segs <= 0;
    if (segs <= 0) {
        static std::mutex mu;
        static int cache[64][2][17];
        static bool have[64][2][17] = {};
        int dev = 0;
        cudaGetDevice(&dev);
        auto cached = [&](int size, bool spread) {
            std::lock_guard<std::mutex> lock(mu);
            if (dev < 0 || dev >= 64) return clusters(size, spread);
            if (!have[dev][spread][size]) {
                cache[dev][spread][size] = clusters(size, spread);
                have[dev][spread][size] = true;
            }
            return cache[dev][spread][size];
        };
        double best = 1e30;
        int best_s = 1;
        for (int cand = 1; cand <= 16 && cand <= q; ++cand) {
            if (ceil_div(q, ceil_div(q, cand)) != cand) continue;     // no empty segment
            const double c = chunk_cost(q, n_pairs, cand, di.sms, cached(cand, true), cached(cand, false));
            if (c < best - 1e-9) {
                best = c;
                best_s = cand;
            }
        }
        segs = best_s;
    }
    if (segs > 16) return GLA_ERR_UNSUPPORTED;
    // Throughput launches of the pipelined kernel (one CTA per pair, more pairs than the device
    // holds) end with a partial wave.  Whole waves stay one CTA per pair; the remaining pairs go
    // to a second launch that cuts each into segments, so they fill the device instead of a
    // fraction of it.  The second launch waits for the first (dependent launch), which ends
    // with its whole waves.
    int head_pairs = n_pairs;
    if (kPipe && auto_segs && segs == 1) {
        const int wave = clusters(1, false);          // resident one-CTA clusters
        const int rem = wave > 0 ? n_pairs % wave : 0;
        if (wave > 0 && n_pairs > wave && rem > 0 && 2 * rem <= wave) {
            int s2 = std::min(std::min(16, q), wave / rem);
            while (s2 > 1 && (ceil_div(q, ceil_div(q, s2)) != s2 || clusters(s2, false) < rem)) --s2;
            if (s2 > 1) {
                head_pairs = n_pairs - rem;
                pl.tail_pairs = rem;
                pl.tail_segs = s2;
            }
        }
    }
    pl.segs = segs;
    pl.seg_len = std::min(L, ceil_div(q, segs) * clen);
    const bool spread = (long long)n_pairs * pl.segs <= di.sms;
    pl.smem = smem_of(spread);
    configure_launch(pl, head_pairs, kThreads, st);
    pl.max_active_clusters = clusters(pl.segs, spread);
    if (pl.max_active_clusters <= 0) return GLA_ERR_UNSUPPORTED;
    pl.ctas = head_pairs * pl.segs + pl.tail_pairs * pl.tail_segs;
    if (query) {
        *query = pl;
        return GLA_OK;
    }
    ck::Maps maps;
    const void *const src[5] = {x.q, x.k, x.a, x.v, x.g};
    const int rows[2] = {hb[0] > 0 ? hb[0] : 64, hb[1] > 0 ? hb[1] : 64};
    if (!make_maps(&maps, src, x.dir, x.B, x.H, x.gh, x.gw, D, rows)) return GLA_ERR_CUDA;
    ck::Params p;
    p.out = static_cast<__half *>(x.out);
    p.w = x.w;
    p.B = x.B; p.H = x.H; p.gh = x.gh; p.gw = x.gw; p.L = L; p.dir = x.dir;
    p.segs = pl.segs; p.chunk_max = chunk;
    p.eps = eps;
    p.scale = 1.0f / sqrtf((float)D);
    p.log2_scale = (float)(-0.5 * std::log2((double)D));
    p.wait_limit = wait_limit;
    p.fault_chunk = fault_chunk;
    p.hb[0] = hb[0];
    p.hb[1] = hb[1];
    p.pair0 = 0;
    if (cudaLaunchKernelEx(&pl.cfg, kern, maps, p) != cudaSuccess) {
        cudaGetLastError();
        return GLA_ERR_CUDA;
    }
    if (pl.tail_pairs > 0) {
        Plan tail = pl;
        tail.segs = pl.tail_segs;
        configure_launch(tail, pl.tail_pairs, kThreads, st);
        p.segs = tail.segs;
        p.pair0 = head_pairs;
        if (cudaLaunchKernelEx(&tail.cfg, kern, maps, p) != cudaSuccess) {
            cudaGetLastError();
            return GLA_ERR_CUDA;
        }
    }
    return GLA_OK;
}

// ------------------------------------------------------------- dispatch
constexpr float kEps = 1e-6f;

// The kernel gla_fwd uses: fp32 I/O on CUDA cores; fp16 d = 64 on the pipelined 64-row kernel
// when the launch has at least one (b, h) pair per SM (throughput-bound: one CTA per pair, two
// chunks in flight) or scans of at least 4096 positions (segments of many chunks: 80 x 80 with
// 10 segments per pair measured 71.6 us against 73.5 us), else on the 128-row kernel
// (latency-bound: one chunk per segment and a mid-chunk exchange; 40 x 40 measured 11.9 us
// against 28 us); fp16 d = 128 on the 64-row kernel (the only one that holds its tiles); other
// head dims on CUDA cores.
int auto_kernel(const Args &x, int dtype, const DeviceInfo &di) {
    if (dtype == 1) return kSimt;
    if (x.dk == 64 && x.dv == 64)
        return ((long long)x.B * x.H >= di.sms || (long long)x.gh * x.gw >= 4096) ? kPipe64 : kTc128;
    if (x.dk == 128 && x.dv == 128) return kTc64;
    return kSimt;
}

// Validate, then launch (query == nullptr) or only report the schedule.
int run(const Args &x, int dtype, int chunk, int segs, float eps, cudaStream_t st,
        Plan *query = nullptr, int kernel = kAuto) {
    int rc = validate(x);
    if (rc != GLA_OK) return rc;
    if (segs < 0 || segs > 16 || chunk < 0 || !(eps >= 0.0f)) return GLA_ERR_UNSUPPORTED;
    if (kernel < kAuto || kernel > kPipe64) return GLA_ERR_UNSUPPORTED;
    if (kernel == kTc128 && !(dtype == 0 && x.dk == 64 && x.dv == 64)) return GLA_ERR_UNSUPPORTED;
    if (kernel == kTc64 && !(dtype == 0 && x.dk == x.dv && (x.dk == 64 || x.dk == 128)))
        return GLA_ERR_UNSUPPORTED;
    if (kernel == kPipe64 && !(dtype == 0 && x.dk == 64 && x.dv == 64)) return GLA_ERR_UNSUPPORTED;
    DeviceInfo di;
    rc = current_device_info(&di);
    if (rc != GLA_OK) return rc;
    if (kernel == kAuto) kernel = auto_kernel(x, dtype, di);
    if (kernel == kTc128) return run_tc(x, chunk, segs, eps, st, di, query);
    if (kernel == kTc64)
        return x.dk == 64 ? run_chunk<64>(x, chunk, segs, eps, st, di, query)
                          : run_chunk<128>(x, chunk, segs, eps, st, di, query);
    if (kernel == kPipe64) return run_chunk<64, true>(x, chunk, segs, eps, st, di, query);
    if (dtype == 1) return run_simt<float>(x, chunk, segs, eps, st, di, query);
    return run_simt<__half>(x, chunk, segs, eps, st, di, query);
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
               int segments, float eps, int kernel, void *stream) {
    if (dtype != 0 && dtype != 1) return GLA_ERR_UNSUPPORTED;
    const Args x = make_args(q, k, v, gate_preact, out_gate_preact, rms_weight, out, B, H, grid_h,
                             grid_w, d_k, d_v, direction, dtype == 0 ? 2 : 4);
    return run(x, dtype, chunk, segments, eps, static_cast<cudaStream_t>(stream), nullptr, kernel);
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
    case GLA_ERR_CHECK: return "GLA_ERR_CHECK: an index check of the checked build failed";
    case GLA_ERR_RANGE: return "GLA_ERR_RANGE: an intermediate left the supported operand range";
    case GLA_ERR_NO_DEVICE: return "GLA_ERR_NO_DEVICE: no usable sm_100 device is current";
    default: return "unknown gla status";
    }
}

int gla_version(void) { return GLA_VERSION_CODE; }

int gla_plan(int B, int H, int grid_h, int grid_w, int d_k, int d_v, int dtype, int *kernel,
             int *segments, int *seg_len, int *ctas, int *max_active_clusters) {
    if (!kernel || !segments || !seg_len || !ctas || !max_active_clusters) return GLA_ERR_NULL;
    if (dtype != 0 && dtype != 1) return GLA_ERR_UNSUPPORTED;
    // placeholder, 16-byte aligned, non-overlapping addresses: only shapes are used
    static const uintptr_t kFake = 1u << 20;
    const size_t span = (size_t)B * grid_h * grid_w * H * 128 * 4 + 4096;
    const uintptr_t base = kFake;
    const Args x = make_args(reinterpret_cast<const void *>(base), reinterpret_cast<const void *>(base + span),
                             reinterpret_cast<const void *>(base + 2 * span),
                             reinterpret_cast<const void *>(base + 3 * span),
                             reinterpret_cast<const void *>(base + 4 * span),
                             reinterpret_cast<const float *>(base + 5 * span),
                             reinterpret_cast<void *>(base + 6 * span), B, H, grid_h, grid_w, d_k, d_v,
                             0, dtype == 0 ? 2 : 4);
    Plan pl;
    const int rc = run(x, dtype, 0, 0, kEps, nullptr, &pl);
    if (rc != GLA_OK) return rc;
    *kernel = pl.kernel;
    *segments = pl.segs;
    *seg_len = pl.seg_len;
    *ctas = pl.ctas > 0 ? pl.ctas : B * H * pl.segs;
    *max_active_clusters = pl.max_active_clusters;
    return GLA_OK;
}

int gla_empty_launch(int B, int H, int grid_h, int grid_w, void *stream) {
    if (B <= 0 || H <= 0 || grid_h <= 0 || grid_w <= 0) return GLA_ERR_SHAPE;
    if (B > (1 << 20) || H > (1 << 20)) return GLA_ERR_SHAPE;
    // the plan gla_fwd makes for fp16 d_k = d_v = 64 at these dimensions (placeholder pointers:
    // only the shapes are used)
    static const uintptr_t kFake = 1u << 20;
    const size_t span = (size_t)B * grid_h * grid_w * H * 128 + 4096;
    const Args x = make_args(reinterpret_cast<const void *>(kFake), reinterpret_cast<const void *>(kFake + span),
                             reinterpret_cast<const void *>(kFake + 2 * span),
                             reinterpret_cast<const void *>(kFake + 3 * span),
                             reinterpret_cast<const void *>(kFake + 4 * span),
                             reinterpret_cast<const float *>(kFake + 5 * span),
                             reinterpret_cast<void *>(kFake + 6 * span), B, H, grid_h, grid_w, 64, 64, 0, 2);
    Plan pl;
    int rc = run(x, 0, 0, 0, kEps, static_cast<cudaStream_t>(stream), &pl);
    if (rc != GLA_OK) return rc;
    if (pl.kernel != kTc128 && pl.kernel != kTc64 && pl.kernel != kPipe64) return GLA_ERR_UNSUPPORTED;
    auto kern = pl.kernel == kTc128 ? tc::gla_empty_kernel : ck::gla_chunk_empty_kernel;
    const int threads = pl.kernel == kTc128  ? tc::kThreads
                        : pl.kernel == kTc64 ? ck::Cfg<64>::kThreads
                                             : ck::PipeCfg::kThreads;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pl.smem) != cudaSuccess ||
        cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
        cudaGetLastError();
        return GLA_ERR_CUDA;
    }
    configure_launch(pl, B * H, threads, static_cast<cudaStream_t>(stream));
    if (cudaLaunchKernelEx(&pl.cfg, kern) != cudaSuccess) {
        cudaGetLastError();
        return GLA_ERR_CUDA;
    }
    return GLA_OK;
}

int gla_selftest_timeout(long long limit_cycles, void *stream) {
    if (limit_cycles <= 0 || limit_cycles > (1LL << 34)) return GLA_ERR_UNSUPPORTED;
    DeviceInfo di;
    int rc = current_device_info(&di);
    if (rc != GLA_OK) return rc;
    tc::gla_timeout_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_cycles);
    if (cudaGetLastError() != cudaSuccess) return GLA_ERR_CUDA;
    return GLA_OK;
}

int gla_selftest_chunk(int d, int kind, const float *A, const float *B, float *Dm, void *stream) {
    if (!A || !B || !Dm) return GLA_ERR_NULL;
    if ((d != 64 && d != 128) || kind < 0 || kind > 4 || (kind == 4 && d != 64)) return GLA_ERR_UNSUPPORTED;
    DeviceInfo di;
    int rc = current_device_info(&di);
    if (rc != GLA_OK) return rc;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    auto launch = [&](auto kern, int threads, size_t smem) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess) {
            cudaGetLastError();
            return (int)GLA_ERR_CUDA;
        }
        kern<<<1, threads, smem, st>>>(kind, A, B, Dm);
        return cudaGetLastError() == cudaSuccess ? (int)GLA_OK : (int)GLA_ERR_CUDA;
    };
    if (d == 64) return launch(ck::gla_chunk_selftest_kernel<64>, ck::Cfg<64>::kThreads, ck::smem_bytes<64>());
    return launch(ck::gla_chunk_selftest_kernel<128>, ck::Cfg<128>::kThreads, ck::smem_bytes<128>());
}

int gla_gate_proj(const void *x, const void *w1, const void *w2, const float *bias, void *a,
                  int tokens, int d_model, int rank, int n_out, void *stream) {
    if (!x || !w1 || !w2 || !bias || !a) return GLA_ERR_NULL;
    if (tokens <= 0 || d_model <= 0 || n_out <= 0) return GLA_ERR_SHAPE;
    if ((long long)tokens * std::max(d_model, n_out) > (1LL << 40)) return GLA_ERR_SHAPE;
    if (rank != gla::gp::kRank || d_model % 64 != 0 || d_model > gla::gp::kMaxD ||
        n_out % (int)gla::gp::kChunkN != 0 || n_out > gla::gp::kMaxN)
        return GLA_ERR_UNSUPPORTED;
    const void *const ptrs[5] = {x, w1, w2, bias, a};
    for (const void *ptr : ptrs)
        if (reinterpret_cast<uintptr_t>(ptr) & 15u) return GLA_ERR_UNSUPPORTED;
    const uintptr_t ab = reinterpret_cast<uintptr_t>(a), ae = ab + (size_t)tokens * n_out * 2;
    const size_t sizes[4] = {(size_t)tokens * d_model * 2, (size_t)d_model * rank * 2, (size_t)rank * n_out * 2,
                             (size_t)n_out * 4};
    for (int i = 0; i < 4; ++i) {
        const uintptr_t pb = reinterpret_cast<uintptr_t>(ptrs[i]), pe = pb + sizes[i];
        if (pb < ae && ab < pe) return GLA_ERR_ALIAS;
    }
    DeviceInfo di;
    int rc = current_device_info(&di);
    if (rc != GLA_OK) return rc;
    EncodeTiledFn fn = encode_fn();
    if (!fn) return GLA_ERR_CUDA;
    // x [tokens][d_model] and a [tokens][n_out] as 3-D maps {width, 1, tokens}, boxes of 64
    // channels x 128 tokens, 128-byte swizzle (the MMA operand / staging layout)
    CUtensorMap xmap, amap;
    const cuuint32_t box[3] = {64, 1, (cuuint32_t)gla::gp::kTileM};
    const cuuint32_t estr[3] = {1, 1, 1};
    const struct { CUtensorMap *map; void *base; int width; } maps[2] = {
        {&xmap, const_cast<void *>(x), d_model}, {&amap, a, n_out}};
    for (const auto &mp : maps) {
        const cuuint64_t dims[3] = {(cuuint64_t)mp.width, 1, (cuuint64_t)tokens};
        const cuuint64_t strides[2] = {(cuuint64_t)mp.width * 2, (cuuint64_t)mp.width * 2};
        if (fn(mp.map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, mp.base, dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return GLA_ERR_CUDA;
    }
    const gla::gp::GateLayout lay = gla::gp::gate_layout(d_model, n_out, (size_t)di.max_smem_optin);
    if (lay.stages < 3) return GLA_ERR_UNSUPPORTED;
    const size_t smem = lay.bytes;
    if (cudaFuncSetAttribute(gla::gp::gla_gate_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess) {
        cudaGetLastError();
        return GLA_ERR_CUDA;
    }
    gla::gp::GateParams p;
    p.w1 = static_cast<const __half *>(w1);
    p.w2 = static_cast<const __half *>(w2);
    p.b = bias;
    p.T = tokens;
    p.d = d_model;
    p.n = n_out;
    p.lay = lay;
    p.wait_limit = 1LL << 32;
    // one CTA per SM, each taking an equal contiguous range of the (tile, output chunk) units
    const long long units = (long long)((tokens + gla::gp::kTileM - 1) / gla::gp::kTileM) *
                            (n_out / (int)gla::gp::kChunkN);
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)std::min<long long>(units, di.sms), 1, 1);
    cfg.blockDim = dim3(gla::gp::kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, gla::gp::gla_gate_kernel, xmap, amap, p) != cudaSuccess) {
        cudaGetLastError();
        return GLA_ERR_CUDA;
    }
    return GLA_OK;
}

int gla_linear(const void *x, const void *w, const float *bias, void *y, int rows, int k_dim, int n_dim,
               int n_part, void *stream) {
    if (!x || !w || !y) return GLA_ERR_NULL;
    if (rows <= 0 || k_dim <= 0 || n_dim <= 0 || n_part <= 0) return GLA_ERR_SHAPE;
    if ((long long)rows * std::max(k_dim, n_dim) > (1LL << 40)) return GLA_ERR_SHAPE;
    if (k_dim % gla::ln::kBK != 0 || n_part % 64 != 0 || n_dim % n_part != 0) return GLA_ERR_UNSUPPORTED;
    const int nt = n_dim % 256 == 0 ? 256 : n_dim % 192 == 0 ? 192 : n_dim % 128 == 0 ? 128 : 0;
    if (nt == 0) return GLA_ERR_UNSUPPORTED;
    const void *const ptrs[4] = {x, w, y, bias};
    for (const void *ptr : ptrs)
        if (reinterpret_cast<uintptr_t>(ptr) & 15u) return GLA_ERR_UNSUPPORTED;
    const uintptr_t yb = reinterpret_cast<uintptr_t>(y), ye = yb + (size_t)rows * n_dim * 2;
    const struct { const void *p; size_t n; } ins[3] = {
        {x, (size_t)rows * k_dim * 2}, {w, (size_t)k_dim * n_dim * 2}, {bias, bias ? (size_t)n_dim * 4 : 0}};
    for (const auto &in : ins) {
        const uintptr_t pb = reinterpret_cast<uintptr_t>(in.p), pe = pb + in.n;
        if (in.n && pb < ye && yb < pe) return GLA_ERR_ALIAS;
    }
    DeviceInfo di;
    int rc = current_device_info(&di);
    if (rc != GLA_OK) return rc;
    EncodeTiledFn fn = encode_fn();
    if (!fn) return GLA_ERR_CUDA;
    // x {K, 1, M} in boxes of 64 x 128 rows; W {N, 1, K} in boxes of 64 columns x 64 K rows;
    // y {n_part, M, parts} in boxes of 64 columns x 128 rows; all 128-byte swizzled
    CUtensorMap xmap, wmap, ymap;
    const struct {
        CUtensorMap *map; void *base; cuuint64_t d0, d1, d2, s1, s2; cuuint32_t b0, b1, b2;
    } maps[3] = {
        {&xmap, const_cast<void *>(x), (cuuint64_t)k_dim, 1, (cuuint64_t)rows, (cuuint64_t)k_dim * 2,
         (cuuint64_t)k_dim * 2, 64, 1, (cuuint32_t)gla::ln::kTileM},
        {&wmap, const_cast<void *>(w), (cuuint64_t)n_dim, 1, (cuuint64_t)k_dim, (cuuint64_t)n_dim * 2,
         (cuuint64_t)n_dim * 2, 64, 1, (cuuint32_t)gla::ln::kBK},
        {&ymap, y, (cuuint64_t)n_part, (cuuint64_t)rows, (cuuint64_t)(n_dim / n_part), (cuuint64_t)n_part * 2,
         (cuuint64_t)rows * n_part * 2, 64, (cuuint32_t)gla::ln::kTileM, 1}};
    const cuuint32_t estr[3] = {1, 1, 1};
    for (const auto &mp : maps) {
        const cuuint64_t dims[3] = {mp.d0, mp.d1, mp.d2};
        const cuuint64_t strides[2] = {mp.s1, mp.s2};
        const cuuint32_t box[3] = {mp.b0, mp.b1, mp.b2};
        if (fn(mp.map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, mp.base, dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return GLA_ERR_CUDA;
    }
    const gla::ln::LinLayout lay = gla::ln::lin_layout(nt, (size_t)di.max_smem_optin);
    if (lay.stages < 2) return GLA_ERR_UNSUPPORTED;
    if (cudaFuncSetAttribute(gla::ln::gla_linear_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)lay.bytes) != cudaSuccess) {
        cudaGetLastError();
        return GLA_ERR_CUDA;
    }
    gla::ln::LinParams p;
    p.bias = bias;
    p.M = rows;
    p.K = k_dim;
    p.N = n_dim;
    p.n_part = n_part;
    p.nt = nt;
    p.lay = lay;
    p.wait_limit = 1LL << 32;
    const long long tiles = (long long)((rows + gla::ln::kTileM - 1) / gla::ln::kTileM) * (n_dim / nt);
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)std::min<long long>(tiles, di.sms), 1, 1);
    cfg.blockDim = dim3(gla::ln::kThreads, 1, 1);
    cfg.dynamicSmemBytes = lay.bytes;
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, gla::ln::gla_linear_kernel, xmap, wmap, ymap, p) != cudaSuccess) {
        cudaGetLastError();
        return GLA_ERR_CUDA;
    }
    return GLA_OK;
}

int gla_sswiglu(const void *value, const void *gate, const float *conv_w, const float *conv_b, void *out,
                int batch, int grid_h, int grid_w, int channels, void *stream) {
    if (!value || !gate || !conv_w || !conv_b || !out) return GLA_ERR_NULL;
    if (batch <= 0 || grid_h <= 0 || grid_w <= 0 || channels <= 0) return GLA_ERR_SHAPE;
    const long long tokens = (long long)batch * grid_h * grid_w;
    if (tokens * channels > (1LL << 40) || grid_h > (1 << 24) || grid_w > (1 << 24)) return GLA_ERR_SHAPE;
    if (channels % gla::sw::kSlab != 0) return GLA_ERR_UNSUPPORTED;
    const void *const io[3] = {value, gate, out};
    for (const void *ptr : io)
        if (reinterpret_cast<uintptr_t>(ptr) & 15u) return GLA_ERR_UNSUPPORTED;
    if ((reinterpret_cast<uintptr_t>(conv_w) | reinterpret_cast<uintptr_t>(conv_b)) & 3u) return GLA_ERR_UNSUPPORTED;
    const size_t act = (size_t)tokens * channels * 2;
    const uintptr_t ob = reinterpret_cast<uintptr_t>(out), oe = ob + act;
    const struct { const void *p; size_t n; } ins[4] = {
        {value, act}, {gate, act}, {conv_w, (size_t)channels * 9 * 4}, {conv_b, (size_t)channels * 4}};
    for (const auto &in : ins) {
        const uintptr_t pb = reinterpret_cast<uintptr_t>(in.p), pe = pb + in.n;
        if (pb < oe && ob < pe) return GLA_ERR_ALIAS;
    }
    DeviceInfo di;
    int rc = current_device_info(&di);
    if (rc != GLA_OK) return rc;
    EncodeTiledFn fn = encode_fn();
    if (!fn) return GLA_ERR_CUDA;
    // tile extents: the grid split into near-equal blocks of at most 16 rows / columns
    gla::sw::SwParams p;
    p.w = conv_w;
    p.b = conv_b;
    p.out = static_cast<__half *>(out);
    p.B = batch;
    p.H = grid_h;
    p.W = grid_w;
    p.C = channels;
    p.nyb = (grid_h + gla::sw::kMaxR - 1) / gla::sw::kMaxR;
    p.nxb = (grid_w + gla::sw::kMaxWt - 1) / gla::sw::kMaxWt;
    p.R = (grid_h + p.nyb - 1) / p.nyb;
    p.Wt = (grid_w + p.nxb - 1) / p.nxb;
    p.nslab = channels / gla::sw::kSlab;
    p.tiles = (long long)batch * p.nyb * p.nxb * p.nslab;
    p.wait_limit = 1LL << 32;
    // value and gate as {C, W, H, B}: boxes of 64 channels x (Wt + 2) columns x (R + 2) rows (the
    // value, with its halo) and 64 x Wt x R (the gate) of one image
    CUtensorMap vmap, gmap;
    const cuuint64_t dims[4] = {(cuuint64_t)channels, (cuuint64_t)grid_w, (cuuint64_t)grid_h, (cuuint64_t)batch};
    const cuuint64_t strides[3] = {(cuuint64_t)channels * 2, (cuuint64_t)grid_w * channels * 2,
                                   (cuuint64_t)grid_h * grid_w * channels * 2};
    const cuuint32_t vbox[4] = {(cuuint32_t)gla::sw::kSlab, (cuuint32_t)p.Wt + 2, (cuuint32_t)p.R + 2, 1};
    const cuuint32_t gbox[4] = {(cuuint32_t)gla::sw::kSlab, (cuuint32_t)p.Wt, (cuuint32_t)p.R, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    if (fn(&vmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4, const_cast<void *>(value), dims, strides, vbox, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS ||
        fn(&gmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4, const_cast<void *>(gate), dims, strides, gbox, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return GLA_ERR_CUDA;
    const size_t smem = 2 * (size_t)gla::sw::sw_buf_bytes(p.R, p.Wt) + 128;
    if (cudaFuncSetAttribute(gla::sw::gla_sswiglu_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess) {
        cudaGetLastError();
        return GLA_ERR_CUDA;
    }
    cudaLaunchConfig_t cfg{};
    // two CTAs per SM; when tiles outnumber them, a multiple of the slab count, so every CTA
    // keeps one channel slab (tiles are numbered slab fastest)
    long long grid = std::min<long long>(p.tiles, 2LL * di.sms);
    if (p.tiles > grid && p.nslab <= grid) grid -= grid % p.nslab;
    cfg.gridDim = dim3((unsigned)grid, 1, 1);
    cfg.blockDim = dim3(gla::sw::kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, gla::sw::gla_sswiglu_kernel, vmap, gmap, p) != cudaSuccess) {
        cudaGetLastError();
        return GLA_ERR_CUDA;
    }
    return GLA_OK;
}

int gla_scan_layout(int kernel, int grid_h, int grid_w, int direction, int chunk, int *spatial,
                    int *box_rows) {
    if (!spatial || !box_rows) return GLA_ERR_NULL;
    if (kernel != kPipe64) return GLA_ERR_UNSUPPORTED;
    if (grid_h <= 0 || grid_w <= 0 || (long long)grid_h * grid_w > (1LL << 30)) return GLA_ERR_SHAPE;
    if (direction < 0 || direction > 3) return GLA_ERR_UNSUPPORTED;
    if (chunk <= 0) chunk = ck::kC;
    if (chunk % 16 != 0 || chunk > ck::kC) return GLA_ERR_UNSUPPORTED;
    const int L = grid_h * grid_w;
    const int fam = direction >> 1;
    const int hb = ck::box_rows(direction, fam, grid_h, grid_w, chunk);
    const ck::Scan sc(direction, grid_h, grid_w, chunk, hb);
    for (int p = 0; p < L; ++p) spatial[p] = -1;
    for (int q = 0; q < sc.chunks; ++q) {
        int p0, n;
        sc.chunk(q, L, p0, n);
        for (int i = 0; i < n; ++i) {
            int line, lp;
            sc.place(p0, n, i, line, lp);
            const int pos = p0 + sc.row_of(i, n);
            if (pos < 0 || pos >= L || spatial[pos] != -1) return GLA_ERR_SHAPE;
            spatial[pos] = fam ? lp * grid_w + line : line * grid_w + lp;
        }
    }
    *box_rows = hb > 0 ? hb : 64;
    return GLA_OK;
}

int gla_selftest_load(const void *q, const void *k, const void *gate_preact, const void *v,
                      const void *out_gate_preact, int B, int H, int grid_h, int grid_w, int d,
                      int direction, int chunk, float *out, int *info, void *stream) {
    if (!q || !k || !gate_preact || !v || !out_gate_preact || !out || !info) return GLA_ERR_NULL;
    if ((d != 64 && d != 128) || direction < 0 || direction > 3) return GLA_ERR_UNSUPPORTED;
    if (B <= 0 || H <= 0 || grid_h <= 0 || grid_w <= 0) return GLA_ERR_SHAPE;
    const ck::Lines ln(direction, grid_h, grid_w, ck::kC);
    if (chunk < 0 || chunk >= ln.chunks) return GLA_ERR_UNSUPPORTED;
    const void *const src[5] = {q, k, gate_preact, v, out_gate_preact};
    for (const void *ptr : src)
        if (reinterpret_cast<uintptr_t>(ptr) & 15u) return GLA_ERR_UNSUPPORTED;
    DeviceInfo di;
    int rc = current_device_info(&di);
    if (rc != GLA_OK) return rc;
    ck::Maps maps;
    const int rows[2] = {64, 64};
    if (!make_maps(&maps, src, direction, B, H, grid_h, grid_w, d, rows)) return GLA_ERR_CUDA;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    auto launch = [&](auto kern, size_t tile) {
        const size_t smem = 5 * tile + 64 + 1024;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess) {
            cudaGetLastError();
            return (int)GLA_ERR_CUDA;
        }
        kern<<<1, 32, smem, st>>>(maps, grid_h, grid_w, H, direction, ck::kC, chunk, out, info);
        return cudaGetLastError() == cudaSuccess ? (int)GLA_OK : (int)GLA_ERR_CUDA;
    };
    if (d == 64) return launch(ck::gla_chunk_load_selftest_kernel<64>, ck::Cfg<64>::kTile);
    return launch(ck::gla_chunk_load_selftest_kernel<128>, ck::Cfg<128>::kTile);
}

int gla_selftest_fault(const void *q, const void *k, const void *v, const void *gate_preact,
                       const void *out_gate_preact, const float *rms_weight, void *out, int B, int H,
                       int grid_h, int grid_w, int d, int direction, int segments,
                       long long wait_limit_cycles, int withheld_chunk, int kernel, void *stream) {
    if (wait_limit_cycles <= 0 || wait_limit_cycles > (1LL << 34)) return GLA_ERR_UNSUPPORTED;
    if (d != 64 && d != 128) return GLA_ERR_UNSUPPORTED;
    if (kernel != kTc128 && kernel != kTc64 && kernel != kPipe64) return GLA_ERR_UNSUPPORTED;
    if ((kernel == kTc128 || kernel == kPipe64) && d != 64) return GLA_ERR_UNSUPPORTED;
    const Args x = make_args(q, k, v, gate_preact, out_gate_preact, rms_weight, out, B, H, grid_h, grid_w,
                             d, d, direction, 2);
    int rc = validate(x);
    if (rc != GLA_OK) return rc;
    if (segments < 0 || segments > 16) return GLA_ERR_UNSUPPORTED;
    DeviceInfo di;
    rc = current_device_info(&di);
    if (rc != GLA_OK) return rc;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (kernel == kTc128) {
        if (segments > 0 && !tc_segs_ok(segments)) return GLA_ERR_UNSUPPORTED;
        return run_tc(x, 0, segments, kEps, st, di, nullptr, wait_limit_cycles, withheld_chunk);
    }
    if (kernel == kPipe64)
        return run_chunk<64, true>(x, 0, segments, kEps, st, di, nullptr, wait_limit_cycles, withheld_chunk);
    if (d == 64) return run_chunk<64>(x, 0, segments, kEps, st, di, nullptr, wait_limit_cycles, withheld_chunk);
    return run_chunk<128>(x, 0, segments, kEps, st, di, nullptr, wait_limit_cycles, withheld_chunk);
}

int gla_selftest_rcp(const float *x, float *y, int n, void *stream) {
    if (!x || !y) return GLA_ERR_NULL;
    if (n <= 0) return GLA_ERR_SHAPE;
    DeviceInfo di;
    int rc = current_device_info(&di);
    if (rc != GLA_OK) return rc;
    tc::gla_rcp_selftest_kernel<<<(n + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y, n);
    return cudaGetLastError() == cudaSuccess ? GLA_OK : GLA_ERR_CUDA;
}

int gla_selftest_mma(int kind, const float *A, const float *B, float *D, void *stream) {
    if (!A || !B || !D) return GLA_ERR_NULL;
    if (kind < 0 || kind > 3) return GLA_ERR_UNSUPPORTED;
    DeviceInfo di;
    int rc = current_device_info(&di);
    if (rc != GLA_OK) return rc;
    auto kern = tc::gla_tc_selftest_kernel;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tc::kSmemBytes) !=
        cudaSuccess) {
        cudaGetLastError();
        return GLA_ERR_CUDA;
    }
    kern<<<1, tc::kSelfThreads, tc::kSmemBytes, static_cast<cudaStream_t>(stream)>>>(kind, A, B, D);
    if (cudaGetLastError() != cudaSuccess) return GLA_ERR_CUDA;
    return GLA_OK;
}

}  // extern "C"
