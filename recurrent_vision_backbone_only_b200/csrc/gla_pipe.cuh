// gla_pipe.cuh -- the 64-row tensor-core kernel of gla_chunk.cuh for d_k = d_v = 64 with two
// chunks in flight: warp-specialised teams and a 3-stage TMA ring.
//
// Operation and chunkwise form: as gla_chunk.cuh (GTR paper, arXiv 2609.26590, method
// section: S_t = Diag(gamma_t) S_{t-1} + k_t^T v_t, o_t = d_k^{-1/2} q_t S_t, u_t = SiLU(g_t) *
// RMSNorm(o_t) * w), with the same 16-bit products and cluster state exchange.  The schedule and
// the chunking differ.
//
// Packed chunks.  Chunk q holds the scan positions [q cl, q cl + cl) whatever lines they
// cross, so every tile row carries a token (a 40-position line no longer leaves 24 of 64 rows
// empty).  When hb -- the largest power of two <= 64 dividing both the line length and cl -- is
// at least 8, every aligned group of hb positions lies in one line and its tokens are equally
// spaced in memory, so a tile is 64 / hb TMA boxes of hb rows.  Each box is loaded in increasing
// spatial order; in R->L and B->T the scan runs against it, so scan offset i sits in tile row
// i ^ (hb - 1).  Other line lengths keep line-aligned chunks (one 64-row box, scan offset i in
// row n - 1 - i when reversed).
//
// Fused product.  The carried state is kept transposed, S^T[j][c] (S_loc^T = V^T Ks), so
// S~^T = S^T Diag(2^r) is a K-major operand like K~, and each stage places S~^T right after K~:
// [K~ | S~^T] is one 128-row operand, and Q~ [K~ | S~^T]^T yields the scores (columns 0-63) and
// the inter-chunk term Q~ S~ (columns 64-127, the output accumulator) in the same tcgen05.mma
// (N = 128): per chunk 4 state, 12 fused and 4 P V products.
//
// Roles (576 threads):
//   front team  (warps 0-7)   per chunk: gate (cumulative log2-decay b), then the operands Kh,
//                             Kl, Ks in place over the raw tiles and Q~ into the chunk's TMEM slot;
//   back team   (warps 8-15)  per chunk: P from the scores (into the dead K~-low tile, as the A
//                             operand of P V), the state fold, the NEXT chunk's S~^T (so its
//                             fused product runs under this chunk's epilogue), the RMSNorm /
//                             SiLU epilogue and the stores;
//   MMA warp    (warp 16)     issues every tcgen05.mma and commit;
//   load warp   (warp 17)     issues the TMA boxes into a 3-stage ring.
// Chunk j uses TMEM slot j % 2 -- lanes 16 (j % 2) .. + 16 of every lane quarter, so one M = 64
// tile of each slot shares the columns of the other -- and smem stage j % 3.  The front team
// builds chunk j + 1 while the tensor core and the back team finish chunk j.
//
// Synchronisation (mbarriers, phase = use count of the slot / stage).  Every chunk completes
// every slot barrier exactly once (a state-only chunk with no-op arrivals and commits), and every
// waiter of a barrier waits on each of its phases in turn, so the k-th use of a slot always waits
// for parity k & 1 and no waiter is ever two phases behind:
//   ld[s]        TMA bytes of a stage landed                       load warp -> front
//   gdone[p]     gate scalars (r) of the slot's chunk ready        front -> back (S~^T)
//   fdone[p]     gate + operands of the slot's chunk ready         front -> MMA, back
//   sl, sc, o[p] chunk state / fused / output products done       tcgen05.commit -> back
//   sx[p]        S~^T of the slot's chunk written                  back -> MMA
//   pfull[p]     P written                                         back -> MMA
//   slotfree[p]  the back team is done with the slot's chunk       back -> front, MMA
//   stfree[s]    the stage may be reloaded (2 arrivals)            tcgen05.commit + back -> load
#pragma once

#include "gla_chunk.cuh"

namespace gla {
namespace ck {

struct PipeCfg {
    static constexpr int D = 64;
    static constexpr int kTeam = 256;                    // threads per team
    static constexpr int kThreads = 2 * kTeam + 64;      // + MMA warp + load warp
    static constexpr int kStages = 3;
    static constexpr uint32_t kAtom = 64 * 128;
    static constexpr uint32_t kTile = 64 * D * 2;        // 8 KB
    // a stage: q (-> Ks), k (-> K~ high), S~^T high, a (-> K~ low -> P), S~^T low, v, g.  K~ and
    // S~^T of one part are adjacent, so [K~ | S~^T] is ONE K-major operand of 128 rows.
    static constexpr uint32_t kTQ = 0, kTK = kTile, kTSH = 2 * kTile, kTA = 3 * kTile, kTSL = 4 * kTile;
    static constexpr uint32_t kTV = 5 * kTile, kTG = 6 * kTile;
    static constexpr uint32_t kStage = 7 * kTile;
    static constexpr uint32_t kB = kStages * kStage;     // b (front team) / exchange rows
    static constexpr uint32_t kBBytes = 20480;           // >= max(64 x 64 x 4, (D + 15) x D x 4)
    static constexpr uint32_t kMisc = kB + kBBytes;
    // TMEM columns; slot p is lanes 16p .. 16p + 15 of every quarter
    static constexpr uint32_t kColSC = 0, kColO = 64, kColQH = 128, kColQL = 160, kColSL = 192;
    static constexpr uint32_t kTmemCols = 256;
    static constexpr int kMaxRecvRows = D + 15;
};

struct PipeMisc {
    uint64_t ld[3], stfree[3];
    uint64_t gdone[2], fdone[2], sl[2], sc[2], sx[2], pfull[2], o[2], slotfree[2];
    uint64_t end;              // teardown after an expired wait: products in flight
    uint32_t tmem_base;
    int abort, range_err;
    int slow[2];               // per slot: the chunk takes the exact CUDA-core score path
    alignas(16) float tot[8][64];     // front: gate block totals
    alignas(16) float b0[64];         // front: b at the first scan position
    alignas(16) float rref[2][64];    // per slot: reference r (log2)
    alignas(16) float rq[2][64];      // per slot: r - log2(d_k^{-1/2}) (the query side's reference)
    alignas(16) float Bc[2][64];      // per slot: B (log2)
    alignas(16) float fB[2][64];      // per slot: 2^{B - r}
    alignas(16) float er[2][64];      // per slot: 2^{r}
    alignas(16) float eB[2][64];      // per slot: 2^{B}
    alignas(16) float dqp[2][4][kC];  // per slot: diagonal score partial sums
    alignas(16) float red[4][kC];     // back: epilogue partial sums of squares
    alignas(16) float Gs[64];         // back: segment aggregate log2-decay
    alignas(16) float w[64];          // RMSNorm weight
    alignas(16) float recvG[PipeCfg::kMaxRecvRows];
};

constexpr size_t pipe_smem_bytes() { return PipeCfg::kMisc + sizeof(PipeMisc) + 1024; }

// Rows per TMA box of a packed chunk for lines of length `len` and chunks of `cl` positions:
// the largest power of two <= 64 dividing both, or 0 (line-aligned chunks) when below 8.
__host__ __device__ inline int pack_rows(int len, int cl) {
    int hb = 64;
    while (hb >= 8 && (len % hb != 0 || cl % hb != 0)) hb >>= 1;
    return hb >= 8 ? hb : 0;
}

// Rows per TMA box for line family `fam` of a launch in direction `dir` (4: cycling).  A
// forward row scan alone (dir 0) visits the token rows in memory order, so a chunk of cl
// positions is consecutive rows whatever lines it spans and needs no line-bounded groups: boxes
// of the largest power of two dividing cl.  Otherwise packed groups within a line (pack_rows).
__host__ __device__ inline int box_rows(int dir, int fam, int gh, int gw, int cl) {
    if (fam == 0 && dir == 0) {
        int hb = 64;
        while (cl % hb != 0) hb >>= 1;
        return hb;
    }
    return pack_rows(fam ? gh : gw, cl);
}

// Chunks of one (b, h) scan.  Packed (hb > 0): chunk q is the scan positions [q cl, q cl + cl);
// line-aligned (hb = 0): every line is cut into `pieces` equal pieces of at most cl positions.
struct Scan {
    int fam;      // 0: lines are grid rows (L->R, R->L), 1: grid columns (T->B, B->T)
    int rev;      // the scan runs against the spatial order within a line (R->L, B->T)
    int len;      // line length
    int hb;       // rows per box of a packed chunk, 0: line-aligned chunks
    bool contig;  // packed forward row scan (L->R): a chunk is consecutive token rows whatever
                  // lines it spans, so its boxes need not stop at a line's end
    int cl;       // chunk length (the last chunk may be shorter)
    int pieces;   // line-aligned: chunks per line
    int chunks;   // chunks per scan
    __host__ __device__ Scan(int dir, int gh, int gw, int chunk_max, int hb_) {
        fam = dir >> 1;
        rev = dir & 1;
        len = fam ? gh : gw;
        hb = hb_;
        contig = hb > 0 && fam == 0 && rev == 0;
        if (hb > 0) {
            cl = chunk_max;
            pieces = 0;
            chunks = (gh * gw + cl - 1) / cl;
        } else {
            pieces = (len + chunk_max - 1) / chunk_max;
            cl = (len + pieces - 1) / pieces;
            chunks = (fam ? gw : gh) * pieces;
        }
    }
    // first scan position and length of chunk q of a scan of L positions
    __host__ __device__ void chunk(int q, int L, int &p0, int &n) const {
        if (hb > 0) {
            p0 = q * cl;
            n = min(cl, L - p0);
        } else {
            const int line = q / pieces, start = (q - line * pieces) * cl;
            p0 = line * len + start;
            n = min(cl, len - start);
        }
    }
    // tile row of scan offset i in a chunk of n positions (an involution: also the offset of row i)
    __host__ __device__ int row_of(int i, int n) const { return rev ? (hb > 0 ? i ^ (hb - 1) : n - 1 - i) : i; }
    // Bit e of the result: the token of tile row s0 + e (s0 a multiple of 16, e < 16) precedes
    // the token of row t in the scan, both rows inside the chunk of n positions.
    __device__ uint32_t before_mask(int n, int t, int s0) const {
        auto span = [](int lo, int hi) -> uint32_t {       // bits lo .. hi - 1, clamped to 0..16
            lo = max(lo, 0);
            hi = min(hi, 16);
            return hi > lo ? ((1u << hi) - 1u) & ~((1u << lo) - 1u) : 0u;
        };
        if (t >= n) return 0u;
        if (rev && hb == 0) return span(t - s0 + 1, n - s0);   // line-aligned, reversed: t < s < n
        // scan offset of row s0 + e is (s0 + e) ^ xm = (s0 ^ (xm & ~15)) + (e ^ x); for rows inside
        // the chunk a smaller offset implies s < n
        const int xm = rev ? hb - 1 : 0, x = xm & 15;
        uint32_t mk = span(0, (t ^ xm) - (s0 ^ (xm & ~15)));   // bits v with v < that bound
        if (x & 1) mk = ((mk & 0x5555u) << 1) | ((mk >> 1) & 0x5555u);    // bit e <- bit e ^ x
        if (x & 2) mk = ((mk & 0x3333u) << 2) | ((mk >> 2) & 0x3333u);
        if (x & 4) mk = ((mk & 0x0F0Fu) << 4) | ((mk >> 4) & 0x0F0Fu);
        if (x & 8) mk = ((mk & 0x00FFu) << 8) | ((mk >> 8) & 0x00FFu);
        return mk;
    }
    // line and position along it of tile row i of the chunk starting at scan position p0
    __host__ __device__ void place(int p0, int n, int i, int &line, int &lp) const {
        if (hb > 0) {
            const int pg = p0 + (i & ~(hb - 1));
            line = pg / len;
            const int o = pg - line * len;
            lp = (rev ? len - o - hb : o) + (i & (hb - 1));
        } else {
            line = p0 / len;
            const int st = p0 - line * len;
            lp = (rev ? len - st - n : st) + i;
        }
    }
};

__device__ __forceinline__ void team_bar(int id) { ptx::named_bar_sync(id, PipeCfg::kTeam); }

__global__ void __launch_bounds__(PipeCfg::kThreads, 1)
    gla_pipe_kernel(const __grid_constant__ Maps maps, const Params p) {
    using C = PipeCfg;
    constexpr int D = 64;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
    const uint32_t sbase = ptx::smem_u32(sm);
    PipeMisc &m = *reinterpret_cast<PipeMisc *>(sm + C::kMisc);
    volatile int *abort_flag = &m.abort;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool front = warp < 8, back = warp >= 8 && warp < 16;
    const bool mma_warp = warp == 16, load_warp = warp == 17;
    // team roles (front and back alike): row t, channels [16 cg, 16 cg + 16); back: state row sc,
    // columns [16 cg, + 16)
    const int wt = warp & 7, qd = warp & 3, hg = wt >> 2, cg = 2 * hg + (lane >> 4);
    const int t = 16 * qd + (lane & 15);
    const int ttid = tid & (C::kTeam - 1);           // thread index within its team

    const int rank = blockIdx.x % p.segs;
    const int pair = p.pair0 + blockIdx.x / p.segs;
    const int bb = pair / p.H, hh = pair - bb * p.H;
    const int dir = p.dir == 4 ? (bb & 3) : p.dir;
    const Scan ln(dir, p.gh, p.gw, p.chunk_max, p.hb[dir >> 1]);
    const int seg_chunks = (ln.chunks + p.segs - 1) / p.segs;
    const int q0 = min(ln.chunks, rank * seg_chunks);
    const int n2 = min(ln.chunks, q0 + seg_chunks) - q0;
    const bool exchange = p.segs > 1;
    const int n1 = (exchange && rank < p.segs - 1) ? n2 : 0;
    const int N = n1 + n2;                             // chunks processed: state-only, then full
    const CUtensorMap *tmaps = ln.fam ? maps.col : maps.row;

    ptx::pdl_launch_dependents();
    if (tid == 0) {
        for (int i = 0; i < 3; ++i) {
            ptx::mbar_init(&m.ld[i], 1);
            ptx::mbar_init(&m.stfree[i], 2);
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(&m.gdone[i], 1);
            ptx::mbar_init(&m.fdone[i], 1);
            ptx::mbar_init(&m.sl[i], 1);
            ptx::mbar_init(&m.sc[i], 1);
            ptx::mbar_init(&m.sx[i], 1);
            ptx::mbar_init(&m.pfull[i], 1);
            ptx::mbar_init(&m.o[i], 1);
            ptx::mbar_init(&m.slotfree[i], 1);
        }
        ptx::mbar_init(&m.end, 1);
        ptx::fence_mbarrier_init();
        m.abort = 0;
        m.range_err = 0;
    }
    if (warp == 0) {
        ptx::tmem_alloc(&m.tmem_base, C::kTmemCols);
        ptx::tmem_relinquish();
    }
    if (load_warp && lane == 0)
        for (int i = 0; i < 5; ++i) ptx::prefetch_tmap(&tmaps[i]);
    if (tid < D) m.Gs[tid] = 0.0f;
    ptx::tc_fence_before_sync();
    __syncthreads();
    ptx::tc_fence_after_sync();
    const uint32_t tmem = m.tmem_base;
    ptx::pdl_wait_prior_grid();
    if (tid < D / 4)
        *reinterpret_cast<float4 *>(&m.w[4 * tid]) = *reinterpret_cast<const float4 *>(p.w + 4 * tid);
    __syncthreads();

    // chunk j of the sequence (state-only chunks, then full chunks) -> chunk of the segment
    struct Chunk {
        int p0, n;          // first scan position, positions
        bool full;
    };
    auto chunk_of = [&](int j) {
        const bool full = j >= n1;
        Chunk c;
        ln.chunk(q0 + (full ? j - n1 : j), p.L, c.p0, c.n);
        if (!GLA_CHECK(c.n >= 1 && c.n <= 64 && c.p0 >= 0 && c.p0 + c.n <= p.L)) c.n = 1;
        c.full = full;
        return c;
    };
    auto token_row = [&](const Chunk &c, int i) {
        int line, lp;
        ln.place(c.p0, c.n, i, line, lp);
        const int s = ln.fam ? lp * p.gw + line : line * p.gw + lp;
        return (bb * p.L + s) * p.H + hh;
    };
    auto wait = [&](uint64_t *bar, int use) { return wait_bar(bar, (uint32_t)(use & 1), p.wait_limit, abort_flag); };
    // lanes of this warp's quarter in TMEM slot `slot`
    auto tmem_rows = [&](int slot) { return tmem + ((uint32_t)(32 * qd + 16 * slot) << 16); };

    // ---------------------------------------------------------------- exchange
    // All 576 threads: barriers A, B, C; the back team holds the aggregate (S^T, Gs).  The state
    // is kept transposed, S^T[j][c] (row j = value column, column c = key channel), so it is the
    // K-major half of the fused operand; the exchange moves rows of S = S^T transposed, staged
    // through fp32 rows [c][j] in stage 0's S~ tiles (free until the first full chunk).
    float S[16];                                      // back: S^T[j = sc][c = 16 cg + i]
#pragma unroll
    for (int i = 0; i < 16; ++i) S[i] = 0.0f;
    const int sc = 16 * qd + (lane & 15);
    auto srow = [&](int c) -> uint32_t {              // fp32 row c of the [c][j] staging, stage 0
        return (c < 32 ? C::kTSH : C::kTSL) + (uint32_t)(c & 31) * (D * 4);
    };
    auto run_exchange = [&]() {
        const int segs = p.segs;
        const int max_own = (D + segs - 1) / segs;
        const float *recv = reinterpret_cast<const float *>(sm + C::kB);
        if (back) {
#pragma unroll
            for (int i = 0; i < 16; ++i) *reinterpret_cast<float *>(sm + srow(16 * cg + i) + 4 * sc) = S[i];
        }
        __syncthreads();
        ptx::cluster_arrive_release();
        ptx::cluster_wait();
        if (back && rank < segs - 1) {                // row c = sc of S, columns [16 cg, + 16)
            const int owner = sc % segs, lc = sc / segs;
            const uint32_t row = (uint32_t)((rank * max_own + lc) * D + 16 * cg) * 4;
            if (GLA_CHECK(rank * max_own + lc < C::kMaxRecvRows && (rank + 1) * max_own <= C::kMaxRecvRows &&
                          (uint32_t)(C::kMaxRecvRows * D * 4) <= C::kBBytes))
#pragma unroll
            for (int i = 0; i < 4; ++i)
                ptx::st_cluster_v4(ptx::mapa(sbase + C::kB + row + 16 * i, owner),
                                   *reinterpret_cast<const float4 *>(sm + srow(sc) + 64 * cg + 16 * i));
        }
        if (tid < D && rank < segs - 1 && GLA_CHECK(rank * max_own + tid / segs < C::kMaxRecvRows)) {
            const int o2 = tid % segs, l2 = tid / segs;
            ptx::st_cluster_f32(ptx::mapa(ptx::smem_u32(&m.recvG[rank * max_own + l2]), o2), m.Gs[tid]);
        }
        ptx::cluster_arrive_release();
        ptx::cluster_wait();
        {
            const int n_own = (D - rank + segs - 1) / segs;
            const int items = n_own * (D / 4);
            for (int it = tid; it < items; it += C::kThreads) {
                const int lc = it / (D / 4), j4 = it - lc * (D / 4);
                const int c = lc * segs + rank;
                if (!GLA_CHECK(c < D && (segs - 1) * max_own + lc < C::kMaxRecvRows)) continue;
                const uint32_t dst = sbase + srow(c) + 16 * j4;
                float4 run = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                for (int q = 0; q < segs; ++q) {
                    ptx::st_cluster_v4(ptx::mapa(dst, q), run);
                    if (q + 1 < segs) {
                        const float g = ptx::ex2(m.recvG[q * max_own + lc]);
                        const float4 agg = *reinterpret_cast<const float4 *>(recv + (q * max_own + lc) * D + 4 * j4);
                        run = make_float4(fmaf(g, run.x, agg.x), fmaf(g, run.y, agg.y),
                                          fmaf(g, run.z, agg.z), fmaf(g, run.w, agg.w));
                    }
                }
            }
        }
        ptx::cluster_arrive_release();
        ptx::cluster_wait();
        if (back) {
#pragma unroll
            for (int i = 0; i < 16; ++i) S[i] = *reinterpret_cast<const float *>(sm + srow(16 * cg + i) + 4 * sc);
        }
        __syncthreads();
    };

    // =================================================================== load warp
    if (load_warp) {
        int last[3] = {-1, -1, -1};                   // last chunk issued into each stage
        auto load = [&](int j) {
            const int s = j % 3;
            if (j >= 3) wait(&m.stfree[s], (j - 3) / 3);
            // lane 0 decides (the abort flag may change under the warp) and sets the byte count;
            // the lanes then issue the boxes
            const bool go = __shfl_sync(0xffffffffu, lane == 0 ? (int)!*abort_flag : 0, 0) != 0;
            if (go) {
                const Chunk c = chunk_of(j);
                const uint32_t mask = c.full ? 0x1Fu : 0x0Eu;
                if (lane == 0) ptx::mbar_arrive_expect_tx(&m.ld[s], (uint32_t)__popc(mask) * C::kTile);
                __syncwarp();
                if (!(c.full && j - n1 == p.fault_chunk)) {
                    // one box per group of hb rows (packed) or one 64-row box.  A group past the
                    // chunk's end reloads the first group's tokens: rows that are masked later
                    // still hold finite values, and no box leaves the tensor.
                    const int rows = ln.hb > 0 ? ln.hb : 64;
                    const uint32_t bar = ptx::smem_u32(&m.ld[s]);
                    constexpr uint32_t kDst[5] = {C::kTQ, C::kTK, C::kTA, C::kTV, C::kTG};
                    auto box = [&](int i, int x) {        // tile x, tile rows [i, i + rows)
                        int line, lp;
                        ln.place(c.p0, c.n, i < c.n ? i : 0, line, lp);
                        const int y = ln.fam ? line * p.H + hh : hh;
                        const int z = ln.fam ? bb * p.gh + lp : bb * p.L + line * p.gw + lp;
                        // a box starts inside its view; a packed group stays inside its line
                        // (except in a forward row scan, whose positions are contiguous rows)
                        if (!GLA_CHECK(y >= 0 && y < (ln.fam ? p.gw * p.H : p.H) && z >= 0 &&
                                       z < (ln.fam ? p.B * p.gh : p.B * p.L) && lp >= 0 &&
                                       (ln.hb == 0 || ln.contig || lp + rows <= ln.len)))
                            return;
                        ptx::tma_load_3d(sbase + s * C::kStage + (uint32_t)i * 128 + kDst[x], &tmaps[x], 0, y, z, bar);
                    };
                    // one group per lane, its tiles in turn (measured at least as fast as one box
                    // per lane, and faster when a chunk has more boxes than the warp has lanes)
                    for (int i = lane * rows; i < 64; i += 32 * rows)
#pragma unroll
                        for (int x = 0; x < 5; ++x)
                            if (mask >> x & 1u) box(i, x);
                }
                last[s] = j;
            }
            __syncwarp();
        };
        const int pre = min(N, n1 + 3);             // everything loadable before the exchange
        for (int j = 0; j < pre; ++j) load(j);
        if (exchange) run_exchange();
        for (int j = pre; j < N; ++j) load(j);
        // teardown: after an expired wait, the boxes already issued land before smem is freed
        __syncthreads();
        if (*abort_flag && lane == 0) {
            volatile int no_abort = 0;
            for (int s = 0; s < 3; ++s)
                if (last[s] >= 0) wait_bar(&m.ld[s], (uint32_t)((last[s] / 3) & 1), p.wait_limit, &no_abort);
        }
    }

    // ==================================================================== MMA warp
    else if (mma_warp) {
        using M = Mma<64>;
        const uint64_t kh0 = ptx::desc_sw128(sbase + C::kTK, 16, 1024);      // [K~ high | S~^T high]
        const uint64_t kl0 = ptx::desc_sw128(sbase + C::kTA, 16, 1024);      // [K~ low | S~^T low]
        const uint64_t ks0 = ptx::desc_sw128(sbase + C::kTQ, C::kAtom, 1024);
        const uint64_t v0 = ptx::desc_sw128(sbase + C::kTV, C::kAtom, 1024);
        const uint64_t pa0 = ptx::desc_sw128(sbase + C::kTA, 16, 1024);      // P: K-major A
        constexpr uint32_t kIdPVss = ptx::idesc_ab(0, 0, false, true, 64, 64);
        constexpr uint32_t kIdFused = ptx::idesc_ab(1, 1, false, false, 64, 128);
        auto step = [&](int j) {
            const int slot = j & 1, s = j % 3;
            const Chunk c = chunk_of(j);
            const uint32_t stg = (uint32_t)s * C::kStage >> 4;               // descriptor address units
            const uint32_t lanes = (uint32_t)(16 * slot) << 16;
            if (j >= 2) wait(&m.slotfree[slot], (j - 2) >> 1);
            wait(&m.fdone[slot], j >> 1);
            if (lane == 0) {
                ptx::tc_fence_after_sync();
                if (!*abort_flag) {                   // S_loc^T = V^T Ks (both MN-major)
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        ptx::mma_f16_ss(tmem + lanes + C::kColSL, v0 + stg + 128 * k, ks0 + stg + 128 * k, M::kIdSL, k > 0);
                }
                ptx::mma_commit(&m.sl[slot]);
            }
            __syncwarp();
            wait(&m.sx[slot], j >> 1);                // S~^T of the chunk (a no-op for a state-only one)
            if (lane == 0) {
                ptx::tc_fence_after_sync();
                if (c.full && !*abort_flag) {
                    // [scores | inter] = Q~ [K~ | S~^T]^T, bf16 split: Qh Kh + Qh Kl + Ql Kh, N = 128
#pragma unroll
                    for (int pass = 0; pass < 3; ++pass)
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            ptx::mma_f16_ts(tmem + lanes + C::kColSC,
                                            tmem + lanes + (pass == 2 ? C::kColQL : C::kColQH) + 8 * k,
                                            (pass == 1 ? kl0 : kh0) + stg + 2 * k, kIdFused, pass > 0 || k > 0);
                }
                ptx::mma_commit(&m.sc[slot]);
            }
            __syncwarp();
            wait(&m.pfull[slot], j >> 1);
            if (lane == 0) {
                ptx::tc_fence_after_sync();
                if (c.full && !*abort_flag) {         // O += P V
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        ptx::mma_f16_ss(tmem + lanes + C::kColO, pa0 + stg + 2 * k, v0 + stg + 128 * k, kIdPVss, true);
                }
                ptx::mma_commit(&m.o[slot]);
                ptx::mma_commit(&m.stfree[s]);        // this chunk's products have read the stage
            }
            __syncwarp();
        };
        for (int j = 0; j < n1; ++j) step(j);
        if (exchange) run_exchange();
        for (int j = n1; j < N; ++j) step(j);
        __syncthreads();
        if (*abort_flag && lane == 0) {
            volatile int no_abort = 0;
            ptx::mma_commit(&m.end);
            wait_bar(&m.end, 0, p.wait_limit, &no_abort);
        }
    }

    // ================================================================== front team
    else if (front) {
        const uint32_t tmem_q = tmem;                 // + slot lanes below
        // gate: thread (channel pair cp, block pb of 8 scan positions), b into kB (fp32 atoms).
        // Rows past the chunk get b = +inf: their decayed keys 2^{r - b} k vanish without a
        // select, and their queries (infinite) only reach score rows and output rows that are
        // masked or never stored.  Returns whether the chunk takes the exact score path.
        auto gate = [&](uint32_t stage, const Chunk &c, int slot) {
            const int cp = ttid & 31, pb = ttid >> 5, ch = 2 * cp;
            const int n = c.n;
            float c0s[8], c1s[8];
            int rows[8];
            float r0 = 0.0f, r1 = 0.0f;
            const uint32_t aoff = stage + C::kTA + (ch & 7) * 2;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int pos = pb * 8 + i;
                const bool ok = pos < n;
                rows[i] = ok ? ln.row_of(pos, n) : pos;
                const float2 af = __half22float2(*reinterpret_cast<const __half2 *>(sm + aoff + ptx::sw128(rows[i], ch >> 3)));
                r0 += ok ? log2_gamma(af.x) : 0.0f;
                r1 += ok ? log2_gamma(af.y) : 0.0f;
                c0s[i] = r0;
                c1s[i] = r1;
            }
            *reinterpret_cast<float2 *>(&m.tot[pb][ch]) = make_float2(r0, r1);
            team_bar(1);
            float a0 = 0.0f, a1 = 0.0f;
#pragma unroll
            for (int q = 0; q < 7; ++q)
                if (q < pb) {
                    const float2 x = *reinterpret_cast<const float2 *>(&m.tot[q][ch]);
                    a0 += x.x;
                    a1 += x.y;
                }
            const int rmid = (n - 1) >> 1;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int pos = pb * 8 + i;
                const float2 bv = pos < n ? make_float2(c0s[i] + a0, c1s[i] + a1) : make_float2(INFINITY, INFINITY);
                *reinterpret_cast<float2 *>(sm + C::kB + off_f<64>(rows[i], ch >> 2) + (ch & 3) * 4) = bv;
                if (pos == rmid) *reinterpret_cast<float2 *>(&m.rref[slot][ch]) = bv;
                if (pos == n - 1) *reinterpret_cast<float2 *>(&m.Bc[slot][ch]) = bv;
                if (pos == 0) *reinterpret_cast<float2 *>(&m.b0[ch]) = bv;
            }
            team_bar(1);
            // per key channel: 2^B, the operand range check, and the fast path's 2^{B - r}, 2^r
            bool oob = false;
            if (ttid < D) {
                const float Bv = m.Bc[slot][ttid], r = m.rref[slot][ttid];
                m.eB[slot][ttid] = ptx::ex2(Bv);
                if (c.full) {
                    oob = m.b0[ttid] - r > kHalfRange || r - Bv > kHalfRange;
                    m.fB[slot][ttid] = ptx::ex2(Bv - r);
                    m.er[slot][ttid] = ptx::ex2(r);
                    m.rq[slot][ttid] = r - p.log2_scale;
                }
            }
            const bool slow = ptx::named_bar_or(1, C::kTeam, oob);
            if (slow) {                              // rare; r = 0 keeps every exponent <= 0
                if (ttid < D) {
                    m.rref[slot][ttid] = 0.0f;
                    m.er[slot][ttid] = 1.0f;
                    m.rq[slot][ttid] = -p.log2_scale;
                }
                team_bar(1);
            }
            if (ttid == 0) m.slow[slot] = slow;
            return slow;
        };
        auto build_ks = [&](uint32_t stage, int slot) {
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
                const int j = 2 * cg + jj;
                const uint32_t o = off_h<64>(t, j);
                const uint4 kraw = *reinterpret_cast<const uint4 *>(sm + stage + C::kTK + o);
                const __half2 *k2 = reinterpret_cast<const __half2 *>(&kraw);
                const float4 bA = *reinterpret_cast<const float4 *>(sm + C::kB + off_f<64>(t, 2 * j));
                const float4 bB = *reinterpret_cast<const float4 *>(sm + C::kB + off_f<64>(t, 2 * j + 1));
                const float4 BA = *reinterpret_cast<const float4 *>(&m.Bc[slot][8 * j]);
                const float4 BB = *reinterpret_cast<const float4 *>(&m.Bc[slot][8 * j + 4]);
                const float bt[8] = {bA.x, bA.y, bA.z, bA.w, bB.x, bB.y, bB.z, bB.w};
                const float Bt[8] = {BA.x, BA.y, BA.z, BA.w, BB.x, BB.y, BB.z, BB.w};
                uint32_t ks[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 kf = __half22float2(k2[e]);
                    ks[e] = pack_h2(kf.x * ptx::ex2(Bt[2 * e] - bt[2 * e]),
                                    kf.y * ptx::ex2(Bt[2 * e + 1] - bt[2 * e + 1]));
                }
                *reinterpret_cast<uint4 *>(sm + stage + C::kTQ + o) = make_uint4(ks[0], ks[1], ks[2], ks[3]);
            }
        };
        // exact scores of a chunk beyond the bf16 operands' range: row t, columns [16 cg, + 16),
        // fp16 into the a tile (the P slot)
        auto exact_p_smem = [&](uint32_t stage, const Chunk &c) {
            const int n = c.n, s0 = 16 * cg, pt = ln.row_of(t, n);
            auto hat = [&](uint32_t tile, int row, int ch) {
                return __half2float(*reinterpret_cast<const __half *>(sm + stage + tile + off_h<64>(row, ch >> 3) + (ch & 7) * 2));
            };
            auto bat = [&](int row, int ch) {
                return *reinterpret_cast<const float *>(sm + C::kB + off_f<64>(row, ch >> 2) + (ch & 3) * 4);
            };
            float pv[16];
            float amax = 0.0f;
            for (int e = 0; e < 16; ++e) {
                const int s = s0 + e;
                const bool causal = ln.row_of(s, n) <= pt;
                float acc = 0.0f;
                if (causal && t < n && s < n)
                    for (int ch = 0; ch < D; ++ch) {
                        const float f = s == t ? 1.0f : ptx::ex2(bat(t, ch) - bat(s, ch));
                        acc = fmaf(hat(C::kTQ, t, ch) * hat(C::kTK, s, ch), f, acc);
                    }
                pv[e] = acc * p.scale;
                amax = fmaxf(amax, fabsf(pv[e]));
            }
            if (amax > 65504.0f) m.range_err = 1;
            team_bar(1);                              // every thread has read the raw a / k / q it needs
#pragma unroll
            for (int h = 0; h < 2; ++h)
                *reinterpret_cast<uint4 *>(sm + stage + C::kTA + off_h<64>(t, 2 * cg + h)) =
                    make_uint4(pack_h2(pv[8 * h], pv[8 * h + 1]), pack_h2(pv[8 * h + 2], pv[8 * h + 3]),
                               pack_h2(pv[8 * h + 4], pv[8 * h + 5]), pack_h2(pv[8 * h + 6], pv[8 * h + 7]));
        };
        // fast path (decay half-range within the bf16 operands' reach): one 8-channel group per
        // iteration, the loop kept rolled so the team's hot code stays small
        auto build_full = [&](uint32_t stage, int slot) {
            float dqs = 0.0f;
            const uint32_t rows = tmem_q + ((uint32_t)(32 * qd + 16 * slot) << 16);
#pragma unroll 1
            for (int jj = 0; jj < 2; ++jj) {
                const int j = 2 * cg + jj;
                const uint32_t o = off_h<64>(t, j);
                const uint4 kraw = *reinterpret_cast<const uint4 *>(sm + stage + C::kTK + o);
                const uint4 qraw = *reinterpret_cast<const uint4 *>(sm + stage + C::kTQ + o);
                const __half2 *k2 = reinterpret_cast<const __half2 *>(&kraw);
                const __half2 *q2 = reinterpret_cast<const __half2 *>(&qraw);
                const float4 bA = *reinterpret_cast<const float4 *>(sm + C::kB + off_f<64>(t, 2 * j));
                const float4 bB = *reinterpret_cast<const float4 *>(sm + C::kB + off_f<64>(t, 2 * j + 1));
                const float4 rA = *reinterpret_cast<const float4 *>(&m.rref[slot][8 * j]);
                const float4 rB = *reinterpret_cast<const float4 *>(&m.rref[slot][8 * j + 4]);
                const float4 qA = *reinterpret_cast<const float4 *>(&m.rq[slot][8 * j]);
                const float4 qB = *reinterpret_cast<const float4 *>(&m.rq[slot][8 * j + 4]);
                const float4 fA = *reinterpret_cast<const float4 *>(&m.fB[slot][8 * j]);
                const float4 fBv = *reinterpret_cast<const float4 *>(&m.fB[slot][8 * j + 4]);
                const float bt[8] = {bA.x, bA.y, bA.z, bA.w, bB.x, bB.y, bB.z, bB.w};
                const float rr[8] = {rA.x, rA.y, rA.z, rA.w, rB.x, rB.y, rB.z, rB.w};
                const float rq[8] = {qA.x, qA.y, qA.z, qA.w, qB.x, qB.y, qB.z, qB.w};
                const float ff[8] = {fA.x, fA.y, fA.z, fA.w, fBv.x, fBv.y, fBv.z, fBv.w};
                uint32_t kh4[4], kl4[4], ks4[4], qh4[4], ql4[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 kf = __half22float2(k2[e]);
                    const float2 qf = __half22float2(q2[e]);
                    dqs = fmaf(qf.x, kf.x, dqs);
                    dqs = fmaf(qf.y, kf.y, dqs);
                    const float q0 = qf.x * ptx::ex2(bt[2 * e] - rq[2 * e]);
                    const float q1 = qf.y * ptx::ex2(bt[2 * e + 1] - rq[2 * e + 1]);
                    const float k0 = kf.x * ptx::ex2(rr[2 * e] - bt[2 * e]);
                    const float k1 = kf.y * ptx::ex2(rr[2 * e + 1] - bt[2 * e + 1]);
                    split_bf2(k0, k1, kh4[e], kl4[e]);
                    split_bf2(q0, q1, qh4[e], ql4[e]);
                    ks4[e] = pack_h2(k0 * ff[2 * e], k1 * ff[2 * e + 1]);
                }
                *reinterpret_cast<uint4 *>(sm + stage + C::kTK + o) = make_uint4(kh4[0], kh4[1], kh4[2], kh4[3]);
                *reinterpret_cast<uint4 *>(sm + stage + C::kTA + o) = make_uint4(kl4[0], kl4[1], kl4[2], kl4[3]);
                *reinterpret_cast<uint4 *>(sm + stage + C::kTQ + o) = make_uint4(ks4[0], ks4[1], ks4[2], ks4[3]);
                ptx::tmem_st16x2_x4<8>(rows + C::kColQH + 16 * hg + 4 * jj, qh4);
                ptx::tmem_st16x2_x4<8>(rows + C::kColQL + 16 * hg + 4 * jj, ql4);
            }
            m.dqp[slot][cg][t] = dqs * p.scale;
            ptx::tmem_st_wait();
        };
        // exact-score path (rare): Q~ = q 2^{b} d_k^{-1/2} into TMEM, Ks = k 2^{B - b}; K~ unused
        auto build_slow = [&](uint32_t stage, int slot) {
            float dqs = 0.0f;
            const uint32_t rows = tmem_q + ((uint32_t)(32 * qd + 16 * slot) << 16);
#pragma unroll 1
            for (int jj = 0; jj < 2; ++jj) {
                const int j = 2 * cg + jj;
                const uint32_t o = off_h<64>(t, j);
                const uint4 kraw = *reinterpret_cast<const uint4 *>(sm + stage + C::kTK + o);
                const uint4 qraw = *reinterpret_cast<const uint4 *>(sm + stage + C::kTQ + o);
                const __half2 *k2 = reinterpret_cast<const __half2 *>(&kraw);
                const __half2 *q2 = reinterpret_cast<const __half2 *>(&qraw);
                uint32_t ks4[4], qh4[4], ql4[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 kf = __half22float2(k2[e]);
                    const float2 qf = __half22float2(q2[e]);
                    dqs = fmaf(qf.x, kf.x, dqs);
                    dqs = fmaf(qf.y, kf.y, dqs);
                    float b2[2], B2[2], rq2[2];
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int ch = 8 * j + 2 * e + h;
                        b2[h] = *reinterpret_cast<const float *>(sm + C::kB + off_f<64>(t, ch >> 2) + (ch & 3) * 4);
                        B2[h] = m.Bc[slot][ch];
                        rq2[h] = m.rq[slot][ch];
                    }
                    split_bf2(qf.x * ptx::ex2(b2[0] - rq2[0]), qf.y * ptx::ex2(b2[1] - rq2[1]), qh4[e], ql4[e]);
                    ks4[e] = pack_h2(kf.x * ptx::ex2(B2[0] - b2[0]), kf.y * ptx::ex2(B2[1] - b2[1]));
                }
                *reinterpret_cast<uint4 *>(sm + stage + C::kTQ + o) = make_uint4(ks4[0], ks4[1], ks4[2], ks4[3]);
                ptx::tmem_st16x2_x4<8>(rows + C::kColQH + 16 * hg + 4 * jj, qh4);
                ptx::tmem_st16x2_x4<8>(rows + C::kColQL + 16 * hg + 4 * jj, ql4);
            }
            m.dqp[slot][cg][t] = dqs * p.scale;
            ptx::tmem_st_wait();
        };
        auto step = [&](int j) {
            const int slot = j & 1, s = j % 3;
            const uint32_t stage = (uint32_t)s * C::kStage;
            const Chunk c = chunk_of(j);
            if (j >= 2) wait(&m.slotfree[slot], (j - 2) >> 1);    // back team done with chunk j - 2
            wait(&m.ld[s], j / 3);
            ptx::tc_fence_after_sync();
            const bool slow = gate(stage, c, slot);
            if (ttid == 0) ptx::mbar_arrive(&m.gdone[slot]);        // r of the chunk: S~ may start
            if (!c.full) {
                build_ks(stage, slot);
            } else {
                if (slow) {
                    exact_p_smem(stage, c);
                    build_slow(stage, slot);
                } else {
                    build_full(stage, slot);
                }
            }
            ptx::fence_proxy_async_smem();
            ptx::tc_fence_before_sync();
            team_bar(1);
            if (ttid == 0) ptx::mbar_arrive(&m.fdone[slot]);
        };
        for (int j = 0; j < n1; ++j) step(j);
        if (exchange) run_exchange();
        for (int j = n1; j < N; ++j) step(j);
        __syncthreads();
    }

    // =================================================================== back team
    else if (back) {
        // S~^T of chunk i = S^T Diag(2^{r_i}) from the carried state: bf16 high / low parts into
        // the stage's S~ tiles (K-major rows j, the second half of the fused product's operand)
        auto prep_sx = [&](int i) {
            const int slot = i & 1;
            wait(&m.gdone[slot], i >> 1);               // r of chunk i
            if (chunk_of(i).full) {
                uint8_t *stg = sm + (uint32_t)(i % 3) * C::kStage;
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const float4 fa = *reinterpret_cast<const float4 *>(&m.er[slot][16 * cg + 8 * q]);
                    const float4 fb = *reinterpret_cast<const float4 *>(&m.er[slot][16 * cg + 8 * q + 4]);
                    const float f[8] = {fa.x, fa.y, fa.z, fa.w, fb.x, fb.y, fb.z, fb.w};
                    uint32_t h[4], l[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        split_bf2(f[2 * e] * S[8 * q + 2 * e], f[2 * e + 1] * S[8 * q + 2 * e + 1], h[e], l[e]);
                    const uint32_t o = off_h<64>(sc, 2 * cg + q);
                    *reinterpret_cast<uint4 *>(stg + C::kTSH + o) = make_uint4(h[0], h[1], h[2], h[3]);
                    *reinterpret_cast<uint4 *>(stg + C::kTSL + o) = make_uint4(l[0], l[1], l[2], l[3]);
                }
                ptx::fence_proxy_async_smem();
                team_bar(2);
            }
            if (ttid == 0) ptx::mbar_arrive(&m.sx[slot]);
        };
        auto step = [&](int j) {
            const int slot = j & 1, s = j % 3;
            const uint32_t stage = (uint32_t)s * C::kStage;
            const Chunk c = chunk_of(j);
            const uint32_t rows = tmem_rows(slot);
            wait(&m.fdone[slot], j >> 1);              // gate scalars, dq, slow flag of chunk j
            wait(&m.sc[slot], j >> 1);                 // [scores | inter] done (a bare commit if state-only)
            if (c.full) {
                ptx::tc_fence_after_sync();
                if (!m.slow[slot]) {
                    float dq = 0.0f;
#pragma unroll
                    for (int g = 0; g < 4; ++g) dq += m.dqp[slot][g][t];
                    const int s0 = 16 * cg, n = c.n;
                    const uint32_t mk = ln.before_mask(n, t, s0);
                    float r[16];
                    ptx::tmem_ld16x2_x16<16>(rows + C::kColSC + 32 * hg, r);
                    ptx::tmem_ld_wait();
                    float amax = 0.0f;
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        r[e] = (mk >> e & 1u) ? r[e] : 0.0f;
                        amax = fmaxf(amax, fabsf(r[e]));
                    }
                    const bool diag = t < n && (unsigned)(t - s0) < 16u;    // exact q_t . k_t
                    if (diag) amax = fmaxf(amax, fabsf(dq));
                    if (amax > 65504.0f) m.range_err = 1;
#pragma unroll
                    for (int h = 0; h < 2; ++h)
                        *reinterpret_cast<uint4 *>(sm + stage + C::kTA + off_h<64>(t, 2 * cg + h)) =
                            make_uint4(pack_h2(r[8 * h], r[8 * h + 1]), pack_h2(r[8 * h + 2], r[8 * h + 3]),
                                       pack_h2(r[8 * h + 4], r[8 * h + 5]), pack_h2(r[8 * h + 6], r[8 * h + 7]));
                    if (diag)
                        *reinterpret_cast<__half *>(sm + stage + C::kTA + off_h<64>(t, t >> 3) + (t & 7) * 2) =
                            __float2half_rn(dq);
                }
                ptx::fence_proxy_async_smem();
                ptx::tc_fence_before_sync();
                team_bar(2);
            }
            if (ttid == 0) ptx::mbar_arrive(&m.pfull[slot]);
            // S^T = S^T Diag(2^{B}) + S_loc^T
            wait(&m.sl[slot], j >> 1);
            ptx::tc_fence_after_sync();
            {
                float sl[16];
                ptx::tmem_ld16x2_x16<16>(rows + C::kColSL + 32 * hg, sl);
                ptx::tmem_ld_wait();
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float4 e = *reinterpret_cast<const float4 *>(&m.eB[slot][16 * cg + 4 * q]);
                    S[4 * q] = fmaf(e.x, S[4 * q], sl[4 * q]);
                    S[4 * q + 1] = fmaf(e.y, S[4 * q + 1], sl[4 * q + 1]);
                    S[4 * q + 2] = fmaf(e.z, S[4 * q + 2], sl[4 * q + 2]);
                    S[4 * q + 3] = fmaf(e.w, S[4 * q + 3], sl[4 * q + 3]);
                }
            }
            if (!c.full && ttid < D) m.Gs[ttid] += m.Bc[slot][ttid];
            // the next chunk's S~ now, so its fused product runs under this chunk's epilogue (the
            // first full chunk after an exchange waits for the incoming state)
            if (j + 1 < N && j + 1 != n1) prep_sx(j + 1);
            wait(&m.o[slot], j >> 1);                   // a state-only chunk's is a bare commit
            if (c.full) {
                ptx::tc_fence_after_sync();
                float o[16];
                ptx::tmem_ld16x2_x16<16>(rows + C::kColO + 32 * hg, o);
                ptx::tmem_ld_wait();
                float ss = 0.0f;
#pragma unroll
                for (int jj = 0; jj < 16; ++jj) ss = fmaf(o[jj], o[jj], ss);
                m.red[cg][t] = ss;
                team_bar(2);
                const float inv = rsqrtf((m.red[0][t] + m.red[1][t] + m.red[2][t] + m.red[3][t]) * (1.0f / D) + p.eps);
                // the TMEM loads are warp-collective: every lane takes them, rows past the chunk
                // only skip the arithmetic and the store
                const int orow = t < c.n ? token_row(c, t) : 0;
                const bool live = t < c.n && GLA_CHECK(orow >= 0 && orow < p.B * p.L * p.H);
                __half *dst = p.out + (size_t)(live ? orow : 0) * D + 16 * cg;
#pragma unroll 1
                for (int jj = 0; jj < 2; ++jj) {
                    const int jp = 2 * cg + jj;
                    float o8[8];
                    ptx::tmem_ld16x2_x8<16>(rows + C::kColO + 32 * hg + 8 * jj, o8);
                    ptx::tmem_ld_wait();
                    if (live) {
                        const uint4 graw = *reinterpret_cast<const uint4 *>(sm + stage + C::kTG + off_h<64>(t, jp));
                        const __half2 *g2 = reinterpret_cast<const __half2 *>(&graw);
                        const float4 wa = *reinterpret_cast<const float4 *>(&m.w[8 * jp]);
                        const float4 wb = *reinterpret_cast<const float4 *>(&m.w[8 * jp + 4]);
                        const float wv[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
                        uint32_t u[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 gf = __half22float2(g2[e]);
                            u[e] = pack_h2(o8[2 * e] * inv * wv[2 * e] * silu_fast(gf.x),
                                           o8[2 * e + 1] * inv * wv[2 * e + 1] * silu_fast(gf.y));
                        }
                        *reinterpret_cast<uint4 *>(dst + 8 * jj) = make_uint4(u[0], u[1], u[2], u[3]);
                    }
                }
            }
            ptx::tc_fence_before_sync();
            team_bar(2);                                // every read of this slot and stage is done
            if (ttid == 0) {
                ptx::mbar_arrive(&m.slotfree[slot]);
                ptx::mbar_arrive(&m.stfree[s]);
            }
        };
        if (n1 > 0) prep_sx(0);
        for (int j = 0; j < n1; ++j) step(j);
        if (exchange) run_exchange();
        if (n1 < N) prep_sx(n1);
        for (int j = n1; j < N; ++j) step(j);
        __syncthreads();
    }

    // ---- teardown (every thread arrives here after the role's own teardown barrier)
    __syncthreads();
    if (tid == 0 && m.range_err) raise_status(8 /* GLA_ERR_RANGE */);
    ptx::tc_fence_after_sync();
    if (warp == 0) ptx::tmem_dealloc(tmem, C::kTmemCols);
}

}  // namespace ck
}  // namespace gla
