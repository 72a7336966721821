/*
 * gla.h -- C ABI of libgla.so, the B200 (sm_100a) key-only gated linear
 * attention (GLA) token mixer of GTR.
 *
 * Operation ("GTR: Gated Token Recurrence for Efficient Dense Prediction",
 * arXiv 2609.26590, method section): for every batch element b and head h,
 * over the L = grid_h * grid_w tokens of a patch grid visited in one of four
 * scan directions,
 *
 *     gamma_t = sigma(a_t)^(1/16)                 (key-wise retention gate)
 *     S_t     = Diag(gamma_t) S_{t-1} + k_t^T v_t, S_0 = 0   (d_k x d_v state)
 *     o_t     = d_k^{-1/2} q_t S_t
 *     u_t     = SiLU(g_t) * o_t / sqrt(mean_j(o_tj^2) + eps) * w   (eps = 1e-6)
 *
 * and u_t is written back at the token's ORIGINAL spatial position.  The
 * value-side decay is fixed to one.  The scan directions (same section, the
 * scan-direction paragraph): 0 = left-to-right (rows top to bottom, each row
 * left to right), 1 = right-to-left (rows top to bottom, each row right to
 * left), 2 = top-to-bottom (columns left to right, each column top to bottom),
 * 3 = bottom-to-top (columns left to right, each column bottom to top); the
 * state carries over from one row/column to the next.  4 = GLA_DIR_CYCLE:
 * batch element b uses direction b % 4 (the paper cycles the four directions
 * across blocks; this batches the four in one launch).
 *
 * Layouts: every array is dense and token-major with the head interleaved:
 *     q, k, gate_preact (a):        [B][L][H][d_k]
 *     v, out_gate_preact (g), out:  [B][L][H][d_v]
 *     rms_weight (w):               [d_v] float32, shared by all heads
 * with L = grid_h * grid_w in row-major spatial order (index y*grid_w + x).
 * gate_preact is the full retention-gate pre-activation (x W1 W2 + b) and
 * out_gate_preact is x W_r; both activations are applied inside the call.
 * Input values must be finite: the kernels do not check them, and an
 * infinite or NaN element leaves the outputs of its (b, h) pair undefined.
 *
 * Pointers are DEVICE pointers (except in gla_fwd_host), 16-byte aligned,
 * owned by the caller; out must not overlap any input.  gla_fwd,
 * gla_fwd_f32 and gla_fwd_ex are asynchronous on their stream, never
 * synchronise and allocate no device memory.
 *
 * Errors: argument errors are returned synchronously before anything is
 * launched; a launch failure returns GLA_ERR_CUDA (the CUDA error is consumed).
 * Device-side faults detected by the kernels (GLA_ERR_TIMEOUT, GLA_ERR_RANGE)
 * are latched in a per-device status word read by gla_get_status().
 *
 * Checked build: libgla_checked.so is compiled from the same sources with
 * -DGLA_CHECKED.  It exports the same calls; in it every computed index that
 * addresses device or shared memory (gathered and stored token rows, TMA box
 * coordinates, remote exchange rows, chunk geometry) is checked against its
 * buffer first, and a violation latches GLA_ERR_CHECK and skips the access.
 * It stands in for a memory checker on hardware where none can run.
 */
#ifndef GLA_H_
#define GLA_H_

#ifdef __cplusplus
extern "C" {
#endif

enum gla_status {
    GLA_OK = 0,
    GLA_ERR_NULL = 1,        /* a required pointer is NULL                     */
    GLA_ERR_SHAPE = 2,       /* B, H, grid_h, grid_w <= 0 or sizes overflow     */
    GLA_ERR_UNSUPPORTED = 3, /* d_k/d_v not in {32,64,128}, misaligned pointer, */
                             /* or an unsupported chunk/segment override        */
    GLA_ERR_DIRECTION = 4,   /* direction not in 0..4                           */
    GLA_ERR_ALIAS = 5,       /* out overlaps an input                           */
    GLA_ERR_CUDA = 6,        /* CUDA launch/runtime error                        */
    GLA_ERR_TIMEOUT = 7,     /* device: a bounded wait ran out                   */
    GLA_ERR_RANGE = 8,       /* device: an intermediate left the operand range   */
    GLA_ERR_NO_DEVICE = 9,   /* no usable sm_100 device                          */
    GLA_ERR_CHECK = 10       /* device: an index check failed (the checked build,  */
                             /* libgla_checked.so, only; the access was skipped)  */
};

enum gla_direction {
    GLA_DIR_L2R = 0,
    GLA_DIR_R2L = 1,
    GLA_DIR_T2B = 2,
    GLA_DIR_B2T = 3,
    GLA_DIR_CYCLE = 4
};

/*
 * gla_fwd -- the operation above with fp16 I/O and fp32 arithmetic.
 * Defined by the GTR paper's method section: the GLA recurrence paragraph (state,
 * gate, readout), the output-gate paragraph (SiLU gate times RMSNorm) and the
 * scan-direction paragraph (four directions, results in the original order).
 * q, k, v, gate_preact, out_gate_preact and out are IEEE binary16 arrays;
 * rms_weight is float32.  `stream` is a cudaStream_t (NULL = legacy default
 * stream).  Supported head dims: d_k, d_v in {32, 64, 128}; d_k = d_v = 64 runs on
 * the pipelined 64-row tensor-core kernel when B * H is at least the device's SM count or
 * grid_h * grid_w >= 4096, else on the 128-row one; d_k = d_v = 128 on the 64-row kernel;
 * the others on CUDA cores (gla_kernel below).  A call may issue two kernel launches: when
 * the pipelined kernel's pairs exceed a whole number of waves, the last partial wave's pairs
 * run as a second launch with several CTAs per pair.
 */
int gla_fwd(const void *q, const void *k, const void *v,
            const void *gate_preact, const void *out_gate_preact,
            const float *rms_weight, void *out,
            int B, int H, int grid_h, int grid_w, int d_k, int d_v,
            int direction, void *stream);

/*
 * gla_fwd_f32 -- the same operation (same paragraphs of the GTR method section) with
 * float32 I/O and float32 arithmetic throughout (CUDA cores; no TF32), for callers
 * that need ~1e-6 agreement.
 */
int gla_fwd_f32(const float *q, const float *k, const float *v,
                const float *gate_preact, const float *out_gate_preact,
                const float *rms_weight, float *out,
                int B, int H, int grid_h, int grid_w, int d_k, int d_v,
                int direction, void *stream);

/*
 * gla_fwd_host -- gla_fwd / gla_fwd_f32 on HOST buffers (dtype 0 = fp16,
 * 1 = fp32); the operation of the GTR method section as above.  Copies the
 * inputs to device buffers owned by the library (grown on demand, kept between
 * calls, one set per device), runs the operation on `stream`, copies `out` back
 * and synchronises `stream` before returning.  Host buffers in page-locked
 * memory make the copies asynchronous DMA.  Not capturable (it synchronises);
 * not thread-safe for concurrent calls on the same device.
 */
int gla_fwd_host(const void *q, const void *k, const void *v,
                 const void *gate_preact, const void *out_gate_preact,
                 const float *rms_weight, void *out,
                 int B, int H, int grid_h, int grid_w, int d_k, int d_v,
                 int direction, int dtype, void *stream);

/* Kernels gla_fwd_ex can be asked for (gla_plan reports the same ids). */
enum gla_kernel {
    GLA_KERNEL_AUTO = 0,   /* the one gla_fwd / gla_fwd_f32 choose                       */
    GLA_KERNEL_TC128 = 1,  /* tensor cores, 128-row chunks: fp16, d_k = d_v = 64           */
    GLA_KERNEL_SIMT = 2,   /* CUDA cores: every supported shape, fp16 or fp32              */
    GLA_KERNEL_TC64 = 3,   /* tensor cores, 64-row chunks, TMA loads: fp16, d_k = d_v in   */
                           /* {64, 128}                                                    */
    GLA_KERNEL_PIPE64 = 4  /* the 64-row kernel with two chunks in flight (warp-specialised */
                           /* teams, 3-stage TMA ring, chunks packed across lines, scores   */
                           /* and inter product in one N = 128 product): fp16, d = 64       */
};

/*
 * gla_fwd_ex -- gla_fwd / gla_fwd_f32 (dtype 0 / 1) with the kernel, the schedule
 * and epsilon exposed, for tests; the operation of the GTR method section as above.
 * `chunk` = tokens per chunk (0 = the default of the kernel; otherwise a multiple
 * of 16 that the kernel supports: up to 128 for GLA_KERNEL_TC128, 64 for the others,
 * else GLA_ERR_UNSUPPORTED), `segments` = CTAs per (b, h) pair splitting the scan
 * (0 = automatic, else 1..16; GLA_KERNEL_TC128 refuses 13, 14 and 15), `eps` the
 * RMSNorm epsilon, `kernel` a gla_kernel (GLA_ERR_UNSUPPORTED when that kernel does
 * not take this dtype or head dim).  Every valid choice computes the same operation
 * (up to rounding order).
 */
int gla_fwd_ex(const void *q, const void *k, const void *v,
               const void *gate_preact, const void *out_gate_preact,
               const float *rms_weight, void *out,
               int B, int H, int grid_h, int grid_w, int d_k, int d_v,
               int direction, int dtype, int chunk, int segments, float eps,
               int kernel, void *stream);

/*
 * gla_get_status -- synchronises `stream`, returns the current device's
 * latched device-side status in *device_status (GLA_OK if none) and clears
 * it.  Returns GLA_ERR_CUDA if the synchronisation itself failed.  The pages
 * define no error reporting; the status word is this library's own.
 */
int gla_get_status(void *stream, int *device_status);

/* gla_status_string -- static, human-readable name of a status code. */
const char *gla_status_string(int code);

/* gla_version -- library version, major*10000 + minor*100 + patch. */
int gla_version(void);

/*
 * gla_plan -- the schedule gla_fwd (dtype 0) / gla_fwd_f32 (dtype 1) would
 * use for these shapes on the current device, without launching anything:
 * *kernel = the gla_kernel it runs (1 to 4), *segments = CTAs (one
 * thread-block cluster) per (b, h) pair, *seg_len = scan positions per
 * segment, *ctas = total CTAs (of both launches when the call is split; then
 * *segments and *seg_len describe the first), *max_active_clusters = clusters
 * of that shape the device can hold at once.  Same argument errors as gla_fwd.
 */
int gla_plan(int B, int H, int grid_h, int grid_w, int d_k, int d_v, int dtype, int *kernel,
             int *segments, int *seg_len, int *ctas, int *max_active_clusters);

/*
 * gla_empty_launch -- measurement aid: launches a kernel with exactly the launch shape
 * gla_fwd uses for fp16 d_k = d_v = 64 at these dimensions (grid, thread-block cluster,
 * block size, dynamic shared memory, programmatic dependent launch) whose body only
 * performs the dependent-launch handshake.  Timing a run of these gives the per-launch
 * floor of that shape.  Asynchronous on `stream`.  GLA_ERR_SHAPE for non-positive
 * dimensions.
 */
int gla_empty_launch(int B, int H, int grid_h, int grid_w, void *stream);

/*
 * gla_selftest_timeout -- diagnostic for device-side failure detection: launches a
 * one-thread kernel that waits, with the kernels' bounded-wait loop but a bound of
 * `limit_cycles` SM clocks (1 .. 2^34), on a barrier nothing ever signals.  The wait
 * expires, GLA_ERR_TIMEOUT is latched in the device status word (read it with
 * gla_get_status) and the kernel returns; the context stays usable.  Asynchronous on
 * `stream`; GLA_ERR_UNSUPPORTED for a bound out of range.
 */
int gla_selftest_timeout(long long limit_cycles, void *stream);

/*
 * gla_selftest_fault -- diagnostic for device-side failure detection in the operator's
 * own tensor-core kernels: runs gla_fwd (fp16, d_k = d_v = d) on `kernel`
 * (GLA_KERNEL_TC128 or GLA_KERNEL_PIPE64 with d = 64, or GLA_KERNEL_TC64 with d in {64, 128};
 * `segments` CTAs
 * per pair or 0 for automatic) with every bounded wait limited to `wait_limit_cycles` SM
 * clocks (1 .. 2^34), while the loads of full-pass chunk `withheld_chunk` of every segment
 * never complete their barrier (-1: none): the 64-row kernel does not issue them, the
 * 128-row kernel issues the q / k copies without their barrier arrival.  The wait on those
 * tiles expires, GLA_ERR_TIMEOUT is latched, the CTA skips its remaining waits and products,
 * drains what is in flight and returns; `out` is then undefined.  Arguments as gla_fwd;
 * asynchronous.
 */
int gla_selftest_fault(const void *q, const void *k, const void *v,
                       const void *gate_preact, const void *out_gate_preact,
                       const float *rms_weight, void *out,
                       int B, int H, int grid_h, int grid_w, int d, int direction,
                       int segments, long long wait_limit_cycles, int withheld_chunk,
                       int kernel, void *stream);

/*
 * gla_selftest_rcp -- diagnostic: y[i] = the 128-row kernel's Newton-Raphson reciprocal of
 * x[i] (n DEVICE floats each), for an error-bound test against 1/x.  The pages have no
 * counterpart; asynchronous on `stream`.
 */
int gla_selftest_rcp(const float *x, float *y, int n, void *stream);

/*
 * gla_selftest_chunk -- diagnostic: runs ONE of the tensor-core kernel's matrix products
 * for head dim d in {64, 128} on a single CTA, with the kernel's own shared-memory and
 * TMEM layouts, descriptors and TMEM accesses, on row-major float32 DEVICE arrays:
 *   kind 0  D[64][64] = A[64][d] * B[64][d]^T   (scores; each operand split into bf16
 *           high + low parts, three products: ~2^-16 relative)
 *   kind 1  D[d][d]   = A[64][d]^T * B[64][d]   (fp16 operands, the chunk-state product)
 *   kind 2  D[64][d]  = A[64][64] * B[64][d]    (fp16 operands, P * V, A held in TMEM)
 *   kind 3  D[64][d]  = A[64][d] * B[d][d]      (bf16 split, the inter-chunk product)
 *   kind 4  D[64][64] = A[64][64] * B[64][64]   (fp16, P * V with P from shared memory, the
 *           pipelined kernel's form; d = 64 only)
 * Inputs are rounded to the operand type on the way in; accumulation is fp32.
 * Asynchronous on `stream`.  Not part of the operation itself.
 */
int gla_selftest_chunk(int d, int kind, const float *A, const float *B, float *D, void *stream);

/*
 * gla_selftest_load -- diagnostic: loads the five 64-row tiles (q, k, gate_preact, v,
 * out_gate_preact, fp16 DEVICE arrays laid out as for gla_fwd with d_k = d_v = d in
 * {64, 128}) of chunk `chunk` of the scan of pair (b, h) = (0, 0) in `direction` (0..3) with
 * the tensor-core kernel's TMA boxes, and writes them to out[5][64][d] (DEVICE float32) in
 * tile-row order, with info[0] = the chunk's token count n and info[1 + i] = the spatial
 * index of tile row i (-1 for rows past the chunk) (DEVICE int[65]).  Chunks are the kernel's
 * default ones (lines cut into pieces of at most 64 positions).  Asynchronous on `stream`.
 * Not part of the operation itself.
 */
int gla_selftest_load(const void *q, const void *k, const void *gate_preact, const void *v,
                      const void *out_gate_preact, int B, int H, int grid_h, int grid_w, int d,
                      int direction, int chunk, float *out, int *info, void *stream);

/*
 * gla_gate_proj -- the retention gate's pre-activation, the input gate_preact of gla_fwd:
 *     a[t][c] = sum_j (sum_i x[t][i] w1[i][j]) w2[j][c] + bias[c]
 * GTR paper's method section, GLA recurrence paragraph: gamma_t = sigma(x_t W_alpha^(1)
 * W_alpha^(2) + b_alpha)^(1/tau), a low-rank projection of rank r = 16, read as GLA builds
 * it: one first factor shared by the heads, a second factor onto every head's
 * key channels.  x: [tokens][d_model] fp16 (token-major, tokens = B * L), w1: [d_model][rank]
 * fp16, w2: [rank][n_out] fp16 (n_out = H * d_k, head-major), bias: [n_out] float32, a:
 * [tokens][n_out] fp16 -- the [B][L][H][d_k] layout gla_fwd reads.  DEVICE pointers, 16-byte
 * aligned, caller-owned; a must not overlap an input (GLA_ERR_ALIAS).  rank must be 16,
 * d_model a multiple of 64 up to 1024, n_out a multiple of 128 up to 1024, else
 * GLA_ERR_UNSUPPORTED.  tcgen05 tensor cores: x W1 with fp32 accumulation, that product split
 * into fp16 high and low parts for the second factor, fp16 output.  Asynchronous on `stream`;
 * an intermediate above the fp16 range latches GLA_ERR_RANGE.
 */
int gla_gate_proj(const void *x, const void *w1, const void *w2, const float *bias, void *a,
                  int tokens, int d_model, int rank, int n_out, void *stream);

/*
 * gla_linear -- the block's dense projections, y = x W (+ bias):
 *     y[part][t][c] = sum_k x[t][k] W[k][part * n_part + c] (+ bias[part * n_part + c])
 * GTR paper's method section: the input projections Q = X W_Q, K = X W_K, V = X W_V (GLA
 * recurrence paragraph) and the output gate's x W_r, and the output projection of the
 * concatenated heads back to the model dimension (output-gate paragraph).  x: [rows][k_dim]
 * fp16, W: [k_dim][n_dim] fp16 (row-major), bias: [n_dim] float32 or NULL, y: fp16 written as
 * n_dim / n_part parts of [rows][n_part] each, one after another (n_part = n_dim: a plain
 * [rows][n_dim] matrix; W = [W_Q | W_K | W_V | W_r] with n_part = H * d: q, k, v and the output
 * gate's pre-activation as four [B][L][H][d] tensors).  DEVICE pointers, 16-byte aligned,
 * caller-owned; y must not overlap an input (GLA_ERR_ALIAS).  k_dim and n_part must be
 * multiples of 64 and n_dim a multiple of 128 or 192 divisible by n_part, else
 * GLA_ERR_UNSUPPORTED.  tcgen05 tensor cores, fp32 accumulation, fp16 output.  Asynchronous
 * on `stream`.
 */
int gla_linear(const void *x, const void *w, const float *bias, void *y, int rows, int k_dim, int n_dim,
               int n_part, void *stream);

/*
 * gla_sswiglu -- Spatial SwiGLU's token mixing step, fused:
 *     h[b][y][x][c] = SiLU(gate[b][y][x][c]) *
 *                     (conv_b[c] + sum_{i,j=0..2} conv_w[c][i][j] value[b][y+i-1][x+j-1][c])
 * GTR paper's method section, Spatial SwiGLU paragraph: the value branch is reshaped to the
 * 2-D patch grid, convolved 3x3 depthwise and restored to sequence order; the gating branch
 * stays tokenwise.  Read as a framework depthwise Conv2d (cross-correlation, zero padding of
 * one token, per-channel bias) times SiLU of the gating branch.  value, gate, h: [batch]
 * [grid_h * grid_w][channels] fp16, row-major grid (s = y * grid_w + x), 16-byte aligned;
 * conv_w [channels][3][3] and conv_b [channels] float32.  DEVICE pointers, caller-owned; h
 * must not overlap an input (GLA_ERR_ALIAS).  channels must be a multiple of 64
 * (GLA_ERR_UNSUPPORTED).  fp32 arithmetic, fp16 output; a result outside the fp16 range (or
 * NaN) latches GLA_ERR_RANGE.  Asynchronous on `stream`.
 */
int gla_sswiglu(const void *value, const void *gate, const float *conv_w, const float *conv_b, void *out,
                int batch, int grid_h, int grid_w, int channels, void *stream);

/*
 * gla_scan_layout -- host-only (no device work, no CUDA call): the token each tile row of
 * each chunk holds when `kernel` (GLA_KERNEL_PIPE64 only) runs a scan of a
 * grid_h x grid_w grid in `direction` (0..3) with chunks of at most `chunk` positions
 * (0: 64).  Writes spatial[p] = the row-major spatial index (y * grid_w + x) of the token the
 * kernel's tiles place at scan position p, for p in [0, grid_h * grid_w) (HOST int array of that
 * length; a position no tile row claims stays -1, one claimed twice returns GLA_ERR_SHAPE),
 * and *box_rows = the rows per TMA box (64 for line-aligned chunks; a forward row scan,
 * direction 0, loads whole chunks of consecutive token rows).  The scan order is the
 * one of the scan-direction paragraph of the GTR paper's method section (lines in increasing
 * order, the state carried from one line's end to the next line's start); the test suite
 * compares this map with the reference's own on the CPU.
 */
int gla_scan_layout(int kernel, int grid_h, int grid_w, int direction, int chunk, int *spatial,
                    int *box_rows);

/*
 * gla_selftest_mma -- diagnostic: runs ONE of the four matrix products of the previous
 * 128-row tensor-core kernel on a single CTA, on row-major float32 DEVICE arrays:
 *   kind 0  D[128][128] = A[128][64] * B[128][64]^T   (split tf32)
 *   kind 1  D[64][64]   = B[128][64]^T * A[128][64]   (fp16)
 *   kind 2  D[128][64]  = A[128][128] * B[128][64]    (fp16)
 *   kind 3  D[128][64]  = A[128][64] * B[64][64]^T    (tf32)
 * Asynchronous on `stream`.  Returns GLA_ERR_UNSUPPORTED for another kind.
 */
int gla_selftest_mma(int kind, const float *A, const float *B, float *D, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* GLA_H_ */
