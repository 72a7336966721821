/*
 * gla.h -- C ABI of libgla.so, the B200 (sm_100a) key-only gated linear
 * attention (GLA) token mixer of GTR.
 *
 * Operation (GTR paper, arXiv 2609.26590, method section): for every batch
 * element b and head h, over the L = grid_h * grid_w tokens of a patch grid
 * visited in one of four scan directions,
 *
 *     gamma_t = sigma(a_t)^(1/16)                 (key-wise retention gate)
 *     S_t     = Diag(gamma_t) S_{t-1} + k_t^T v_t, S_0 = 0   (d_k x d_v state)
 *     o_t     = d_k^{-1/2} q_t S_t
 *     u_t     = SiLU(g_t) * o_t / sqrt(mean_j(o_tj^2) + eps) * w   (eps = 1e-6)
 *
 * and u_t is written back at the token's ORIGINAL spatial position.  The
 * value-side decay is fixed to one.  The scan directions (same paper, method
 * section, "four scan directions"): 0 = left-to-right (rows top to bottom,
 * each row left to right), 1 = right-to-left (rows top to bottom, each row
 * right to left), 2 = top-to-bottom (columns left to right, each column top
 * to bottom), 3 = bottom-to-top (columns left to right, each column bottom to
 * top); the state carries over from one row/column to the next.  4 =
 * GLA_DIR_CYCLE: batch element b uses direction b % 4 (the paper cycles the
 * four directions across blocks; this batches the four in one launch).
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
    GLA_ERR_NO_DEVICE = 9    /* no usable sm_100 device                          */
};

enum gla_direction {
    GLA_DIR_L2R = 0,
    GLA_DIR_R2L = 1,
    GLA_DIR_T2B = 2,
    GLA_DIR_B2T = 3,
    GLA_DIR_CYCLE = 4
};

/*
 * gla_fwd -- fp16 I/O, fp32 arithmetic.  q, k, v, gate_preact,
 * out_gate_preact and out are IEEE binary16 arrays; rms_weight is float32.
 * `stream` is a cudaStream_t (NULL = legacy default stream).
 * Supported head dims: d_k, d_v in {32, 64, 128}.
 */
int gla_fwd(const void *q, const void *k, const void *v,
            const void *gate_preact, const void *out_gate_preact,
            const float *rms_weight, void *out,
            int B, int H, int grid_h, int grid_w, int d_k, int d_v,
            int direction, void *stream);

/*
 * gla_fwd_f32 -- the same operation with float32 I/O and float32 arithmetic
 * throughout (CUDA cores; no TF32), for callers that need ~1e-6 agreement.
 */
int gla_fwd_f32(const float *q, const float *k, const float *v,
                const float *gate_preact, const float *out_gate_preact,
                const float *rms_weight, float *out,
                int B, int H, int grid_h, int grid_w, int d_k, int d_v,
                int direction, void *stream);

/*
 * gla_fwd_host -- gla_fwd / gla_fwd_f32 on HOST buffers (dtype 0 = fp16,
 * 1 = fp32).  Copies the inputs to device buffers owned by the library
 * (grown on demand, kept between calls, one set per device), runs the
 * operation on `stream`, copies `out` back and synchronises `stream` before
 * returning.  Host buffers in page-locked memory make the copies
 * asynchronous DMA.  Not capturable (it synchronises); not thread-safe for
 * concurrent calls on the same device.
 */
int gla_fwd_host(const void *q, const void *k, const void *v,
                 const void *gate_preact, const void *out_gate_preact,
                 const float *rms_weight, void *out,
                 int B, int H, int grid_h, int grid_w, int d_k, int d_v,
                 int direction, int dtype, void *stream);

/*
 * gla_fwd_ex -- gla_fwd / gla_fwd_f32 (dtype 0 / 1) with the schedule and
 * epsilon exposed, for tests: `chunk` = tokens per chunk (0 = the default
 * of the chosen kernel; otherwise a multiple of 16 that the kernel supports,
 * else GLA_ERR_UNSUPPORTED), `segments` = CTAs per (b, h) pair splitting the
 * scan (0 = automatic, else 1..16; the tensor-core kernel refuses 13, 14 and
 * 15 with GLA_ERR_UNSUPPORTED, as their key-channel groups do not fit its
 * state-exchange buffer), `eps` the RMSNorm epsilon.  Every valid choice
 * computes the same operation (up to rounding order).
 */
int gla_fwd_ex(const void *q, const void *k, const void *v,
               const void *gate_preact, const void *out_gate_preact,
               const float *rms_weight, void *out,
               int B, int H, int grid_h, int grid_w, int d_k, int d_v,
               int direction, int dtype, int chunk, int segments, float eps,
               void *stream);

/*
 * gla_get_status -- synchronises `stream`, returns the current device's
 * latched device-side status in *device_status (GLA_OK if none) and clears
 * it.  Returns GLA_ERR_CUDA if the synchronisation itself failed.
 */
int gla_get_status(void *stream, int *device_status);

/* gla_status_string -- static, human-readable name of a status code. */
const char *gla_status_string(int code);

/* gla_version -- library version, major*10000 + minor*100 + patch. */
int gla_version(void);

/*
 * gla_plan -- the schedule gla_fwd (dtype 0) / gla_fwd_f32 (dtype 1) would
 * use for these shapes on the current device, without launching anything:
 * *kernel = 1 (tensor-core kernel) or 2 (CUDA-core kernel), *segments = CTAs
 * (one thread-block cluster) per (b, h) pair, *seg_len = scan positions per
 * segment, *ctas = total CTAs, *max_active_clusters = clusters of that shape
 * the device can hold at once.  Same argument errors as gla_fwd.
 */
int gla_plan(int B, int H, int grid_h, int grid_w, int d_k, int d_v, int dtype, int *kernel,
             int *segments, int *seg_len, int *ctas, int *max_active_clusters);

/*
 * gla_empty_launch -- measurement aid: launches a kernel with exactly the launch shape
 * gla_fwd uses for fp16 d_k = d_v = 64 at these dimensions (grid, thread-block cluster,
 * block size, dynamic shared memory, programmatic dependent launch) whose body only
 * performs the dependent-launch handshake.  Timing a run of these gives the per-launch
 * floor of that shape.  Asynchronous on `stream`.  GLA_ERR_SHAPE for non-positive
 * dimensions; GLA_ERR_UNSUPPORTED when those dimensions would not use the tensor-core kernel.
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
 * gla_selftest_mma -- diagnostic: runs ONE of the tensor-core kernel's four
 * matrix products on a single CTA, with the kernel's own shared-memory
 * layouts and descriptors, on row-major float32 DEVICE arrays:
 *   kind 0  D[128][128] = A[128][64] * B[128][64]^T   (split tf32: each operand is
 *           held as tf32 high + low parts, three products; ~fp32 accuracy)
 *   kind 1  D[64][64]   = B[128][64]^T * A[128][64]   (fp16 operands, the state product,
 *           kept transposed: A plays the decayed keys, B the values)
 *   kind 2  D[128][64]  = A[128][128] * B[128][64]    (fp16 operands, P * V)
 *   kind 3  D[128][64]  = A[128][64] * B[64][64]^T    (tf32, the inter-chunk product)
 * Inputs are rounded to the operand type (tf32 or fp16; kind 0 splits them)
 * on the way in; accumulation is fp32.  Asynchronous on `stream`.  Returns GLA_ERR_UNSUPPORTED
 * for another kind.  Not part of the operation itself.
 */
int gla_selftest_mma(int kind, const float *A, const float *B, float *D, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* GLA_H_ */
