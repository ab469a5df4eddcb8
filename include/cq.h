/*
 * cq.h -- C ABI of the B200 (sm_100a) CodeQuant LUT MoE linear layer.
 *
 * The layer is the low-precision MoE linear layer of CodeQuant / CodeQuant2:
 *   - activations get an online block Walsh-Hadamard rotation and per-token
 *     symmetric int4 (A4W4) or int8 (A8W4) quantization
 *     (CodeQuant abstract: rotation smooths activation outliers; CodeQuant2
 *     Figure 1: rotation fused into the model; CodeQuant2 Tables 1, 2, 9:
 *     the A4W4 / A8W4 settings);
 *   - each weight W[n,k] is a 4-bit index I[n,k] into a per-output-row codebook
 *     of 16 fp16 centroids C[n,0..15] (CodeQuant2 Figure 3: centroid matrix and
 *     per-row assignment matrices);
 *   - y[m,n] = s_x[m] * sum_k C[n, I[n,k]] * q[m,k], computed by a one-time
 *     lookup-table precompute followed by table lookups (CodeQuant2 Figure 4);
 *   - the product runs per expert after top-k routing (the MoE router of the
 *     CodeQuant podcast transcript, "Summary").
 *
 * Conventions for every entry point
 *   Memory      every pointer is DEVICE memory owned by the caller unless the
 *               argument says otherwise.  The library keeps no pointer after a
 *               call returns and allocates no device memory: scratch space is
 *               the caller's `workspace`.  Apart from the measurement aids at
 *               the end of this header it keeps no state between calls.
 *   Streams     work is enqueued on `stream` (NULL = legacy default stream)
 *               and the call returns without synchronizing.  Kernel faults
 *               surface at the caller's next synchronization.  Kernels are
 *               launched with programmatic stream serialization: one may start
 *               while the previous kernel on the stream is finishing, and it
 *               waits for that kernel to complete before it reads any output
 *               of it or writes global memory.
 *   Layout      row-major, densely packed (leading dimension = row length).
 *               Packed 4-bit data: element 2j in the LOW nibble of byte j,
 *               element 2j+1 in the high nibble.  int4 activation codes are
 *               two's complement in [-7, 7]; weight indices are unsigned 0..15.
 *   Alignment   every pointer must be 16-byte aligned.
 *   Errors      arguments are checked on the host before anything is
 *               launched; a failed check returns CQ_ERR_INVALID_ARGUMENT (bad
 *               value, null or misaligned pointer), CQ_ERR_UNSUPPORTED (valid
 *               but outside what the kernels handle), or CQ_ERR_WORKSPACE
 *               (workspace too small) and enqueues nothing.  CQ_ERR_CUDA
 *               reports a launch error.
 *   Inputs      must be finite; NaN / Inf give unspecified outputs.
 *   Threads     re-entrant; calls on different streams may run concurrently.
 */
#ifndef CQ_H_
#define CQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define CQ_API __attribute__((visibility("default")))
#else
#define CQ_API
#endif

/* ABI-compatible with cudaStream_t / CUstream. */
typedef struct CUstream_st *cq_stream_t;

typedef enum {
    CQ_OK = 0,
    CQ_ERR_INVALID_ARGUMENT = 1,
    CQ_ERR_UNSUPPORTED = 2,
    CQ_ERR_WORKSPACE = 3,
    CQ_ERR_CUDA = 4
} cq_status;

/* Static string describing a status code. */
CQ_API const char *cq_status_string(cq_status s);

/* Library version string. */
CQ_API const char *cq_version(void);

/*
 * cq_rotate_quantize -- fused online rotation + per-token absmax quantization.
 *
 * For each token m (row of x):
 *   x_rot = x[m,:] . (I_{K/b} (x) H_b), H_b[i][j] = (-1)^popcount(i & j)
 *           (Sylvester order, unnormalised, contiguous blocks of b = had_block)
 *   A     = max_k |x_rot[k]|
 *   q     = round_half_to_even(qmax * x_rot / A), qmax = 2^(act_bits-1) - 1,
 *           decided in exact arithmetic (the rotation of fp16 inputs is exact)
 *   s_out = (float)((A / sqrt(b)) / qmax)  (IEEE fp64 steps, then to fp32)
 *   A zero row gives q = 0 and s = 0.
 * Passages: CodeQuant abstract (rotation-based outlier smoothing of
 * activations); CodeQuant2 Tables 1, 2, 9 (A4W4 / A8W4 per-token codes).
 *
 * x       fp16 [M, K]
 * q_out   act_bits = 4: uint8 [M, K/2] packed int4; act_bits = 8: int8 [M, K]
 * s_out   fp32 [M]
 * Requires had_block a power of two in [1, 8192], K % had_block == 0,
 * K % 8 == 0, 1 <= K <= 16384 (else CQ_ERR_UNSUPPORTED), M >= 0 (M = 0 is a
 * no-op), act_bits in {4, 8}.
 */
CQ_API cq_status cq_rotate_quantize(const void *x, int64_t M, int64_t K, int32_t had_block,
                             int32_t act_bits, void *q_out, float *s_out, cq_stream_t stream);

/*
 * cq_rotate_quantize_ex -- cq_rotate_quantize with the online smoothing scale
 * and the channel grouping applied to x first:
 *   x'[m, j] = fp16( x[m, perm[j]] * scale[perm[j]] )   (round to nearest even
 *              of the exact product), then x' is rotated and quantized.
 * Passages: CodeQuant2 Figure 1 (rotation and scaling fused into the model)
 * and Table 5 (SmoothQuant scaling); CodeQuant podcast transcript, "Summary"
 * (the channels are reordered before clustering so that outliers spread over
 * different groups -- here, over different rotation blocks).
 *
 * scale   fp16 [K] per-channel multiplier (the reciprocals of the smoothing
 *         factors folded into the weights), or NULL for 1
 * perm    int32 [K], the order in which the weights' K columns are packed: a
 *         permutation of 0..K-1, or NULL for the identity.  A value outside
 *         [0, K) is clamped into range (nothing is read outside the row) and
 *         the result is then unspecified.
 * The scaled values must be finite (|x * scale| < 65520).  Other arguments,
 * requirements and errors as cq_rotate_quantize.
 */
CQ_API cq_status cq_rotate_quantize_ex(const void *x, int64_t M, int64_t K, int32_t had_block,
                                       int32_t act_bits, const void *scale, const int32_t *perm,
                                       void *q_out, float *s_out, cq_stream_t stream);

/*
 * cq_lut_gemm -- LUT (codebook) product of quantized activations with
 * 4-bit-index weights.
 *
 *   y[m,n] = s_x[m] * sum_k C[n, I[n,k]] * q[m,k]
 *   centroid_sums[m,n,c] = sum over k with I[n,k] = c of q[m,k]  (if non-NULL)
 * Passage: CodeQuant2 Figure 3 (codebook + assignment matrices) and Figure 4
 * (one-time LUT precompute, then lookups).  The codebook is expanded once per
 * row tile into lookup tables (register byte planes, or a byte-pair table in
 * shared memory); M <= 16 runs on mma.sync, larger M on the tcgen05 kernel
 * with the looked-up weights in tensor memory as the MMA's A operand.  q is
 * applied exactly (int codes as fp16) and the sum is accumulated in fp32.  Error bound per
 * output: |y - y_exact| <= 1e-4 * |s_x[m]| * sum_k |C[n,I[n,k]] q[m,k]| + 1e-6.
 *
 * q          codes as written by cq_rotate_quantize (act_bits 4: uint8 [M, K/2];
 *            8: int8 [M, K])
 * s_x        fp32 [M]
 * w_idx      uint8 [N, K/2] packed unsigned 4-bit indices
 * codebook   fp16 [N, 16]
 * y          fp32 [M, N] (written, not accumulated)
 * centroid_sums  int32 [M, N, 16] or NULL (parity / debug output; slow path)
 * workspace  scratch of at least cq_lut_gemm_workspace_size(M, N, K, act_bits)
 *            bytes (may be NULL when that size is 0).  Its contents on entry
 *            are ignored and on exit are undefined.
 * Requires K % 32 == 0, K >= 32, N % 64 == 0, act_bits in {4, 8}, M >= 0.
 */
CQ_API size_t cq_lut_gemm_workspace_size(int64_t M, int64_t N, int64_t K, int32_t act_bits);
CQ_API cq_status cq_lut_gemm(const void *q, const float *s_x, int64_t M, int64_t K, int32_t act_bits,
                      const uint8_t *w_idx, const void *codebook, int64_t N, float *y,
                      int32_t *centroid_sums, void *workspace, size_t workspace_bytes,
                      cq_stream_t stream);

/*
 * cq_lut_gemm_ex -- cq_lut_gemm with a per-layer codebook size: 2^idx_bits
 * centroids per output row, idx_bits in {3, 4, 5} (8, 16 or 32 centroids).
 * Passages: CodeQuant2 abstract (codebook sizes adapted to each layer's
 * quantization difficulty) and Figure 3 (adaptive cluster allocation).
 *
 *   y[m,n] = s_x[m] * sum_k C[n, I[n,k]] * q[m,k],   I[n,k] < 2^idx_bits
 *
 * w_idx      uint8 [N, K*idx_bits/8]: index k of row n occupies bits
 *            [idx_bits*k, idx_bits*k + idx_bits) of the row's byte string,
 *            least significant bit first (bit i of byte j is bit 8j + i).
 *            idx_bits = 4 is cq_lut_gemm's nibble format.
 * codebook   fp16 [N, 2^idx_bits]
 * idx_bits = 4 runs exactly cq_lut_gemm (same kernels, same results); 3 and 5
 * run a dedicated mma.sync kernel.  The error bound, the other arguments and
 * the requirements (K % 32 == 0, N % 64 == 0) are those of cq_lut_gemm; the
 * workspace is sized by cq_lut_gemm_ex_workspace_size.  Other idx_bits:
 * CQ_ERR_UNSUPPORTED.
 */
CQ_API size_t cq_lut_gemm_ex_workspace_size(int64_t M, int64_t N, int64_t K, int32_t act_bits,
                                            int32_t idx_bits);
CQ_API cq_status cq_lut_gemm_ex(const void *q, const float *s_x, int64_t M, int64_t K,
                                int32_t act_bits, const uint8_t *w_idx, int32_t idx_bits,
                                const void *codebook, int64_t N, float *y, void *workspace,
                                size_t workspace_bytes, cq_stream_t stream);

/*
 * cq_lut_gemm_noalloc -- cq_lut_gemm for callers that cannot allocate device
 * memory.  The pages have no counterpart: this is a deployment variant.
 *
 * Some callers can pass a kernel only its inputs and outputs: plugins and
 * custom-op hosts whose framework owns all device memory and exposes no
 * allocator, and serving processes that forbid cudaMalloc after start-up
 * because it synchronizes the device and fragments a pre-sized pool.  This
 * entry point runs exactly cq_lut_gemm's plan and kernels (so its results are
 * bitwise identical to cq_lut_gemm's for every shape it accepts), but keeps
 * the scratch -- the split-K partial sums and, on the tensor-memory kernels,
 * the fp16 copy of the codes -- in a fixed array of CQ_NOALLOC_SCRATCH_BYTES
 * bytes compiled into the library.  It calls no cudaMalloc / cudaFree and no
 * allocating library routine.
 *   - The array occupies CQ_NOALLOC_SCRATCH_BYTES of memory on every GPU that
 *     loads the library, until the process exits.
 *   - The first call on a device looks up the array's device address (once
 *     per device, under a lock) and keeps it; make that first call before any
 *     stream capture.  The kept address does not survive cudaDeviceReset: do
 *     not call this entry point again after resetting the device.
 *   - All calls share the array and it keeps the last call's contents; each
 *     call overwrites every scratch value it reads, so nothing needs clearing.
 *     Calls whose work overlaps on the GPU (other streams, other threads)
 *     race on the array and must be serialized by the caller.
 *   - A problem whose scratch needs more than CQ_NOALLOC_SCRATCH_BYTES (as
 *     cq_lut_gemm_workspace_size reports) returns CQ_ERR_UNSUPPORTED and
 *     enqueues nothing.
 * Arguments, layouts and the other checks are those of cq_lut_gemm (without
 * centroid_sums and workspace).
 */
#define CQ_NOALLOC_SCRATCH_BYTES (4u << 20)
CQ_API cq_status cq_lut_gemm_noalloc(const void *q, const float *s_x, int64_t M, int64_t K,
                                     int32_t act_bits, const uint8_t *w_idx,
                                     const void *codebook, int64_t N, float *y,
                                     cq_stream_t stream);

/*
 * MoE (or dense SwiGLU) FFN layer.
 *
 *   xq, s_x = rotate_quantize(x, had_block_h)              once per token
 *             (after the optional smoothing scale / channel order of w)
 *   routing: per token the top_k largest router logits (descending, ties to
 *            the lower expert id); weights = softmax over the selected logits
 *            (renormalize = 1) or over all E logits (renormalize = 0)
 *   per routed slot (t, j) with expert e, and per shared expert s for every t:
 *     g = LUT(xq[t], gate_e), u = LUT(xq[t], up_e)          N = I rows
 *     h = fp16(silu(g) * u)                                  round to nearest even
 *     hq, s_h = rotate_quantize(h, had_block_i)              per (t, e) row
 *     y = LUT(hq, down_e)                                     N = H rows
 *   out[t] = sum_{j < top_k} w[t,j] * y(t,j)  (j in order)  + sum_s y_s(t)
 * A dense SwiGLU FFN is E = 0, top_k = 0, n_shared = 1.
 * Passages: CodeQuant podcast transcript "Summary" (router and experts);
 * CodeQuant2 Figure 4 (LUT kernel per linear); the A4W4 / A8W4 settings of
 * CodeQuant2 Tables 1, 2, 9.
 *
 * Internal row order (used by the debug outputs): rows [0, T*top_k) are the
 * routed slots in `perm` order (grouped by expert, slot order inside a
 * group); row T*top_k + s*T + t is shared expert s for token t.
 */
typedef struct {
    int64_t H;            /* hidden size (input of gate/up, output of down) */
    int64_t I;            /* routed-expert intermediate size */
    int64_t E;            /* routed experts (0 = none) */
    int64_t top_k;        /* experts per token (0 when E = 0) */
    int64_t n_shared;     /* always-on shared experts (weight 1) */
    int64_t I_shared;     /* shared-expert intermediate size */
    int32_t act_bits;     /* 4 (A4W4) or 8 (A8W4) */
    int32_t had_block_h;  /* rotation block over H */
    int32_t had_block_i;  /* rotation block over I */
    int32_t had_block_i_shared; /* rotation block over I_shared */
    int32_t renormalize;  /* 1: softmax over the selected logits */
} cq_moe_desc;

typedef struct {
    const uint8_t *gate_idx;     /* [E, I, H/2] */
    const uint8_t *up_idx;       /* [E, I, H/2] */
    const uint8_t *down_idx;     /* [E, H, I/2] */
    const void *gate_cb;         /* fp16 [E, I, 16] */
    const void *up_cb;           /* fp16 [E, I, 16] */
    const void *down_cb;         /* fp16 [E, H, 16] */
    const uint8_t *sh_gate_idx;  /* [n_shared, I_shared, H/2] */
    const uint8_t *sh_up_idx;    /* [n_shared, I_shared, H/2] */
    const uint8_t *sh_down_idx;  /* [n_shared, H, I_shared/2] */
    const void *sh_gate_cb;      /* fp16 [n_shared, I_shared, 16] */
    const void *sh_up_cb;        /* fp16 [n_shared, I_shared, 16] */
    const void *sh_down_cb;      /* fp16 [n_shared, H, 16] */
    /* online smoothing scale and channel order of the layer input x, as in
     * cq_rotate_quantize_ex (NULL: none); the gate/up weights' H columns are
     * packed in the order x_perm gives */
    const void *x_scale;         /* fp16 [H] or NULL */
    const int32_t *x_perm;       /* int32 [H] or NULL */
} cq_moe_weights;

/* Optional copies of intermediate results (any field may be NULL).
 * R = T*top_k + n_shared*T rows; I_r = I for routed rows, I_shared for shared
 * rows (a row of h / h_codes has the width of its own expert; rows are packed
 * with the larger width max(I, I_shared) as the stride). */
typedef struct {
    int32_t *topk_ids;   /* [T, top_k] */
    float *topk_w;       /* [T, top_k] */
    int32_t *counts;     /* [E] */
    int32_t *offsets;    /* [E + 1] */
    int32_t *perm;       /* [T*top_k]  slot t*top_k + j listed in row order */
    void *x_codes;       /* codes of x, as cq_rotate_quantize writes them */
    float *x_scales;     /* [T] */
    void *h;             /* fp16 [R, Imax] */
    void *h_codes;       /* codes of h, row stride Imax (int4: Imax/2 bytes) */
    float *h_scales;     /* [R] */
    float *y_rows;       /* fp32 [R, H]  down-projection output per row (scaled) */
} cq_moe_debug;

CQ_API size_t cq_moe_ffn_workspace_size(const cq_moe_desc *d, int64_t T);

/*
 * x       fp16 [T, H]
 * router_logits fp32 [T, E] (NULL iff E = 0)
 * out     fp32 [T, H]
 * dbg     NULL or a cq_moe_debug with device pointers to fill
 * Requires H % 64 == 0, I % 64 == 0, I_shared % 64 == 0 (when used),
 * H, I <= 16384, 1 <= top_k <= min(E, 16) when E > 0, E <= 256, n_shared <= 4,
 * had blocks powers of two dividing their dimension, act_bits in {4, 8}.
 */
CQ_API cq_status cq_moe_ffn(const cq_moe_desc *d, const void *x, const float *router_logits, int64_t T,
                     const cq_moe_weights *w, void *workspace, size_t workspace_bytes,
                     float *out, const cq_moe_debug *dbg, cq_stream_t stream);

/*
 * Measurement aids (not part of the layer's computation).
 *
 * cq_launch_count   number of kernels this library has launched since it was
 *                   loaded (process-wide).
 * cq_timing_enable  on = 1: every LUT GEMM kernel launch is bracketed by two
 *                   CUDA events on its stream; on = 2: every launch of the
 *                   library (LUT GEMMs, rotate-quantize, routing, combine,
 *                   code conversion, reductions); on = 0 stops recording.
 * cq_timing_read    waits for the recorded events, returns the number of timed
 *                   launches and their summed device time in ms, and clears
 *                   the record.  Returns CQ_ERR_CUDA if an event failed.
 * cq_timing_read_launches
 *                   the same record launch by launch, in launch order: for the
 *                   first min(*n, cap) launches, kinds[i] (CQ_KERNEL_*: which
 *                   kernel ran) and ms[i] (device time; -1 if its
 *                   events failed, and the call then returns CQ_ERR_CUDA).
 *                   *n = number of recorded launches.  Host arrays of cap
 *                   entries, owned by the caller (NULL allowed when cap = 0).
 *                   Clears the record.
 * The timing record is the one piece of process-wide state in the library;
 * it is guarded by a mutex.  Enable it only around single-threaded use.
 */
enum cq_kernel_kind {
    CQ_KERNEL_LUT_MMA = 0, /* mma.sync kernel, register / shared lookup tables */
    CQ_KERNEL_LUT_TC = 1,  /* tcgen05 kernel for wide token tiles (> 32 rows per group) */
    CQ_KERNEL_LUT_TS = 2,  /* tcgen05 decode kernel (<= 32 rows per group): pair tables */
    CQ_KERNEL_LUT_VB = 3,  /* mma.sync kernel for 3- / 5-bit indices (cq_lut_gemm_ex) */
    /* recorded with cq_timing_enable(2) only */
    CQ_KERNEL_ROTATE_QUANTIZE = 4, /* rotation + quantization of x or h (SwiGLU fused) */
    CQ_KERNEL_CODES_F16 = 5,       /* activation codes -> fp16 B operand rows */
    CQ_KERNEL_ROUTE = 6,           /* router top-k and expert grouping (two kernels) */
    CQ_KERNEL_COMBINE = 7,         /* weighted sum of expert outputs */
    CQ_KERNEL_REDUCE = 8,          /* split-K partial sums -> y */
    CQ_KERNEL_CENTROID_SUMS = 9    /* per-centroid integer sums */
};
CQ_API int64_t cq_launch_count(void);

/*
 * cq_device_error -- the device error word: 0 if no kernel of this library
 * stopped early since the last call, else a nonzero code (1 = a bounded wait
 * inside a tensor-core kernel gave up; its outputs are then unspecified).
 * Synchronizes the current device and clears the word; -1 if it could not be
 * read.
 */
CQ_API int32_t cq_device_error(void);

/*
 * cq_selftest_wait_timeout -- runs one kernel whose bounded wait can never be
 * satisfied (an mbarrier nothing arrives on): it gives up after about one
 * second, sets the device error word to 1 and returns, leaving the context
 * usable.  Exercises the error path of the tensor-core kernels' waits for
 * tests.  Asynchronous on stream; CQ_ERR_CUDA if the launch failed.
 */
CQ_API cq_status cq_selftest_wait_timeout(cq_stream_t stream);
CQ_API cq_status cq_timing_enable(int32_t on);
CQ_API cq_status cq_timing_read(int64_t *launches, double *total_ms);
CQ_API cq_status cq_timing_read_launches(int32_t *kinds, float *ms, int64_t cap, int64_t *n);

#ifdef __cplusplus
}
#endif

#endif /* CQ_H_ */
