/*
 * w4.h -- C ABI of libw4: weight-only, per-group INT4 (W4A16) linear layers
 * on NVIDIA B200 (sm_100a).
 *
 * What is computed (sources cited by page and section):
 *   - Quantization maps a float range onto integers through a scale and a
 *     zero point, per group of 128 elements ("LLM inference acceleration"
 *     article, discosf.com, section 2.1).  Here: asymmetric uint4 codes in
 *     [0,15], one fp16 scale and one fp16 zero point per group of G = 128
 *     consecutive input channels k of an output row n.
 *   - Weight-only quantization: the weights are dequantized back to 16-bit and
 *     multiplied by 16-bit activations, or a mixed-precision kernel does both
 *     at once (aiwing.uk ch. 22 "Advanced inference optimisation", section
 *     22.3 "Model quantization").  w4a16_gemm is that fused kernel.
 *   - AWQ: weights are divided by a per-input-channel activation magnitude s
 *     before quantization and multiplied back after, W^ = quant(W/s) * s
 *     (ch. 22, section 22.3, AWQ equation).
 *   - Scale and zero point travel with the packed weights as one unit
 *     (article section 2.3); INT4 takes 0.5 byte per parameter (ch. 22,
 *     section 22.3 table).
 *
 * Exact rule (the pages leave it open; this is the library's definition):
 *   w'    = s ? w / s[k] : w                         (fp32, IEEE division)
 *   mn,mx = min, max of w' over the group
 *   scale = fp16_rn((mx - mn) / 15), taken as 1.0 if that is 0
 *   z     = clamp(rint(-mn / scale), 0, 15)          (fp32, ties to even)
 *   q     = clamp(rint(w' / scale) + z, 0, 15)
 *   packed byte j of a row = q[2j] | q[2j+1] << 4    (low nibble = even k)
 *   W^[n][k] = (q - z) * scale * (s ? s[k] : 1)
 *   Y[m][n]  = sum_k X[m][k] * W^[n][k]               (fp32 accumulation)
 *
 * Layouts (all row-major, all buffers owned by the caller):
 *   W       [N][K]   fp32, fp16 or bf16          (quantize input)
 *   awq_s   [K]      fp32, > 0, or NULL
 *   packed  [N][K/2] uint8
 *   scales  [N][K/G] IEEE binary16 bit patterns
 *   zeros   [N][K/G] IEEE binary16 bit patterns (integers 0..15)
 *   codes   [N][K]   uint8, one code per byte (optional quantize output)
 *   X       [M][K]   fp16 or bf16
 *   Y       [M][N]   fp32 or bf16
 *
 * Conventions:
 *   - Device pointers are device memory of the current CUDA device; every
 *     device pointer must be 16-byte aligned.  The library allocates nothing.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream) and never synchronize the device, except the
 *     host-buffer entry point, which waits for its own stream.
 *   - Arguments are validated on the host before anything is launched; a
 *     failed check returns W4_ERR_INVALID_ARG or W4_ERR_UNSUPPORTED and
 *     launches nothing.  A CUDA launch error returns W4_ERR_CUDA.
 *     w4_last_error() gives a message for the last failure on this thread.
 *   - Non-finite weights give unspecified codes.
 *   - Thread-safe: no global state is written on the host except the
 *     per-thread error message and a per-device cache of driver entry points.
 */
#ifndef W4_H_
#define W4_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  W4_OK = 0,
  W4_ERR_INVALID_ARG = 1, /* bad size, null or misaligned pointer, short workspace */
  W4_ERR_UNSUPPORTED = 2, /* valid but not served: group not 32/64/128, dtype combination */
  W4_ERR_CUDA = 3         /* a CUDA call or kernel launch failed */
} w4_status;

typedef enum { W4_F32 = 0, W4_F16 = 1, W4_BF16 = 2 } w4_dtype;

/* Same type as cudaStream_t, declared here so this header needs no CUDA headers. */
typedef struct CUstream_st *w4_stream_t;

/*
 * Quantize and pack W (the whole a1..a5 path in one kernel launch).
 *   W        device [N][K], dtype w_dtype (F32, F16 or BF16)
 *   awq_s    device [K] fp32 or NULL (no AWQ)
 *   N, K     N >= 1, K >= 1, K % group == 0
 *   group    128; 32 and 64 are also served (scales, zeros [N][K/group])
 *   packed   device [N][K/2] out; scales, zeros device [N][K/group] out
 *   codes    device [N][K] out, or NULL (unpacked codes, a test aid)
 * Outputs match the rule above bit for bit.
 */
w4_status w4_quantize(const void *W, w4_dtype w_dtype, const float *awq_s,
                      int64_t N, int64_t K, int group, uint8_t *packed,
                      uint16_t *scales, uint16_t *zeros, uint8_t *codes,
                      w4_stream_t stream);

/*
 * Symmetric variant of w4_quantize: INT4 as the symmetric value set
 * {-7, ..., 7} (mhpq.cn practitioner's article, section 2.1).  Per group:
 *   amax = max |w'|;  scale = fp16(amax / 7), 1.0 if that is 0;
 *   q = clamp(rint(w' / scale), -7, 7);  stored code = q + 8 (1..15), zero = 8.
 * The outputs have the same layout as w4_quantize's (every zero is 8.0), so
 * w4a16_gemm consumes them unchanged: (code - 8) * scale = q * scale.
 * Arguments and errors as for w4_quantize.
 */
w4_status w4_quantize_symmetric(const void *W, w4_dtype w_dtype,
                                const float *awq_s, int64_t N, int64_t K,
                                int group, uint8_t *packed, uint16_t *scales,
                                uint16_t *zeros, uint8_t *codes,
                                w4_stream_t stream);

/*
 * Pack one-code-per-byte codes [N][K] (device) into packed [N][K/2]
 * (device): two 4-bit codes per byte, 0.5 byte per parameter (ch. 22,
 * section 22.3 table); low nibble = even k.  Values above 15 are masked to
 * 4 bits.  K must be a positive multiple of 32.
 */
w4_status w4_pack(const uint8_t *codes, int64_t N, int64_t K, uint8_t *packed,
                  w4_stream_t stream);

/*
 * Fused dequantize-matmul Y = X . W^T (a6..a7).
 *   X         device [M][K], x_dtype F16 or BF16
 *   M, N, K   >= 1; K % group == 0
 *   group     the group given to w4_quantize: 128, or 32 / 64 (then K must be
 *             a multiple of 64, and the tensor-core kernel serves every M)
 *   packed, scales, zeros   as produced by w4_quantize
 *   awq_s     device [K] fp32, the SAME vector given to w4_quantize, or NULL
 *   Y         device [M][N], y_dtype F32 or BF16 (overwritten)
 *   workspace device scratch of at least w4a16_gemm_workspace_size(M,N,K)
 *             bytes (may be NULL when that size is 0).  It must be zero-filled
 *             once before its first use.  Every call leaves its first 128 KiB
 *             (tile arrival counters) zero again; the bytes after them hold
 *             partial sums that each call writes before it reads them.  Calls
 *             that share a workspace must not overlap in time.
 * Accuracy: |Y - Y_exact| <= 2e-3 * sum_k |X[m][k] * W^[n][k]| per element on
 * the library's test distributions (fp32 accumulation; the prefill path rounds
 * W^ to 16 bits once, the decode path keeps (q - z) exact and, with AWQ,
 * rounds x * s to fp16 once).
 */
w4_status w4a16_gemm(const void *X, w4_dtype x_dtype, int64_t M, int64_t N,
                     int64_t K, int group, const uint8_t *packed,
                     const uint16_t *scales, const uint16_t *zeros,
                     const float *awq_s, void *Y, w4_dtype y_dtype,
                     void *workspace, size_t workspace_bytes,
                     w4_stream_t stream);

/*
 * Bytes of workspace w4a16_gemm needs for this shape (0 if none): split-K
 * counters and fp32 partials of the fused dequantize-matmul (ch. 22, section
 * 22.3).  Covers every plan the call may take for (M, N, K), with or without
 * AWQ, for groups of 32, 64 or 128; 0 also for invalid sizes.
 */
size_t w4a16_gemm_workspace_size(int64_t M, int64_t N, int64_t K);

/*
 * End-to-end variant with HOST activations and outputs: copies X_host
 * (pinned host memory, [M][K]) into X_dev, runs w4a16_gemm, copies Y_dev
 * back into Y_host (pinned host memory, [M][N]) and waits for `stream`.
 * X_dev and Y_dev are caller-owned device staging buffers of the same sizes.
 * The computation is w4a16_gemm's (ch. 22, section 22.3); the stream wait
 * inside every call makes Y_host valid on return.
 */
w4_status w4a16_gemm_host(const void *X_host, void *X_dev, w4_dtype x_dtype,
                          int64_t M, int64_t N, int64_t K, int group,
                          const uint8_t *packed, const uint16_t *scales,
                          const uint16_t *zeros, const float *awq_s,
                          void *Y_host, void *Y_dev, w4_dtype y_dtype,
                          void *workspace, size_t workspace_bytes,
                          w4_stream_t stream);

/*
 * The same without the wait: the copy of X_host, the matmul and the copy back
 * into Y_host are enqueued on `stream` and the call returns; Y_host is valid
 * once the caller has synchronized `stream` (ch. 22, section 22.3, as for
 * w4a16_gemm).  A decode step of several layers then waits once per step
 * instead of once per layer.  X_host and Y_host must stay valid and unchanged
 * (X_host) or unread (Y_host) until the stream reaches the copies.  Errors:
 * as for w4a16_gemm_host; failures of the enqueued work surface at the
 * caller's synchronization.
 */
w4_status w4a16_gemm_host_async(const void *X_host, void *X_dev, w4_dtype x_dtype,
                                int64_t M, int64_t N, int64_t K, int group,
                                const uint8_t *packed, const uint16_t *scales,
                                const uint16_t *zeros, const float *awq_s,
                                void *Y_host, void *Y_dev, w4_dtype y_dtype,
                                void *workspace, size_t workspace_bytes,
                                w4_stream_t stream);

/*
 * One matmul of a host-buffer batch (w4a16_gemm_host_batch_async): the
 * arguments of w4a16_gemm, with X and Y given as byte offsets into the batch's
 * staging buffers instead of as pointers.
 */
typedef struct {
  int64_t M, N, K;
  int group;
  w4_dtype x_dtype;        /* F16 or BF16 */
  w4_dtype y_dtype;        /* F32 or BF16 */
  const uint8_t *packed;   /* device, as produced by w4_quantize */
  const uint16_t *scales;  /* device */
  const uint16_t *zeros;   /* device */
  const float *awq_s;      /* device [K] or NULL */
  size_t x_offset;         /* bytes into X_host / X_dev, a multiple of 16 */
  size_t y_offset;         /* bytes into Y_host / Y_dev, a multiple of 16 */
} w4_gemm_item;

/*
 * Several independent fused dequantize-matmuls with host activations and
 * outputs, in one call (ch. 22, section 22.3, as for w4a16_gemm): one copy of
 * X_host[0, x_bytes) into X_dev, then items[0..count) in order on `stream` (item
 * i reads [M][K] at X_dev + x_offset and writes [M][N] at Y_dev + y_offset), then
 * one copy of Y_dev[0, y_bytes) into Y_host.  Nothing waits: Y_host is valid once
 * the caller has synchronized `stream`.  A step of independent layers (projections
 * with separate weights, experts) then pays two copies and one wait in all.
 *   X_host, Y_host   HOST, pinned for asynchronous copies; unchanged (X_host) and
 *                    unread (Y_host) until the stream reaches the copies
 *   X_dev, Y_dev     device staging buffers of x_bytes and y_bytes
 *   workspace        as for w4a16_gemm, at least the largest
 *                    w4a16_gemm_workspace_size of the items; the items run one
 *                    after another, so they share it
 *   count            1 .. 4096
 * Errors: every item is checked (shape, dtypes, offsets 16-byte aligned and
 * inside x_bytes / y_bytes, pointers, workspace size) before anything is
 * enqueued; W4_ERR_INVALID_ARG or W4_ERR_UNSUPPORTED then names the item in
 * w4_last_error().  Failures of the enqueued work surface at the caller's
 * synchronization.
 */
w4_status w4a16_gemm_host_batch_async(const w4_gemm_item *items, int count,
                                      const void *X_host, void *X_dev,
                                      size_t x_bytes, void *Y_host, void *Y_dev,
                                      size_t y_bytes, void *workspace,
                                      size_t workspace_bytes,
                                      w4_stream_t stream);

/*
 * AWQ scale search (offline, before w4_quantize).  AWQ quantizes W / s and
 * multiplies back by s, with s a per-input-channel activation magnitude from
 * calibration data (ch. 22 "Advanced inference optimisation", section 22.3);
 * a quantized layer is judged by its output error || X W^T - X W^^T ||_F^2 on
 * calibration activations X (same section).  Here s = m^a with
 * m_k = mean over the calibration rows of |x_k| (fp64; s = 1 where m_k = 0),
 * and a is the exponent of `alphas` with the smallest error (the first on ties).
 *   W         device [N][K] fp32 (the dense weights)
 *   Xcal      device [Mc][K] F16 or BF16 calibration activations
 *   group     32, 64 or 128 (as for w4_quantize)
 *   alphas    HOST array of 1..256 finite exponents (negative ones protect the
 *             channels with large activations: W / s is then larger there)
 *   awq_s     device [K] fp32 out: s for the best exponent, to be given to
 *             w4_quantize and w4a16_gemm
 *   errors    HOST [n_alpha] out (fp64 output error per exponent), or NULL
 *   best      HOST out: index of the best exponent
 *   workspace device scratch of w4_awq_search_workspace_size(Mc, N, K, group)
 *             bytes, zero-filled before its first use (it holds a w4a16_gemm
 *             workspace, whose counters every call leaves zero).
 * Runs the quantizer and w4a16_gemm once per exponent and a dense fp32
 * reference GEMM once; synchronizes `stream` before returning.
 */
w4_status w4_awq_search(const float *W, int64_t N, int64_t K, int group,
                        const void *Xcal, w4_dtype x_dtype, int64_t Mc,
                        const float *alphas, int n_alpha, float *awq_s,
                        double *errors, int *best, void *workspace,
                        size_t workspace_bytes, w4_stream_t stream);

/* Bytes of workspace w4_awq_search needs (0 for invalid sizes). */
size_t w4_awq_search_workspace_size(int64_t Mc, int64_t N, int64_t K,
                                    int group);

/*
 * Dense + sparse split (mhpq.cn practitioner's article, section 2.2: the top
 * 0.1% of weights by magnitude stay in FP16, the rest go to INT4).  The sparse
 * part holds every weight with |w| >= tau, tau = the count-th largest |w| of the
 * matrix (ties at tau are all kept), as fp16.  The dense part is quantized as
 * by w4_quantize with those weights taken as 0, so their dequantized value is
 * exactly 0 and  W^ = dequant(dense) + sparse.
 *   W         device [N][K] fp32 (N*K < 2^31)
 *   awq_s, group, packed, scales, zeros   as for w4_quantize
 *   count     1 <= count <= N*K, or 0 for w4_outliers_default_count(N, K)
 *   row_ptr   device [N+1] int32 out: CSR row offsets by output row
 *   col, val  device [capacity] int32 / fp16 bit patterns out: the entries of
 *             each row in increasing k
 *   nnz       HOST out: entries found (count, more with ties at tau)
 *   workspace device, w4_outliers_workspace_size(N) bytes, zero-filled before
 *             its first use (every call leaves it so)
 * If capacity < nnz, returns W4_ERR_INVALID_ARG with nnz set (col / val then
 * hold the first `capacity` entries).  Synchronizes `stream`.
 */
w4_status w4_quantize_outliers(const float *W, const float *awq_s, int64_t N,
                               int64_t K, int group, int64_t count,
                               uint8_t *packed, uint16_t *scales,
                               uint16_t *zeros, int32_t *row_ptr,
                               int32_t *col, uint16_t *val, int64_t capacity,
                               int64_t *nnz, void *workspace,
                               size_t workspace_bytes, w4_stream_t stream);

/* Bytes of workspace w4_quantize_outliers needs for N rows (radix-select
 * histograms and per-row counts of the split of the mhpq.cn article, 2.2). */
size_t w4_outliers_workspace_size(int64_t N);

/*
 * Default outlier count of the dense + sparse split: the top 0.1 % of the
 * weights (mhpq.cn practitioner's article, section 2.2), ceil(N * K / 1000),
 * at least 1 (0 for invalid sizes).  w4_quantize_outliers uses it when given
 * count = 0.
 */
int64_t w4_outliers_default_count(int64_t N, int64_t K);

/*
 * w4a16_gemm on the dense part, then the sparse part added to Y:
 * y[m][n] += sum over row n's entries of x[m][col] * val (fp32, entry order).
 * Arguments as for w4a16_gemm, plus the CSR from w4_quantize_outliers.
 */
w4_status w4a16_gemm_outliers(const void *X, w4_dtype x_dtype, int64_t M,
                              int64_t N, int64_t K, int group,
                              const uint8_t *packed, const uint16_t *scales,
                              const uint16_t *zeros, const float *awq_s,
                              const int32_t *row_ptr, const int32_t *col,
                              const uint16_t *val, void *Y, w4_dtype y_dtype,
                              void *workspace, size_t workspace_bytes,
                              w4_stream_t stream);

/*
 * GPTQ quantization (ch. 22 "Advanced inference optimisation", section 22.3:
 * quantize W so as to minimize || W X - W^ X ||_F^2 on calibration inputs,
 * the Hessian H = 2 X X^T deciding how each weight's quantization error is
 * compensated on the weights not yet quantized).  The column sweep, in fp64
 * with a fixed order of operations:
 *   H = 2 Xcal^T Xcal, plus damp_frac * trace(H) / K on the diagonal;
 *   U = upper Cholesky factor of H^-1;
 *   per row, k = 0..K-1: at each group start, scale and zero from the current
 *   weights by the rule of w4_quantize; q = code of the current weight;
 *   err = (w - w^) / U[k][k];  w[k'] -= err * U[k][k'] for k' > k.
 *   W         device [N][K] fp32 (left unchanged)
 *   Xcal      device [Mc][K] F16 or BF16 calibration activations
 *   group     32, 64 or 128; K a multiple of 32 and at most 32768
 *   damp_frac >= 0 (0.01 is usual)
 *   packed, scales, zeros, codes   as for w4_quantize (codes may be NULL)
 *   workspace device, w4_gptq_workspace_size(N, K) bytes (3 K^2 + N K doubles)
 * The outputs are consumed by w4a16_gemm like those of w4_quantize.  Returns
 * W4_ERR_INVALID_ARG if the damped Hessian is not positive definite.
 * Synchronizes `stream`.
 */
w4_status w4_quantize_gptq(const float *W, int64_t N, int64_t K, int group,
                           const void *Xcal, w4_dtype x_dtype, int64_t Mc,
                           double damp_frac, uint8_t *packed,
                           uint16_t *scales, uint16_t *zeros, uint8_t *codes,
                           void *workspace, size_t workspace_bytes,
                           w4_stream_t stream);

/* Bytes of workspace w4_quantize_gptq needs (0 for invalid sizes). */
size_t w4_gptq_workspace_size(int64_t N, int64_t K);

/*
 * Decode GEMM with library-owned scratch: the same computation and result as
 * w4a16_gemm for decode shapes, with no workspace argument.  The source pages
 * have no counterpart to this call; it exists for callers that cannot allocate
 * device memory where they run the layer (an engine plugin with no allocator of
 * its own, a loop that must not take cudaMalloc).
 *   Arguments as for w4a16_gemm.  M <= 64, else W4_ERR_UNSUPPORTED.
 *   Scratch: a fixed array of w4a16_gemm_decode_static_capacity() bytes
 *   (8 MiB) per device, part of the library's own module.  A tensor-core plan
 *   takes fewer K splits where its fp32 partials would not fit it, and a
 *   decode-kernel plan whose k-slice partials would not fit is replaced by that
 *   tensor-core plan, so every M <= 64 shape is served.  (With the decode
 *   kernel forced through W4_FORCE_PATH=gemv, such a plan returns
 *   W4_ERR_UNSUPPORTED with the sizes in w4_last_error() and launches nothing.)
 *   The first call in a CUDA context looks up the scratch address there (the
 *   device must be current); make it before any stream capture.  A context that
 *   is destroyed and created again (cudaDeviceReset) gets a fresh lookup.
 *   The scratch starts zero-filled and every completed call leaves its
 *   counters at zero.  Calls on one device share it: calls that overlap in
 *   time (other streams or threads) race on it and give wrong results.
 */
w4_status w4a16_gemm_decode_static(const void *X, w4_dtype x_dtype, int64_t M,
                                   int64_t N, int64_t K, int group,
                                   const uint8_t *packed,
                                   const uint16_t *scales,
                                   const uint16_t *zeros, const float *awq_s,
                                   void *Y, w4_dtype y_dtype,
                                   w4_stream_t stream);

/* Bytes of the static scratch behind w4a16_gemm_decode_static. */
size_t w4a16_gemm_decode_static_capacity(void);

/*
 * Device-side error word: kernels whose bounded waits run out set it instead
 * of hanging.  Copies its value to *flag (0 = no error) and clears it; this
 * call synchronizes the current device.  Library error reporting: the pages
 * define no counterpart.
 */
w4_status w4_device_error(int *flag);

/* Human-readable name of a status code (static string).  Library error
 * reporting: the pages define no counterpart. */
const char *w4_status_string(w4_status status);

/* Message of the last failed call on this thread ("" if none), naming the
 * argument or CUDA call that failed.  Library error reporting: the pages define
 * no counterpart. */
const char *w4_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* W4_H_ */
