// awq_search.cu -- kernels of the AWQ scale search (offline, before quantization).
//
// AWQ divides each input channel of W by an activation magnitude s before
// quantizing and multiplies it back after, W^ = quant(W / s) * s, with s taken
// from calibration statistics (ch. 22 "Advanced inference optimisation",
// section 22.3, AWQ).  The layer-output error of a quantized weight matrix on
// calibration activations X is || X W^T - X W^^T ||_F^2 (same section, the
// objective given for GPTQ).  The search here takes the per-channel mean
// magnitude m_k = mean_rows |x_k| of X, tries s = m^a for each exponent a of
// a grid, and keeps the one with the smallest output error.
//
// Kernels: the fp64 column mean of |X| (exact for 16-bit inputs), the
// per-exponent scale, a plain fp32 dense GEMM for the reference X W^T (run once
// per search), and a fixed-order fp64 sum of squared differences.
#include "common.cuh"

namespace w4 {
namespace awq_impl {

// m[k] = (sum over the Mc rows of |x[r][k]|) / Mc, summed in fp64 in row order.
// The sum of Mc 16-bit magnitudes is exact in fp64 for any realistic Mc, so the
// result does not depend on the order.
template <bool kBf16>
__global__ void __launch_bounds__(256) mean_abs_kernel(const uint16_t *__restrict__ X, int64_t Mc, int64_t K,
                                                       double *__restrict__ m) {
  const int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= K) return;
  double acc = 0.0;
  for (int64_t r = 0; r < Mc; ++r) {
    const uint16_t b = X[r * K + k];
    const float v = kBf16 ? __uint_as_float((uint32_t)b << 16) : __half2float(__ushort_as_half(b));
    acc += (double)fabsf(v);
  }
  m[k] = acc / (double)Mc;
}

// s[k] = m[k]^a rounded to fp32 (computed in fp64), 1 where m[k] = 0.
__global__ void __launch_bounds__(256) scale_kernel(const double *__restrict__ m, int64_t K, double a,
                                                    float *__restrict__ s) {
  const int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= K) return;
  const double v = m[k];
  s[k] = v > 0.0 ? (float)pow(v, a) : 1.0f;
}

// Yref[r][n] = sum_k x[r][k] * w[n][k] in fp32: 64 x 64 output tiles, k in
// steps of 32 through shared memory, 4 x 4 outputs per thread.
constexpr int kT = 64, kKT = 32;
template <bool kBf16>
__global__ void __launch_bounds__(256) dense_ref_kernel(const uint16_t *__restrict__ X, const float *__restrict__ W,
                                                        int64_t Mc, int64_t N, int64_t K, float *__restrict__ Y) {
  __shared__ float xs[kKT][kT + 1];
  __shared__ float ws[kKT][kT + 1];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int64_t r0 = (int64_t)blockIdx.y * kT, n0 = (int64_t)blockIdx.x * kT;
  float acc[4][4] = {};
  for (int64_t k0 = 0; k0 < K; k0 += kKT) {
    for (int i = threadIdx.x; i < kT * kKT; i += 256) {
      const int row = i / kKT, kk = i % kKT;
      const int64_t r = r0 + row, n = n0 + row, k = k0 + kk;
      float xv = 0.0f, wv = 0.0f;
      if (r < Mc && k < K) {
        const uint16_t b = X[r * K + k];
        xv = kBf16 ? __uint_as_float((uint32_t)b << 16) : __half2float(__ushort_as_half(b));
      }
      if (n < N && k < K) wv = W[n * K + k];
      xs[kk][row] = xv;
      ws[kk][row] = wv;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < kKT; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = xs[kk][ty + 16 * i];
        b[i] = ws[kk][tx + 16 * i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t r = r0 + ty + 16 * i, n = n0 + tx + 16 * j;
      if (r < Mc && n < N) Y[r * N + n] = acc[i][j];
    }
}

constexpr int kErrBlocks = 256;

// partial[b] = sum over a fixed strided subset of (a - b)^2, fp64, fixed order.
__global__ void __launch_bounds__(256) sq_err_partial_kernel(const float *__restrict__ A, const float *__restrict__ B,
                                                             int64_t count, double *__restrict__ partial) {
  __shared__ double red[256];
  double acc = 0.0;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count; i += (int64_t)gridDim.x * blockDim.x) {
    const double d = (double)A[i] - (double)B[i];
    acc = fma(d, d, acc);
  }
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int o = 128; o > 0; o >>= 1) {
    if (threadIdx.x < o) red[threadIdx.x] += red[threadIdx.x + o];
    __syncthreads();
  }
  if (threadIdx.x == 0) partial[blockIdx.x] = red[0];
}

// out = sum of the kErrBlocks partials in index order (one thread).
__global__ void sq_err_final_kernel(const double *__restrict__ partial, double *__restrict__ out) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  double acc = 0.0;
  for (int i = 0; i < kErrBlocks; ++i) acc += partial[i];
  *out = acc;
}

}  // namespace awq_impl

cudaError_t launch_mean_abs(const void *X, bool x_bf16, int64_t Mc, int64_t K, double *m, cudaStream_t stream) {
  const int grid = (int)((K + 255) / 256);
  if (x_bf16) awq_impl::mean_abs_kernel<true><<<grid, 256, 0, stream>>>(static_cast<const uint16_t *>(X), Mc, K, m);
  else awq_impl::mean_abs_kernel<false><<<grid, 256, 0, stream>>>(static_cast<const uint16_t *>(X), Mc, K, m);
  return cudaGetLastError();
}

cudaError_t launch_awq_scale(const double *m, int64_t K, double a, float *s, cudaStream_t stream) {
  awq_impl::scale_kernel<<<(int)((K + 255) / 256), 256, 0, stream>>>(m, K, a, s);
  return cudaGetLastError();
}

cudaError_t launch_dense_ref(const void *X, bool x_bf16, const float *W, int64_t Mc, int64_t N, int64_t K, float *Y,
                             cudaStream_t stream) {
  const dim3 grid((unsigned)((N + awq_impl::kT - 1) / awq_impl::kT), (unsigned)((Mc + awq_impl::kT - 1) / awq_impl::kT));
  if (x_bf16)
    awq_impl::dense_ref_kernel<true><<<grid, 256, 0, stream>>>(static_cast<const uint16_t *>(X), W, Mc, N, K, Y);
  else
    awq_impl::dense_ref_kernel<false><<<grid, 256, 0, stream>>>(static_cast<const uint16_t *>(X), W, Mc, N, K, Y);
  return cudaGetLastError();
}

// err = sum (A - B)^2 over count elements; partial needs kErrBlocks doubles.
cudaError_t launch_sq_err(const float *A, const float *B, int64_t count, double *partial, double *err,
                          cudaStream_t stream) {
  awq_impl::sq_err_partial_kernel<<<awq_impl::kErrBlocks, 256, 0, stream>>>(A, B, count, partial);
  awq_impl::sq_err_final_kernel<<<1, 32, 0, stream>>>(partial, err);
  return cudaGetLastError();
}

}  // namespace w4
