// outliers.cu -- dense + sparse split of a weight matrix (mhpq.cn practitioner's
// article, section 2.2: the top 0.1% of weights by magnitude are kept in FP16,
// the rest are quantized to INT4, W^ = where(mask, fp16(w), int4 dequant)).
//
//   * Threshold: tau = the k-th largest |w| over the whole matrix, found by a
//     three-pass radix select on the 31 bits of |w| (11 + 11 + 9; for
//     non-negative floats the bit patterns order like the values).  The mask is
//     |w| >= tau, so ties at tau are all kept.
//   * The dense part is quantized with the masked weights replaced by 0 (see
//     quantize.cu); their dequantized value is then exactly 0, since a zero
//     weight gets the code z.
//   * The sparse part is CSR by output row: column indices in increasing k and
//     fp16 values, built by one warp per row (deterministic order).
//   * The GEMM adds it afterwards: y[m][n] += sum_j x[m][col_j] * val_j.
#include "common.cuh"

namespace w4 {
namespace outlier_impl {

constexpr int kBins = 2048;  // per radix pass

// state[0] = bits fixed so far (a prefix of tau's bit pattern), state[1] = the
// rank still wanted among the elements matching that prefix (1-based),
// state[2] = how many bits are fixed.
__device__ __forceinline__ uint32_t abs_bits(float v) { return __float_as_uint(v) & 0x7FFFFFFFu; }

__global__ void state_init_kernel(uint32_t *state, uint32_t count) {
  if (threadIdx.x == 0 && blockIdx.x == 0) {
    state[0] = 0u;
    state[1] = count;
    state[2] = 0u;
  }
}

// Histogram of the next `width` bits below the fixed prefix, over elements that match it.
__global__ void __launch_bounds__(256) radix_hist_kernel(const float *__restrict__ W, int64_t E,
                                                         const uint32_t *__restrict__ state, int width,
                                                         uint32_t *__restrict__ hist) {
  __shared__ uint32_t h[kBins];
  for (int i = threadIdx.x; i < kBins; i += blockDim.x) h[i] = 0;
  __syncthreads();
  const uint32_t fixed = state[2];
  const uint32_t prefix = state[0];
  const int shift = 31 - (int)fixed - width;  // bits of |w| live in 0..30
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < E; i += (int64_t)gridDim.x * blockDim.x) {
    const uint32_t b = abs_bits(W[i]);
    const bool match = fixed == 0 || (b >> (31 - fixed)) == prefix;
    if (match) atomicAdd(&h[(b >> shift) & ((1u << width) - 1u)], 1u);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < (1 << width); i += blockDim.x)
    if (h[i]) atomicAdd(&hist[i], h[i]);
}

// Walk the histogram from the top bin down to the one holding the wanted rank,
// extend the prefix by that bin and update the remaining rank; clear the histogram.
__global__ void radix_pick_kernel(uint32_t *__restrict__ state, int width, uint32_t *__restrict__ hist) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  uint32_t want = state[1];
  int bin = (1 << width) - 1;
  for (; bin > 0; --bin) {
    if (hist[bin] >= want) break;
    want -= hist[bin];
  }
  state[0] = (state[0] << width) | (uint32_t)bin;
  state[1] = want;
  state[2] += (uint32_t)width;
  for (int i = 0; i < (1 << width); ++i) hist[i] = 0;
}

// counts[n] = number of entries of row n with |w| >= tau (one warp per row).
__global__ void __launch_bounds__(256) row_count_kernel(const float *__restrict__ W, int64_t N, int64_t K,
                                                        const uint32_t *__restrict__ state,
                                                        int32_t *__restrict__ counts) {
  const int lane = threadIdx.x & 31;
  const int64_t row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (row >= N) return;
  const uint32_t tau = state[0];
  int c = 0;
  for (int64_t k = lane; k < K; k += 32) c += abs_bits(W[row * K + k]) >= tau;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
  if (lane == 0) counts[row] = c;
}

// row_ptr[0] = 0, row_ptr[n+1] = row_ptr[n] + counts[n]: one block, in order.
__global__ void __launch_bounds__(1024) row_scan_kernel(const int32_t *__restrict__ counts, int64_t N,
                                                        int32_t *__restrict__ row_ptr) {
  __shared__ int64_t part[1024];
  const int64_t per = (N + blockDim.x - 1) / blockDim.x;
  const int64_t a = (int64_t)threadIdx.x * per, b = min(N, a + per);
  int64_t s = 0;
  for (int64_t i = a; i < b; ++i) s += counts[i];
  part[threadIdx.x] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    int64_t run = 0;
    for (int i = 0; i < (int)blockDim.x; ++i) {
      const int64_t v = part[i];
      part[i] = run;
      run += v;
    }
    row_ptr[N] = (int32_t)run;
  }
  __syncthreads();
  int64_t run = part[threadIdx.x];
  for (int64_t i = a; i < b; ++i) {
    row_ptr[i] = (int32_t)run;
    run += counts[i];
  }
}

// Entries of row n in increasing k (one warp per row; ballots keep the order).
// Nothing is written at or beyond `cap`.
__global__ void __launch_bounds__(256) row_fill_kernel(const float *__restrict__ W, int64_t N, int64_t K,
                                                       const uint32_t *__restrict__ state,
                                                       const int32_t *__restrict__ row_ptr, int64_t cap,
                                                       int32_t *__restrict__ col, uint16_t *__restrict__ val) {
  const int lane = threadIdx.x & 31;
  const int64_t row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (row >= N) return;
  const uint32_t tau = state[0];
  int64_t pos = row_ptr[row];
  for (int64_t k0 = 0; k0 < K; k0 += 32) {
    const int64_t k = k0 + lane;
    const float w = k < K ? W[row * K + k] : 0.0f;
    const bool hit = k < K && abs_bits(w) >= tau;
    const uint32_t m = __ballot_sync(0xffffffffu, hit);
    if (hit) {
      const int64_t at = pos + __popc(m & ((1u << lane) - 1u));
      if (at < cap) {
        col[at] = (int32_t)k;
        val[at] = __half_as_ushort(__float2half_rn(w));
      }
    }
    pos += __popc(m);
  }
}

// y[m][n] += sum over row n's entries of x[m][col] * val, fp32 in entry order
// (one thread per (token, row)).
template <bool kBf16X, bool kBf16Y>
__global__ void __launch_bounds__(256) sparse_add_kernel(const uint16_t *__restrict__ X, int64_t M, int64_t N,
                                                         int64_t K, const int32_t *__restrict__ row_ptr,
                                                         const int32_t *__restrict__ col,
                                                         const uint16_t *__restrict__ val, void *__restrict__ Y) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= M * N) return;
  const int64_t m = i / N, n = i % N;
  const int32_t a = row_ptr[n], b = row_ptr[n + 1];
  if (a == b) return;
  float acc = 0.0f;
  for (int32_t j = a; j < b; ++j) {
    const uint16_t xb = X[m * K + col[j]];
    const float x = kBf16X ? __uint_as_float((uint32_t)xb << 16) : __half2float(__ushort_as_half(xb));
    acc = fmaf(x, __half2float(__ushort_as_half(val[j])), acc);
  }
  if (kBf16Y) {
    __nv_bfloat16 *y = static_cast<__nv_bfloat16 *>(Y) + i;
    *y = __float2bfloat16_rn(__bfloat162float(*y) + acc);
  } else {
    float *y = static_cast<float *>(Y) + i;
    *y = *y + acc;
  }
}

}  // namespace outlier_impl

// tau of the `count`-th largest |w| (count >= 1) into state[0] (as |w| bits).
// state: 3 uint32, set here; hist: 2048 uint32, zero-filled beforehand and left zeroed.
cudaError_t launch_outlier_threshold(const float *W, int64_t E, int64_t count, uint32_t *state, uint32_t *hist,
                                     int sm_count, cudaStream_t stream) {
  using namespace outlier_impl;
  state_init_kernel<<<1, 32, 0, stream>>>(state, (uint32_t)count);
  const int widths[3] = {11, 11, 9};  // bits 30..0 of |w|
  int64_t blocks = (E + 255) / 256;
  if (blocks > (int64_t)sm_count * 8) blocks = (int64_t)sm_count * 8;
  for (int pass = 0; pass < 3; ++pass) {
    radix_hist_kernel<<<(int)blocks, 256, 0, stream>>>(W, E, state, widths[pass], hist);
    radix_pick_kernel<<<1, 32, 0, stream>>>(state, widths[pass], hist);
  }
  return cudaGetLastError();
}

cudaError_t launch_outlier_csr(const float *W, int64_t N, int64_t K, const uint32_t *state, int32_t *counts,
                               int32_t *row_ptr, int64_t cap, int32_t *col, uint16_t *val, cudaStream_t stream) {
  using namespace outlier_impl;
  const int blocks = (int)((N * 32 + 255) / 256);
  row_count_kernel<<<blocks, 256, 0, stream>>>(W, N, K, state, counts);
  row_scan_kernel<<<1, 1024, 0, stream>>>(counts, N, row_ptr);
  row_fill_kernel<<<blocks, 256, 0, stream>>>(W, N, K, state, row_ptr, cap, col, val);
  return cudaGetLastError();
}

cudaError_t launch_sparse_add(const void *X, bool x_bf16, int64_t M, int64_t N, int64_t K, const int32_t *row_ptr,
                              const int32_t *col, const uint16_t *val, void *Y, bool y_bf16, cudaStream_t stream) {
  using namespace outlier_impl;
  const int64_t total = M * N;
  const int blocks = (int)((total + 255) / 256);
  const uint16_t *x = static_cast<const uint16_t *>(X);
  if (x_bf16) {
    if (y_bf16) sparse_add_kernel<true, true><<<blocks, 256, 0, stream>>>(x, M, N, K, row_ptr, col, val, Y);
    else sparse_add_kernel<true, false><<<blocks, 256, 0, stream>>>(x, M, N, K, row_ptr, col, val, Y);
  } else {
    if (y_bf16) sparse_add_kernel<false, true><<<blocks, 256, 0, stream>>>(x, M, N, K, row_ptr, col, val, Y);
    else sparse_add_kernel<false, false><<<blocks, 256, 0, stream>>>(x, M, N, K, row_ptr, col, val, Y);
  }
  return cudaGetLastError();
}

}  // namespace w4
