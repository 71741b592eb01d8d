// gptq.cu -- GPTQ quantization of one weight matrix (ch. 22 "Advanced inference
// optimisation", section 22.3: minimize || W X - W^ X ||_F^2 on calibration
// inputs X, with the Hessian H = 2 X X^T deciding how each weight's quantization
// error is compensated on the weights not yet quantized).
//
// Every step is fp64 with explicit round-to-nearest operations (no fused
// multiply-add) and a fixed summation order, so the result is reproducible and
// equals a plain-loop evaluation of the same definition:
//   * H[a][b] = 2 sum_m x[m][a] x[m][b]  (m increasing); the diagonal gets
//     damp = damp_frac * trace(H) / K added (trace summed in index order);
//   * U, the upper Cholesky factor of H^-1, is P inv(L') P with L' the lower
//     Cholesky factor of P H P (P reverses k).  Both factorizations are
//     right-looking and blocked by panels of kPanel columns (rows): a one-CTA
//     kernel finalizes the panel in order, then one launch applies the panel's
//     updates to every trailing element.  Each element still receives its
//     updates one at a time in increasing k -- exactly the sequential
//     subtraction (Cholesky) and summation (inverse) of the plain loops:
//       L'[i][j] = (R[i][j] - L'[i][0] L'[j][0] - ... - L'[i][j-1] L'[j][j-1]) / L'[j][j],
//       inv[i][c] = -(0 + L'[i][c] inv[c][c] + ... + L'[i][i-1] inv[i-1][c]) / L'[i][i];
//   * the column sweep: one warp per weight row, k = 0..K-1 in order; at each
//     group start the scale and zero come from the current weights by the RTN
//     rule (fp32, as in quantize.cu); err = (w - w^) / U[k][k] and every later
//     weight moves by w[k'] -= err * U[k][k'] (a CTA of 8 row-warps stages each
//     row of U in shared memory once for all of them).
#include "common.cuh"

namespace w4 {
namespace gptq_impl {

constexpr int kHT = 16;  // Hessian tile (16 x 16 outputs per block)
constexpr int kHM = 32;  // calibration rows per shared-memory chunk

template <bool kBf16>
__device__ __forceinline__ double x_val(uint16_t b) {
  return (double)(kBf16 ? __uint_as_float((uint32_t)b << 16) : __half2float(__ushort_as_half(b)));
}

template <bool kBf16>
__global__ void __launch_bounds__(256) hessian_kernel(const uint16_t *__restrict__ X, int64_t Mc, int64_t K,
                                                      double *__restrict__ H) {
  __shared__ double xa[kHM][kHT], xb[kHM][kHT];
  const int ta = threadIdx.x / kHT, tb = threadIdx.x % kHT;
  const int64_t a0 = (int64_t)blockIdx.y * kHT, b0 = (int64_t)blockIdx.x * kHT;
  double acc = 0.0;
  for (int64_t m0 = 0; m0 < Mc; m0 += kHM) {
    for (int i = threadIdx.x; i < kHM * kHT; i += blockDim.x) {
      const int mm = i / kHT, c = i % kHT;
      const int64_t m = m0 + mm;
      xa[mm][c] = (m < Mc && a0 + c < K) ? x_val<kBf16>(X[m * K + a0 + c]) : 0.0;
      xb[mm][c] = (m < Mc && b0 + c < K) ? x_val<kBf16>(X[m * K + b0 + c]) : 0.0;
    }
    __syncthreads();
    const int lim = (int)min((int64_t)kHM, Mc - m0);
    for (int mm = 0; mm < lim; ++mm) acc = __dadd_rn(acc, __dmul_rn(xa[mm][ta], xb[mm][tb]));
    __syncthreads();
  }
  const int64_t a = a0 + ta, b = b0 + tb;
  if (a < K && b < K) H[a * K + b] = __dmul_rn(2.0, acc);
}

__global__ void damp_kernel(double *__restrict__ H, int64_t K, double damp_frac) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  double tr = 0.0;
  for (int64_t a = 0; a < K; ++a) tr = __dadd_rn(tr, H[a * K + a]);
  const double damp = __dmul_rn(damp_frac, __ddiv_rn(tr, (double)K));
  for (int64_t a = 0; a < K; ++a) H[a * K + a] = __dadd_rn(H[a * K + a], damp);
}

constexpr int kPanel = 8;     // columns (rows) per panel
constexpr int kPanelThreads = 1024;

// R = P H P into the lower triangle of A (row-major): A[i][j] = H[K-1-i][K-1-j], j <= i.
__global__ void __launch_bounds__(256) reverse_kernel(const double *__restrict__ H, int64_t K, double *__restrict__ A) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= K * K) return;
  const int64_t i = e / K, j = e - i * K;
  if (j <= i) A[e] = H[(K - 1 - i) * K + (K - 1 - j)];
}

__global__ void __launch_bounds__(256) zero_lower_kernel(double *__restrict__ A, int64_t K) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= K * K) return;
  const int64_t i = e / K, j = e - i * K;
  if (j <= i) A[e] = 0.0;
}

// Cholesky panel: columns j0 .. j0 + nb - 1 of A (updated through column j0 - 1)
// become columns of L' in order; PT[jj][i] = L'[i][j0 + jj] is a transposed copy
// for the trailing update's coalesced reads.  One CTA.
__global__ void __launch_bounds__(kPanelThreads) chol_panel_kernel(double *__restrict__ A, int64_t K, int64_t j0,
                                                                   int nb, double *__restrict__ PT,
                                                                   int *__restrict__ bad) {
  __shared__ double s_piv;
  for (int jj = 0; jj < nb; ++jj) {
    const int64_t c = j0 + jj;
    if (threadIdx.x == 0) {
      double d = A[c * K + c];
      if (!(d > 0.0)) {
        *bad = 1;
        d = 1.0;  // keeps the values finite; the call reports the failure
      }
      const double l = __dsqrt_rn(d);
      A[c * K + c] = l;
      s_piv = l;
    }
    __syncthreads();
    const double l = s_piv;
    for (int64_t i = c + 1 + threadIdx.x; i < K; i += blockDim.x) {
      const double v = __ddiv_rn(A[i * K + c], l);
      A[i * K + c] = v;
      PT[jj * K + i] = v;
    }
    __syncthreads();
    // the rest of the panel: A[i][c'] -= L'[i][c] L'[c'][c], c < c' <= i
    for (int cc = jj + 1; cc < nb; ++cc) {
      const int64_t c2 = j0 + cc;
      const double lc2 = A[c2 * K + c];
      for (int64_t i = c2 + threadIdx.x; i < K; i += blockDim.x)
        A[i * K + c2] = __dsub_rn(A[i * K + c2], __dmul_rn(A[i * K + c], lc2));
    }
    __syncthreads();
  }
}

// Cholesky trailing update: every A[i][c], c >= j1 = j0 + nb, i >= c, minus
// L'[i][k] L'[c][k] for k = j0 .. j1 - 1 in increasing k.  blockIdx.x is the row
// i - j1, blockIdx.y a tile of 256 columns; tiles right of the diagonal exit.
__global__ void __launch_bounds__(256) chol_trail_kernel(double *__restrict__ A, const double *__restrict__ PT,
                                                         int64_t K, int64_t j0, int nb) {
  const int64_t j1 = j0 + nb;
  const int64_t i = j1 + blockIdx.x, c = j1 + (int64_t)blockIdx.y * blockDim.x + threadIdx.x;
  if (c > i) return;
  double a = A[i * K + c];
  const double *li = A + i * K + j0;  // the same row for the whole CTA
#pragma unroll
  for (int k = 0; k < kPanel; ++k)
    if (k < nb) a = __dsub_rn(a, __dmul_rn(li[k], PT[k * K + c]));
  A[i * K + c] = a;
}

// Inverse panel: rows r0 .. r0 + nb - 1 of Li = inv(L') from their sums S (updated
// through row r0 - 1): Li[r][c] = -S[r][c] / L'[r][r] for c < r, Li[r][r] = 1 / L'[r][r];
// then the later rows of the panel add L'[r'][r] Li[r][c] to S[r'][c].  One CTA.
__global__ void __launch_bounds__(kPanelThreads) inv_panel_kernel(const double *__restrict__ L, double *__restrict__ S,
                                                                  int64_t K, int64_t r0, int nb,
                                                                  double *__restrict__ Li) {
  for (int rr = 0; rr < nb; ++rr) {
    const int64_t r = r0 + rr;
    const double lrr = L[r * K + r];
    for (int64_t c = threadIdx.x; c <= r; c += blockDim.x)
      Li[r * K + c] = c == r ? __ddiv_rn(1.0, lrr) : __ddiv_rn(-S[r * K + c], lrr);
    __syncthreads();
    for (int q = rr + 1; q < nb; ++q) {
      const int64_t r2 = r0 + q;
      const double l = L[r2 * K + r];
      for (int64_t c = threadIdx.x; c <= r; c += blockDim.x)
        S[r2 * K + c] = __dadd_rn(S[r2 * K + c], __dmul_rn(l, Li[r * K + c]));
    }
    __syncthreads();
  }
}

// Inverse trailing update: every S[i][c], i >= r1 = r0 + nb, c < r1, plus
// L'[i][k] Li[k][c] for k = max(c, r0) .. r1 - 1 in increasing k.  blockIdx.x is
// the row i - r1, blockIdx.y a tile of 256 columns.
__global__ void __launch_bounds__(256) inv_trail_kernel(const double *__restrict__ L, double *__restrict__ S,
                                                        const double *__restrict__ Li, int64_t K, int64_t r0, int nb) {
  const int64_t r1 = r0 + nb;
  const int64_t i = r1 + blockIdx.x, c = (int64_t)blockIdx.y * blockDim.x + threadIdx.x;
  if (c >= r1) return;
  double a = S[i * K + c];
#pragma unroll
  for (int k = 0; k < kPanel; ++k) {
    const int64_t kk = r0 + k;
    if (k < nb && kk >= c) a = __dadd_rn(a, __dmul_rn(L[i * K + kk], Li[kk * K + c]));
  }
  S[i * K + c] = a;
}

__device__ __forceinline__ float clamp15f(float v) { return fminf(fmaxf(v, 0.0f), 15.0f); }

// One warp per weight row, kSweepRows rows per CTA; U[j][k] = Li[K-1-j][K-1-k].
// At every step j the CTA stages the row U[j][j..K) in shared memory once for
// all its warps (the same values in the same order as reading them directly).
constexpr int kSweepRows = 8;
constexpr int kUChunk = 2048;  // U entries staged per round (16 KiB)

template <int kG>
__global__ void __launch_bounds__(32 * kSweepRows) sweep_kernel(const float *__restrict__ W, int64_t N, int64_t K,
                                                                 const double *__restrict__ Li,
                                                                 double *__restrict__ Wd, uint8_t *__restrict__ codes,
                                                                 uint16_t *__restrict__ scales,
                                                                 uint16_t *__restrict__ zeros) {
  constexpr int kPer = kG / 32;  // group elements per lane
  __shared__ double us[kUChunk];
  __shared__ double errs[kSweepRows];
  const int lane = threadIdx.x & 31;
  const int wid = threadIdx.x >> 5;
  const int64_t n = (int64_t)blockIdx.x * kSweepRows + wid;
  const bool row_ok = n < N;
  double *w = Wd + (row_ok ? n : 0) * K;
  if (row_ok)
    for (int64_t k = lane; k < K; k += 32) w[k] = (double)W[n * K + k];
  __syncwarp();
  const int64_t Kg = K / kG;
  float sc = 1.0f, z = 0.0f;
  for (int64_t j = 0; j < K; ++j) {
    const double *urow = Li + (K - 1 - j) * K + (K - 1);  // urow[-k] = U[j][k]
    if (row_ok) {
      if (j % kG == 0) {
        float mn, mx;
#pragma unroll
        for (int e = 0; e < kPer; ++e) {
          const float v = __double2float_rn(w[j + lane * kPer + e]);
          mn = e == 0 ? v : fminf(mn, v);
          mx = e == 0 ? v : fmaxf(mx, v);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        }
        __half sc16 = __float2half_rn(__fdiv_rn(__fsub_rn(mx, mn), 15.0f));
        sc = __half2float(sc16);
        if (sc == 0.0f) {
          sc = 1.0f;
          sc16 = __float2half_rn(1.0f);
        }
        z = clamp15f(rintf(__fdiv_rn(-mn, sc)));
        if (lane == 0) {
          scales[n * Kg + j / kG] = __half_as_ushort(sc16);
          zeros[n * Kg + j / kG] = __half_as_ushort(__float2half_rn(z));
        }
      }
      const double wj = w[j];
      const float q = clamp15f(__fadd_rn(rintf(__fdiv_rn(__double2float_rn(wj), sc)), z));
      if (lane == 0) codes[n * K + j] = (uint8_t)q;
      const float wq = __fmul_rn(__fsub_rn(q, z), sc);
      if (lane == 0) errs[wid] = __ddiv_rn(__dsub_rn(wj, (double)wq), urow[-j]);
    }
    // every later weight of every row: w[k] -= err * U[j][k], U staged chunk by chunk
    for (int64_t c0 = j + 1; c0 < K; c0 += kUChunk) {
      const int64_t cn = min((int64_t)kUChunk, K - c0);
      __syncthreads();  // errs written; the previous chunk fully used
      for (int64_t t = threadIdx.x; t < cn; t += blockDim.x) us[t] = urow[-(c0 + t)];
      __syncthreads();
      if (row_ok) {
        const double err = errs[wid];
        for (int64_t t = lane; t < cn; t += 32) w[c0 + t] = __dsub_rn(w[c0 + t], __dmul_rn(err, us[t]));
      }
    }
    __syncthreads();  // this step's updates are visible before the next step reads them
  }
}

}  // namespace gptq_impl

// Hessian, damping, Cholesky and inverse: Li (row-major K x K) holds inv(L').
// H, Lc, Li: K*K doubles each (Lc need not be zeroed: only its lower part is
// read; H is reused for the inverse's running sums once L' is formed);
// bad: one int, zero on entry, set when H is not positive definite.
cudaError_t launch_gptq_hinv(const void *X, bool x_bf16, int64_t Mc, int64_t K, double damp_frac, double *H,
                             double *Lc, double *Li, int *bad, cudaStream_t stream) {
  using namespace gptq_impl;
  const dim3 hg((unsigned)((K + kHT - 1) / kHT), (unsigned)((K + kHT - 1) / kHT));
  const uint16_t *x = static_cast<const uint16_t *>(X);
  if (x_bf16) hessian_kernel<true><<<hg, kHT * kHT, 0, stream>>>(x, Mc, K, H);
  else hessian_kernel<false><<<hg, kHT * kHT, 0, stream>>>(x, Mc, K, H);
  damp_kernel<<<1, 32, 0, stream>>>(H, K, damp_frac);
  const unsigned sq = (unsigned)((K * K + 255) / 256);
  reverse_kernel<<<sq, 256, 0, stream>>>(H, K, Lc);  // Lc: row-major, becomes L'
  double *PT = Li;  // kPanel x K transposed panel; Li is written only after the Cholesky
  for (int64_t j0 = 0; j0 < K; j0 += kPanel) {
    const int nb = (int)std::min<int64_t>(kPanel, K - j0);
    chol_panel_kernel<<<1, kPanelThreads, 0, stream>>>(Lc, K, j0, nb, PT, bad);
    const int64_t T = K - j0 - nb;
    if (T > 0) chol_trail_kernel<<<dim3((unsigned)T, (unsigned)((T + 255) / 256)), 256, 0, stream>>>(Lc, PT, K, j0, nb);
  }
  zero_lower_kernel<<<sq, 256, 0, stream>>>(H, K);  // H becomes the inverse's running sums
  for (int64_t r0 = 0; r0 < K; r0 += kPanel) {
    const int nb = (int)std::min<int64_t>(kPanel, K - r0);
    inv_panel_kernel<<<1, kPanelThreads, 0, stream>>>(Lc, H, K, r0, nb, Li);
    const int64_t rows = K - r0 - nb, r1 = r0 + nb;
    if (rows > 0)
      inv_trail_kernel<<<dim3((unsigned)rows, (unsigned)((r1 + 255) / 256)), 256, 0, stream>>>(Lc, H, Li, K, r0, nb);
  }
  return cudaGetLastError();
}

cudaError_t launch_gptq_sweep(const float *W, int64_t N, int64_t K, int group, const double *Li, double *Wd,
                              uint8_t *codes, uint16_t *scales, uint16_t *zeros, cudaStream_t stream) {
  using namespace gptq_impl;
  const unsigned blocks = (unsigned)((N + kSweepRows - 1) / kSweepRows);
  const int threads = 32 * kSweepRows;
  switch (group) {
    case 32: sweep_kernel<32><<<blocks, threads, 0, stream>>>(W, N, K, Li, Wd, codes, scales, zeros); break;
    case 64: sweep_kernel<64><<<blocks, threads, 0, stream>>>(W, N, K, Li, Wd, codes, scales, zeros); break;
    default: sweep_kernel<128><<<blocks, threads, 0, stream>>>(W, N, K, Li, Wd, codes, scales, zeros); break;
  }
  return cudaGetLastError();
}

}  // namespace w4
