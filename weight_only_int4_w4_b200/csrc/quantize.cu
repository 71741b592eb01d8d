// quantize.cu -- K0: per-group uint4 RTN quantize + nibble pack.
//
// Asymmetric codes: an affine map through a scale and a zero point per group of
// 128 input channels ("LLM inference acceleration" article, section 2.1), also
// served with groups of 32 and 64.  Symmetric variant: INT4 as the value set
// {-7..7} (mhpq.cn practitioner's article, section 2.1), stored as q + 8 with
// zero point 8.  Each lane holds 8 weights; a group is held by G/8 lanes.  Optional AWQ prescale w / s[k] is applied on load (ch. 22
// "Advanced inference optimisation", section 22.3, AWQ equation).  Every
// step uses IEEE fp32 round-to-nearest intrinsics so the results are bit-exact
// with the definition in w4.h.  The kernel is HBM-bound: it reads W once and
// writes 0.5 B of codes + 4 B of scale/zero per 128 weights.
#include <type_traits>

#include "common.cuh"

namespace w4 {

namespace quant_impl {

template <typename T>
struct Load4;

template <>
struct Load4<float> {
  static __device__ __forceinline__ void run(const float *p, float (&v)[4]) {
    float4 t = __ldcs(reinterpret_cast<const float4 *>(p));
    v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
  }
};

template <>
struct Load4<__half> {
  static __device__ __forceinline__ void run(const __half *p, float (&v)[4]) {
    uint2 t = __ldcs(reinterpret_cast<const uint2 *>(p));
    v[0] = __half2float(__ushort_as_half((unsigned short)(t.x & 0xFFFF)));
    v[1] = __half2float(__ushort_as_half((unsigned short)(t.x >> 16)));
    v[2] = __half2float(__ushort_as_half((unsigned short)(t.y & 0xFFFF)));
    v[3] = __half2float(__ushort_as_half((unsigned short)(t.y >> 16)));
  }
};

template <>
struct Load4<__nv_bfloat16> {
  static __device__ __forceinline__ void run(const __nv_bfloat16 *p, float (&v)[4]) {
    uint2 t = __ldcs(reinterpret_cast<const uint2 *>(p));
    v[0] = __uint_as_float(t.x << 16);
    v[1] = __uint_as_float(t.x & 0xFFFF0000u);
    v[2] = __uint_as_float(t.y << 16);
    v[3] = __uint_as_float(t.y & 0xFFFF0000u);
  }
};

__device__ __forceinline__ float clamp15(float v) { return fminf(fmaxf(v, 0.0f), 15.0f); }

// fl32(d / c) for a small odd integer constant c (7 or 15), without an fp32
// division: the double product d * RN64(1 / c) is within 2^-52 relative of d / c,
// while d / c, unless it is an fp32 value itself, lies at least about 2^-29
// relative from every fp32 rounding midpoint (d has 24 significant bits), so
// rounding the product to fp32 gives the correctly rounded quotient.  Checked
// exhaustively for c = 7 and 15 over every fp32 d in the subnormal and lowest
// binades, [1, 4) and the top binades (the binades between scale exactly).
template <int kC>
__device__ __forceinline__ float div_by_const(float d) {
  return __double2float_rn(__dmul_rn((double)d, 1.0 / (double)kC));
}

// Reciprocal within 1 ulp (PTX rcp.approx.f32: relative error at most 2^-23).
// Only ever applied to fp16 scales in [2^-24, 65504], whose reciprocals are normal.
__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// rint(fl(v / sc)) -- the rounded IEEE quotient, as the codes are defined -- without
// a division per weight.  With inv = 1 / sc within 1 ulp and r = fl(v * inv),
//   r = (v / sc)(1 + e1)(1 + e2),  |e1| <= 2^-23, |e2| <= 2^-24,
// and fl(v / sc) = (v / sc)(1 + e3), |e3| <= 2^-24, so the two differ by at most
// 2^-22 |v / sc| < 2^-16 while |v / sc| < 64.  When r is farther than 2^-15 from
// every half-integer, r and fl(v / sc) lie strictly between the same two
// half-integers and round to the same integer.  When |r| >= 64 both roundings are
// beyond +-62, and every caller clamps the code to at most 15 (after adding a zero
// point in [0, 15]) or to [-7, 7], so the code is the same.  Only an r within
// 2^-15 of a half-integer takes the exact quotient (always correct).  NaN stays NaN.
// near_half: |r - rint(r)| >= 0.5 - 2^-15 (r - rint(r) is exact).
__device__ __forceinline__ bool near_half(float r, float t) { return fabsf(__fsub_rn(r, t)) >= 0.5f - 0x1p-15f; }
__device__ __forceinline__ float rint_quotient(float v, float sc, float inv) {
  const float r = __fmul_rn(v, inv);
  const float t = rintf(r);
  return near_half(r, t) ? rintf(__fdiv_rn(v, sc)) : t;
}

// Order-preserving integer key of a float (not NaN): signed-integer order of the
// keys is the order of the values (with -0 just below +0).
__device__ __forceinline__ int f2key(float f) {
  const int b = __float_as_int(f);
  return b ^ ((b >> 31) & 0x7FFFFFFF);
}
__device__ __forceinline__ float key2f(int k) { return __int_as_float(k ^ ((k >> 31) & 0x7FFFFFFF)); }
__device__ __forceinline__ float clamp7(float v) { return fminf(fmaxf(v, -7.0f), 7.0f); }

constexpr int kQuantUnroll = 2;  // 256-element chunks in flight per warp
constexpr int kWPL = 8;          // weights per lane

// The matrix is walked as its flattened N*K elements in chunks of 256: lane l of
// a warp holds elements 8l..8l+7 of a chunk, and a group of G (32, 64 or 128)
// consecutive elements (groups never straddle rows, since G divides K) is held
// by G/8 consecutive lanes, which reduce its min and max with shuffles.  A warp
// thus works on 2 to 8 groups at once, and the per-group steps (scale, zero
// point, reciprocal) are shared by 8 weights per lane.  Group j of the flattened
// order is scales[j] / zeros[j] of the [N][K/G] arrays.
template <typename TW, bool kAwq, bool kCodes, bool kSym, int kG, bool kMask>
__global__ void __launch_bounds__(256) quantize_kernel(const TW *__restrict__ W, const float *__restrict__ awq_s,
                                                       int64_t E, int64_t K,
                                                       const uint32_t *__restrict__ outlier_tau,
                                                       uint8_t *__restrict__ packed, uint16_t *__restrict__ scales,
                                                       uint16_t *__restrict__ zeros, uint8_t *__restrict__ codes) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  constexpr int kChunk = 32 * kWPL;
  const int64_t chunks = (E + kChunk - 1) / kChunk;
  constexpr int lg = kG / kWPL;  // lanes per group
  // dense part of a dense + sparse split: weights with |w| >= tau count as 0 here
  const uint32_t tau = kMask ? *outlier_tau : 0xFFFFFFFFu;

  for (int64_t base = warp * kQuantUnroll; base < chunks; base += nwarps * kQuantUnroll) {
    float v[kQuantUnroll][kWPL];
#pragma unroll
    for (int u = 0; u < kQuantUnroll; ++u) {
      const int64_t e = (base + u) * kChunk + lane * kWPL;
      if (e < E) {  // E is a multiple of 32 (G divides K), so a lane's 8 are all in range
        float h[4];
        Load4<TW>::run(W + e, h);
#pragma unroll
        for (int j = 0; j < 4; ++j) v[u][j] = h[j];
        Load4<TW>::run(W + e + 4, h);
#pragma unroll
        for (int j = 0; j < 4; ++j) v[u][4 + j] = h[j];
        if constexpr (kMask) {
#pragma unroll
          for (int j = 0; j < kWPL; ++j)
            if ((__float_as_uint(v[u][j]) & 0x7FFFFFFFu) >= tau) v[u][j] = 0.0f;
        }
        if (kAwq) {
          const int64_t k = e % K;  // a lane's 8 weights lie in one row (K is a multiple of 32)
          const float4 s0 = __ldg(reinterpret_cast<const float4 *>(awq_s + k));
          const float4 s1 = __ldg(reinterpret_cast<const float4 *>(awq_s + k + 4));
          const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
          for (int j = 0; j < kWPL; ++j) v[u][j] = __fdiv_rn(v[u][j], sv[j]);
        }
      } else {
#pragma unroll
        for (int j = 0; j < kWPL; ++j) v[u][j] = 0.0f;
      }
    }
#pragma unroll
    for (int u = 0; u < kQuantUnroll; ++u) {
      const int64_t e = (base + u) * kChunk + lane * kWPL;
      float mn = v[u][0], mx = v[u][0];
#pragma unroll
      for (int j = 1; j < kWPL; ++j) {
        mn = fminf(mn, v[u][j]);
        mx = fmaxf(mx, v[u][j]);
      }
#pragma unroll
      for (int o = lg >> 1; o > 0; o >>= 1) {  // within each aligned run of lg lanes
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      }
      uint32_t q[kWPL];
      __half sc16;
      float z;
      if constexpr (kSym) {
        // scale = fp16(max|w| / 7) (1.0 if 0); q = clamp(rint(w / scale), -7, 7), stored as q + 8
        const float amax = fmaxf(fabsf(mn), fabsf(mx));
        sc16 = __float2half_rn(div_by_const<7>(amax));
        float sc = __half2float(sc16);
        if (sc == 0.0f) {
          sc = 1.0f;
          sc16 = __float2half_rn(1.0f);
        }
        z = 8.0f;
        const float inv = rcp_approx(sc);
#pragma unroll
        for (int j = 0; j < kWPL; ++j) q[j] = (uint32_t)(clamp7(rint_quotient(v[u][j], sc, inv)) + 8.0f);
      } else {
        // scale = fp16((mx - mn) / 15); a zero fp16 scale is taken as 1.0
        sc16 = __float2half_rn(div_by_const<15>(__fsub_rn(mx, mn)));
        float sc = __half2float(sc16);
        if (sc == 0.0f) {
          sc = 1.0f;
          sc16 = __float2half_rn(1.0f);
        }
        const float inv = rcp_approx(sc);
        z = clamp15(rint_quotient(-mn, sc, inv));
        // the lane's rounded quotients, one (rare) exact pass if any of them lies
        // near a half-integer
        float t[kWPL];
        bool near = false;
#pragma unroll
        for (int j = 0; j < kWPL; ++j) {
          const float r = __fmul_rn(v[u][j], inv);
          t[j] = rintf(r);
          near |= near_half(r, t[j]);
        }
        if (near) {
#pragma unroll
          for (int j = 0; j < kWPL; ++j) t[j] = rintf(__fdiv_rn(v[u][j], sc));
        }
        // clamp(t + z, 0, 15): t + z is an integer-valued float; the conversion to
        // unsigned saturates negatives (and NaN) to 0
#pragma unroll
        for (int j = 0; j < kWPL; ++j) q[j] = min(__float2uint_rz(__fadd_rn(t[j], z)), 15u);
      }
      if (e < E) {
        uint32_t pk = 0;
#pragma unroll
        for (int j = 0; j < kWPL; ++j) pk |= q[j] << (4 * j);
        reinterpret_cast<uint32_t *>(packed)[e >> 3] = pk;
        if (kCodes) {
          const uint32_t c0 = q[0] | (q[1] << 8) | (q[2] << 16) | (q[3] << 24);
          const uint32_t c1 = q[4] | (q[5] << 8) | (q[6] << 16) | (q[7] << 24);
          reinterpret_cast<uint2 *>(codes)[e >> 3] = make_uint2(c0, c1);
        }
        if ((lane & (lg - 1)) == 0) {
          const int64_t gi = e / kG;
          scales[gi] = __half_as_ushort(sc16);
          zeros[gi] = __half_as_ushort(__float2half_rn(z));
        }
      }
    }
  }
}

// 32 codes (two 16-B loads) -> 16 packed bytes (one 16-B store).
__global__ void __launch_bounds__(256) pack_kernel(const uint8_t *__restrict__ codes, int64_t chunks,
                                                   uint8_t *__restrict__ packed) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < chunks;
       i += (int64_t)gridDim.x * blockDim.x) {
    const uint4 a = __ldcs(reinterpret_cast<const uint4 *>(codes + i * 32));
    const uint4 b = __ldcs(reinterpret_cast<const uint4 *>(codes + i * 32 + 16));
    const uint32_t in[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t out[4];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      uint32_t r = 0;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t c = in[2 * w + h] & 0x0F0F0F0Fu;  // 4 codes, masked to 4 bits
        // bytes c0 c1 c2 c3 -> (c0 | c1 << 4) and (c2 | c3 << 4)
        const uint32_t lo = (c & 0xFFu) | ((c >> 4) & 0xF0u);
        const uint32_t hi = ((c >> 16) & 0xFFu) | ((c >> 20) & 0xF0u);
        r |= (lo | (hi << 8)) << (16 * h);
      }
      out[w] = r;
    }
    __stcs(reinterpret_cast<uint4 *>(packed + i * 16), make_uint4(out[0], out[1], out[2], out[3]));
  }
}

int grid_for(int64_t work_items, int items_per_block, int sm_count, int blocks_per_sm) {
  int64_t need = (work_items + items_per_block - 1) / items_per_block;
  int64_t cap = (int64_t)sm_count * blocks_per_sm;
  if (need > cap) need = cap;
  if (need < 1) need = 1;
  return (int)need;
}

template <typename TW, bool kSym, int kG, bool kMask>
cudaError_t launch_quantize_g(const void *W, const float *awq_s, int64_t N, int64_t K, const uint32_t *tau,
                              uint8_t *packed, uint16_t *scales, uint16_t *zeros, uint8_t *codes, int sm_count,
                              cudaStream_t stream) {
  const int64_t E = N * K;
  const int64_t chunks = (E + 32 * kWPL - 1) / (32 * kWPL);
  const int grid = grid_for(chunks, 8 * kQuantUnroll, sm_count, 8);
  const TW *w = static_cast<const TW *>(W);
  if (awq_s) {
    if (codes)
      quantize_kernel<TW, true, true, kSym, kG, kMask><<<grid, 256, 0, stream>>>(w, awq_s, E, K, tau, packed, scales,
                                                                                  zeros, codes);
    else
      quantize_kernel<TW, true, false, kSym, kG, kMask><<<grid, 256, 0, stream>>>(w, awq_s, E, K, tau, packed, scales,
                                                                                   zeros, codes);
  } else {
    if (codes)
      quantize_kernel<TW, false, true, kSym, kG, kMask><<<grid, 256, 0, stream>>>(w, awq_s, E, K, tau, packed, scales,
                                                                                   zeros, codes);
    else
      quantize_kernel<TW, false, false, kSym, kG, kMask><<<grid, 256, 0, stream>>>(w, awq_s, E, K, tau, packed,
                                                                                    scales, zeros, codes);
  }
  return cudaGetLastError();
}

template <typename TW, bool kSym>
cudaError_t launch_quantize_t(const void *W, const float *awq_s, int64_t N, int64_t K, int group,
                              const uint32_t *tau, uint8_t *packed, uint16_t *scales, uint16_t *zeros,
                              uint8_t *codes, int sm_count, cudaStream_t stream) {
  if (tau) {  // dense part of the outlier split: fp32 weights, asymmetric codes (see libw4.cu)
    if constexpr (std::is_same<TW, float>::value && !kSym) {
      switch (group) {
        case 32: return launch_quantize_g<TW, false, 32, true>(W, awq_s, N, K, tau, packed, scales, zeros, codes,
                                                              sm_count, stream);
        case 64: return launch_quantize_g<TW, false, 64, true>(W, awq_s, N, K, tau, packed, scales, zeros, codes,
                                                              sm_count, stream);
        default: return launch_quantize_g<TW, false, 128, true>(W, awq_s, N, K, tau, packed, scales, zeros, codes,
                                                               sm_count, stream);
      }
    } else {
      return cudaErrorInvalidValue;
    }
  }
  switch (group) {
    case 32: return launch_quantize_g<TW, kSym, 32, false>(W, awq_s, N, K, tau, packed, scales, zeros, codes, sm_count,
                                                           stream);
    case 64: return launch_quantize_g<TW, kSym, 64, false>(W, awq_s, N, K, tau, packed, scales, zeros, codes, sm_count,
                                                           stream);
    default: return launch_quantize_g<TW, kSym, 128, false>(W, awq_s, N, K, tau, packed, scales, zeros, codes,
                                                            sm_count, stream);
  }
}

template <bool kSym>
cudaError_t launch_quantize_s(const void *W, int dtype, const float *awq_s, int64_t N, int64_t K, int group,
                              const uint32_t *tau, uint8_t *packed, uint16_t *scales, uint16_t *zeros,
                              uint8_t *codes, int sm_count, cudaStream_t stream) {
  switch (dtype) {
    case 0:
      return launch_quantize_t<float, kSym>(W, awq_s, N, K, group, tau, packed, scales, zeros, codes, sm_count, stream);
    case 1:
      return launch_quantize_t<__half, kSym>(W, awq_s, N, K, group, tau, packed, scales, zeros, codes, sm_count, stream);
    default:
      return launch_quantize_t<__nv_bfloat16, kSym>(W, awq_s, N, K, group, tau, packed, scales, zeros, codes, sm_count,
                                                    stream);
  }
}

}  // namespace quant_impl

// dtype: 0 = fp32, 1 = fp16, 2 = bf16; group 32, 64 or 128; symmetric selects the {-7..7} variant
// tau: device pointer to the outlier threshold (bits of |w|), or NULL for none.
cudaError_t launch_quantize(const void *W, int dtype, const float *awq_s, int64_t N, int64_t K, int group,
                            bool symmetric, const uint32_t *tau, uint8_t *packed, uint16_t *scales, uint16_t *zeros,
                            uint8_t *codes, int sm_count, cudaStream_t stream) {
  return symmetric ? quant_impl::launch_quantize_s<true>(W, dtype, awq_s, N, K, group, tau, packed, scales, zeros,
                                                         codes, sm_count, stream)
                   : quant_impl::launch_quantize_s<false>(W, dtype, awq_s, N, K, group, tau, packed, scales, zeros,
                                                          codes, sm_count, stream);
}

cudaError_t launch_pack(const uint8_t *codes, int64_t N, int64_t K, uint8_t *packed, int sm_count,
                        cudaStream_t stream) {
  const int64_t chunks = N * K / 32;
  const int grid = quant_impl::grid_for(chunks, 256, sm_count, 8);
  quant_impl::pack_kernel<<<grid, 256, 0, stream>>>(codes, chunks, packed);
  return cudaGetLastError();
}

}  // namespace w4
