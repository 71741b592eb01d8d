// gemv_mma.cu -- K1: decode / small-batch W4A16 matmul, M <= 64 tokens.
//
// Decode is bound by the weight bytes read per token, not by arithmetic
// ("LLM inference acceleration" article, section 1.1; ch. 22 "Advanced
// inference optimisation", section 22.2 table).  This kernel therefore keeps
// HBM busy with a deep TMA ring and spends about one LOP3 per two weights:
//
//   * Work unit ("task"): a tile of 64 output rows x KS quantization groups
//     (KS x 128 input channels).  A CTA owns one k-slice (KS groups) and walks
//     over row tiles; its activations for that k-slice stay in registers as
//     mma.sync B fragments for the whole kernel (x is reused by every row).
//   * Warp 4 (producer) streams each task's packed codes [64 rows x KS*64 B]
//     (128-byte swizzle when rows are 128 B), and the tile's fp16 scales and
//     zeros [64 rows x 8 groups], into an NST-deep shared-memory ring with TMA.
//   * Warps 0..3 (compute) own 16 rows each: no cross-warp reduction.  A 4-bit
//     code becomes the 16-bit value OFF + q with one LOP3 against a magic
//     exponent (OFF = 128 for bf16, 1024 for fp16), exact, so the tensor core
//     computes D = sum_k (OFF + q) x up to fp32 accumulation.  Per group the
//     result is promoted once:  y += scale * D - scale * (OFF + z) * S  with
//     S = sum_k x over the group, i.e. scale * sum_k (q - z) x: the
//     dequantize-then-matmul of the weight-only path (ch. 22, section 22.3),
//     without rounding the dequantized weight to 16 bits.
//   * AWQ (W^ = quant(W/s) * s, ch. 22 section 22.3) folds s into x: x*s is
//     split into a 16-bit high and a 16-bit low part, two MMAs each.
//   * k-slices of different CTAs (split-K) write fp32 partials to the
//     workspace; the last warp to arrive on a 16-row block (atomic counter)
//     sums them.  No warp ever waits on another CTA.
//
// mma.sync m16n8k16 fragments (g = lane / 4, t = lane % 4):
//   A regs: {row g, k 2t..2t+1}, {row g+8, k 2t..}, {row g, k 2t+8..}, {row g+8, k 2t+8..}
//   B regs: {k 2t..2t+1, col g}, {k 2t+8.., col g};  C: {row g, col 2t..2t+1}, {row g+8, ...}
// The MMA's k order is a permutation of the group's 128 channels chosen so
// that lane (g, t) feeds A from the 16 bytes of chunk t of its rows; the B
// fragments follow the same permutation.
#include "common.cuh"

namespace w4 {

struct GemvParams {
  const void *X;
  int64_t M, N, K;
  const uint16_t *scales;
  const uint16_t *zeros;
  const float *awq_s;
  void *Y;
  int y_bf16;
  float *ws;           // [kslices][M][N] fp32 partials (split-K only)
  uint32_t *counters;  // [ceil(N/16)] arrival counters (split-K only)
  int kslices;
  int grid_x;          // CTAs per k-slice
};

namespace gemv_impl {

constexpr int kRows = 64;        // rows per task (4 compute warps x 16)
constexpr int kScaleBox = 8;     // groups per scale/zero TMA box (16 bytes)

template <int KS>
struct GemvCfg {
  static constexpr int kPBytes = kRows * KS * 64;
  static constexpr int kSBytes = kRows * kScaleBox * 2;
  static constexpr int kStage = kPBytes + 2 * kSBytes;
  static constexpr int kNst = KS == 4 ? 6 : 8;
  static constexpr int kSmem = 1024 + kNst * kStage + 256;
};

template <bool kBf16>
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  if constexpr (kBf16) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  }
}

template <bool kBf16>
__device__ __forceinline__ float h16_to_f32(uint32_t bits16) {
  if constexpr (kBf16) return __uint_as_float(bits16 << 16);
  else return __half2float(__ushort_as_half((unsigned short)bits16));
}

template <bool kBf16>
__device__ __forceinline__ uint32_t f32_to_h16(float v) {
  if constexpr (kBf16) return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v));
  else return (uint32_t)__half_as_ushort(__float2half_rn(v));
}

// Byte offset of 16-byte chunk `t` of group `gi` of smem row `r` in a packed stage.
template <int KS>
__device__ __forceinline__ uint32_t chunk_offset(int r, int gi, int t) {
  if constexpr (KS == 1) {
    return (uint32_t)(r * 64 + t * 16);  // 64-byte rows, no swizzle (conflict-free already)
  } else {
    const int box = gi >> 1;                         // 128-byte boxes of two groups
    const int chunk = ((gi & 1) * 4 + t) ^ (r & 7);  // 128-byte swizzle
    return (uint32_t)(box * (kRows * 128) + r * 128 + chunk * 16);
  }
}

template <int T8, int KS, bool kBf16, bool kAwq, bool kScTma>
__global__ void __launch_bounds__(160) gemv_kernel(const __grid_constant__ CUtensorMap tmP,
                                                   const __grid_constant__ CUtensorMap tmS,
                                                   const __grid_constant__ CUtensorMap tmZ, const GemvParams p) {
  using Cfg = GemvCfg<KS>;
  constexpr uint32_t kMagic = kBf16 ? 0x43004300u : 0x64006400u;
  constexpr float kOff = kBf16 ? 128.0f : 1024.0f;
  constexpr int kParts = kAwq ? 2 : 1;  // high / low halves of x * s

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + Cfg::kNst * Cfg::kStage);
  uint64_t *empty = full + Cfg::kNst;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2;
  const int t = lane & 3;
  const int64_t M = p.M, N = p.N, K = p.K;
  const int64_t Kg = K / kGroup;
  const int64_t RT = (N + kRows - 1) / kRows;
  const int64_t RB16 = (N + 15) / 16;
  const int kslice = blockIdx.y;
  const int64_t g_first = (int64_t)kslice * KS;
  const int64_t g0 = g_first & ~(int64_t)(kScaleBox - 1);
  const int64_t ntask = (int64_t)blockIdx.x < RT ? (RT - blockIdx.x + p.grid_x - 1) / p.grid_x : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < Cfg::kNst; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 4);
    }
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == 4) {
    // ---------------- producer: one thread drives the TMA ring
    if (lane == 0) {
      prefetch_tensormap(&tmP);
      if (kScTma) {
        prefetch_tensormap(&tmS);
        prefetch_tensormap(&tmZ);
      }
      for (int64_t j = 0; j < ntask; ++j) {
        const int s = (int)(j % Cfg::kNst);
        const uint32_t ph = (uint32_t)(j / Cfg::kNst) & 1u;
        if (!mbar_wait(&empty[s], ph ^ 1u, kErrTimeoutTma)) break;
        const int32_t row0 = (int32_t)((blockIdx.x + j * p.grid_x) * kRows);
        uint8_t *st = smem + s * Cfg::kStage;
        mbar_arrive_expect_tx(&full[s], kScTma ? Cfg::kStage : Cfg::kPBytes);
        const int32_t xb = (int32_t)(g_first * 64);
        if constexpr (KS == 1) {
          tma_load_2d(st, &tmP, &full[s], xb, row0);
        } else {
#pragma unroll
          for (int b = 0; b < KS / 2; ++b) tma_load_2d(st + b * (kRows * 128), &tmP, &full[s], xb + 128 * b, row0);
        }
        if constexpr (kScTma) {
          tma_load_2d(st + Cfg::kPBytes, &tmS, &full[s], (int32_t)g0, row0);
          tma_load_2d(st + Cfg::kPBytes + Cfg::kSBytes, &tmZ, &full[s], (int32_t)g0, row0);
        }
      }
    }
    return;
  }

  // ---------------- compute warps: activations of this k-slice -> B fragments
  const uint16_t *xg = static_cast<const uint16_t *>(p.X);
  uint32_t B[KS][T8][kParts][8][2];
  float Sv[KS][T8][2];
#pragma unroll
  for (int gi = 0; gi < KS; ++gi) {
    const int64_t kg = g_first + gi;
#pragma unroll
    for (int o = 0; o < T8; ++o) {
      const int64_t tok = o * 8 + g;
      uint32_t r[kParts][16];
      float ssum = 0.0f;
      if (kg < Kg && tok < M) {
        const uint16_t *src = xg + tok * K + kg * kGroup + 32 * t;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint4 v = __ldg(reinterpret_cast<const uint4 *>(src + 8 * c));
          r[0][4 * c + 0] = v.x; r[0][4 * c + 1] = v.y; r[0][4 * c + 2] = v.z; r[0][4 * c + 3] = v.w;
        }
        if constexpr (kAwq) {
          const float *sk = p.awq_s + kg * kGroup + 32 * t;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const float4 s4 = __ldg(reinterpret_cast<const float4 *>(sk + 4 * c));
            const float sv[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const uint32_t w = r[0][2 * c + e];
              const float x0 = h16_to_f32<kBf16>(w & 0xFFFFu) * sv[2 * e];
              const float x1 = h16_to_f32<kBf16>(w >> 16) * sv[2 * e + 1];
              const uint32_t h0 = f32_to_h16<kBf16>(x0), h1 = f32_to_h16<kBf16>(x1);
              const uint32_t l0 = f32_to_h16<kBf16>(x0 - h16_to_f32<kBf16>(h0));
              const uint32_t l1 = f32_to_h16<kBf16>(x1 - h16_to_f32<kBf16>(h1));
              r[0][2 * c + e] = h0 | (h1 << 16);
              r[1][2 * c + e] = l0 | (l1 << 16);
              ssum += (h16_to_f32<kBf16>(h0) + h16_to_f32<kBf16>(l0)) + (h16_to_f32<kBf16>(h1) + h16_to_f32<kBf16>(l1));
            }
          }
        } else {
#pragma unroll
          for (int c = 0; c < 16; ++c) ssum += h16_to_f32<kBf16>(r[0][c] & 0xFFFFu) + h16_to_f32<kBf16>(r[0][c] >> 16);
        }
      } else {
#pragma unroll
        for (int pp = 0; pp < kParts; ++pp)
#pragma unroll
          for (int c = 0; c < 16; ++c) r[pp][c] = 0u;
      }
      // pairs for MMA block b = 2i + h: B0 = (v[8i+2h], v[8i+2h+4]), B1 = (v[8i+2h+1], v[8i+2h+5])
#pragma unroll
      for (int pp = 0; pp < kParts; ++pp)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          B[gi][o][pp][2 * i + 0][0] = __byte_perm(r[pp][4 * i + 0], r[pp][4 * i + 2], 0x5410);
          B[gi][o][pp][2 * i + 0][1] = __byte_perm(r[pp][4 * i + 0], r[pp][4 * i + 2], 0x7632);
          B[gi][o][pp][2 * i + 1][0] = __byte_perm(r[pp][4 * i + 1], r[pp][4 * i + 3], 0x5410);
          B[gi][o][pp][2 * i + 1][1] = __byte_perm(r[pp][4 * i + 1], r[pp][4 * i + 3], 0x7632);
        }
      // group sum S of x for token g, then for the C-fragment tokens 2t and 2t+1
      ssum += __shfl_xor_sync(0xffffffffu, ssum, 1);
      ssum += __shfl_xor_sync(0xffffffffu, ssum, 2);
      Sv[gi][o][0] = __shfl_sync(0xffffffffu, ssum, (2 * t) * 4);
      Sv[gi][o][1] = __shfl_sync(0xffffffffu, ssum, (2 * t + 1) * 4);
    }
  }

  // ---------------- stream the row tiles of this k-slice
  const int ra = warp * 16 + g;  // smem rows of this lane's A fragments
  const int rb = ra + 8;
  int64_t done = 0;  // tasks whose split-K partials this warp has stored
  for (int64_t j = 0; j < ntask; ++j) {
    const int s = (int)(j % Cfg::kNst);
    const uint32_t ph = (uint32_t)(j / Cfg::kNst) & 1u;
    const int64_t row0 = (blockIdx.x + j * p.grid_x) * kRows;
    if (!mbar_wait(&full[s], ph, kErrTimeoutDequant)) break;
    const uint8_t *st = smem + s * Cfg::kStage;

    float acc[T8][4];
#pragma unroll
    for (int o = 0; o < T8; ++o) acc[o][0] = acc[o][1] = acc[o][2] = acc[o][3] = 0.0f;

#pragma unroll
    for (int gi = 0; gi < KS; ++gi) {
      if (g_first + gi >= Kg) continue;
      const uint4 pa = *reinterpret_cast<const uint4 *>(st + chunk_offset<KS>(ra, gi, t));
      const uint4 pb = *reinterpret_cast<const uint4 *>(st + chunk_offset<KS>(rb, gi, t));
      uint32_t sa, sb, za, zb;
      if constexpr (kScTma) {
        const int off = (int)(g_first + gi - g0) * 2;
        sa = *reinterpret_cast<const uint16_t *>(st + Cfg::kPBytes + ra * 16 + off);
        sb = *reinterpret_cast<const uint16_t *>(st + Cfg::kPBytes + rb * 16 + off);
        za = *reinterpret_cast<const uint16_t *>(st + Cfg::kPBytes + Cfg::kSBytes + ra * 16 + off);
        zb = *reinterpret_cast<const uint16_t *>(st + Cfg::kPBytes + Cfg::kSBytes + rb * 16 + off);
      } else {
        const int64_t na = row0 + ra, nb = row0 + rb, kg = g_first + gi;
        sa = na < N ? __ldg(p.scales + na * Kg + kg) : 0u;
        sb = nb < N ? __ldg(p.scales + nb * Kg + kg) : 0u;
        za = na < N ? __ldg(p.zeros + na * Kg + kg) : 0u;
        zb = nb < N ? __ldg(p.zeros + nb * Kg + kg) : 0u;
      }
      // two independent accumulation chains (even / odd MMA blocks) halve the MMA latency chain
      float d[2][T8][4];
#pragma unroll
      for (int e = 0; e < 2; ++e)
#pragma unroll
        for (int o = 0; o < T8; ++o) d[e][o][0] = d[e][o][1] = d[e][o][2] = d[e][o][3] = 0.0f;
      const uint32_t wa[4] = {pa.x, pa.y, pa.z, pa.w};
      const uint32_t wb[4] = {pb.x, pb.y, pb.z, pb.w};
#pragma unroll
      for (int b = 0; b < 8; ++b) {
        const int i = b >> 1, h = b & 1;
        const uint32_t a0 = lop3_and_or(wa[i] >> (8 * h), 0x000F000Fu, kMagic);
        const uint32_t a2 = lop3_and_or(wa[i] >> (8 * h + 4), 0x000F000Fu, kMagic);
        const uint32_t a1 = lop3_and_or(wb[i] >> (8 * h), 0x000F000Fu, kMagic);
        const uint32_t a3 = lop3_and_or(wb[i] >> (8 * h + 4), 0x000F000Fu, kMagic);
#pragma unroll
        for (int o = 0; o < T8; ++o)
#pragma unroll
          for (int pp = 0; pp < kParts; ++pp)
            mma16816<kBf16>(d[h][o], a0, a1, a2, a3, B[gi][o][pp][b][0], B[gi][o][pp][b][1]);
      }
      const float sca = half_bits_to_float((uint16_t)sa);
      const float scb = half_bits_to_float((uint16_t)sb);
      const float ca = sca * (kOff + half_bits_to_float((uint16_t)za));
      const float cb = scb * (kOff + half_bits_to_float((uint16_t)zb));
#pragma unroll
      for (int o = 0; o < T8; ++o) {
        acc[o][0] = fmaf(-ca, Sv[gi][o][0], fmaf(sca, d[0][o][0] + d[1][o][0], acc[o][0]));
        acc[o][1] = fmaf(-ca, Sv[gi][o][1], fmaf(sca, d[0][o][1] + d[1][o][1], acc[o][1]));
        acc[o][2] = fmaf(-cb, Sv[gi][o][0], fmaf(scb, d[0][o][2] + d[1][o][2], acc[o][2]));
        acc[o][3] = fmaf(-cb, Sv[gi][o][1], fmaf(scb, d[0][o][3] + d[1][o][3], acc[o][3]));
      }
    }
    // release the stage (all lanes' shared-memory reads are consumed above)
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);

    // ---------------- outputs of this warp's 16 rows
    const int64_t blk = row0 / 16 + warp;
    if (blk >= RB16) {
      ++done;
      continue;
    }
    const int64_t rowa = row0 + ra, rowb = row0 + rb;
    if (p.kslices == 1) {
#pragma unroll
      for (int o = 0; o < T8; ++o)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int64_t row = (c < 2) ? rowa : rowb;
          const int64_t tok = o * 8 + 2 * t + (c & 1);
          if (row < N && tok < M) {
            if (p.y_bf16) static_cast<__nv_bfloat16 *>(p.Y)[tok * N + row] = __float2bfloat16_rn(acc[o][c]);
            else static_cast<float *>(p.Y)[tok * N + row] = acc[o][c];
          }
        }
    } else {
      // split-K: plain stores of this k-slice's partials; arrival is deferred to the end
#pragma unroll
      for (int o = 0; o < T8; ++o)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int64_t row = (c < 2) ? rowa : rowb;
          const int64_t tok = o * 8 + 2 * t + (c & 1);
          if (row < N && tok < M) p.ws[((int64_t)kslice * M + tok) * N + row] = acc[o][c];
        }
      ++done;
    }
  }

  // ---------------- split-K arrival: one fence for all of this warp's partials, then
  // one counter per 16-row block; the last of the k-slices to arrive sums them.
  if (p.kslices > 1 && done > 0) {
    __threadfence();
    __syncwarp();
    for (int64_t j = 0; j < done; ++j) {
      const int64_t row0 = (blockIdx.x + j * p.grid_x) * kRows;
      const int64_t blk = row0 / 16 + warp;
      if (blk >= RB16) continue;
      uint32_t prev = 0;
      if (lane == 0) prev = atomicAdd(&p.counters[blk], 1u);
      prev = __shfl_sync(0xffffffffu, prev, 0);
      if (prev != (uint32_t)(p.kslices - 1)) continue;
      __threadfence();
      const int64_t rowa = row0 + ra, rowb = row0 + rb;
#pragma unroll
      for (int o = 0; o < T8; ++o)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int64_t row = (c < 2) ? rowa : rowb;
          const int64_t tok = o * 8 + 2 * t + (c & 1);
          if (row < N && tok < M) {
            float v = 0.0f;
            for (int sl = 0; sl < p.kslices; ++sl) v += __ldcg(p.ws + ((int64_t)sl * M + tok) * N + row);
            if (p.y_bf16) static_cast<__nv_bfloat16 *>(p.Y)[tok * N + row] = __float2bfloat16_rn(v);
            else static_cast<float *>(p.Y)[tok * N + row] = v;
          }
        }
      __syncwarp();
      if (lane == 0) atomicExch(&p.counters[blk], 0u);
    }
  }
}

template <int T8, int KS, bool kBf16, bool kAwq, bool kScTma>
cudaError_t launch_t(const CUtensorMap &tmP, const CUtensorMap &tmS, const CUtensorMap &tmZ, const GemvParams &p,
                     cudaStream_t stream) {
  auto kern = gemv_kernel<T8, KS, kBf16, kAwq, kScTma>;
  constexpr int smem = GemvCfg<KS>::kSmem;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)p.grid_x, (unsigned)p.kslices);
  kern<<<grid, 160, smem, stream>>>(tmP, tmS, tmZ, p);
  return cudaGetLastError();
}

template <int T8, int KS, bool kScTma>
cudaError_t launch_d(const CUtensorMap &tmP, const CUtensorMap &tmS, const CUtensorMap &tmZ, const GemvParams &p,
                     bool bf16, cudaStream_t stream) {
  const bool awq = p.awq_s != nullptr;
  if constexpr (T8 * KS <= 4) {
    if (awq)
      return bf16 ? launch_t<T8, KS, true, true, kScTma>(tmP, tmS, tmZ, p, stream)
                  : launch_t<T8, KS, false, true, kScTma>(tmP, tmS, tmZ, p, stream);
  } else {
    if (awq) return cudaErrorNotSupported;  // AWQ with this many tokens runs on the tensor-core path
  }
  return bf16 ? launch_t<T8, KS, true, false, kScTma>(tmP, tmS, tmZ, p, stream)
              : launch_t<T8, KS, false, false, kScTma>(tmP, tmS, tmZ, p, stream);
}

template <int T8, int KS>
cudaError_t launch_s(const CUtensorMap &tmP, const CUtensorMap &tmS, const CUtensorMap &tmZ, const GemvParams &p,
                     bool bf16, bool sc_tma, cudaStream_t stream) {
  return sc_tma ? launch_d<T8, KS, true>(tmP, tmS, tmZ, p, bf16, stream)
                : launch_d<T8, KS, false>(tmP, tmS, tmZ, p, bf16, stream);
}

}  // namespace gemv_impl

// Largest KS (groups per task) whose B fragments fit the register budget.
int gemv_max_ks(int t8, bool awq) {
  const int regs_per_group = 16 * t8 * (awq ? 2 : 1);
  const int ks = 64 / regs_per_group;
  return ks >= 4 ? 4 : ks >= 2 ? 2 : 1;
}

bool gemv_supports(int64_t M, bool awq) { return M <= 64 && !(awq && M > 32); }

int gemv_smem_bytes(int ks) {
  return ks == 1 ? gemv_impl::GemvCfg<1>::kSmem : ks == 2 ? gemv_impl::GemvCfg<2>::kSmem : gemv_impl::GemvCfg<4>::kSmem;
}

cudaError_t launch_gemv(const CUtensorMap &tmP, const CUtensorMap &tmS, const CUtensorMap &tmZ, const GemvParams &p,
                        bool x_bf16, int t8, int ks, bool sc_tma, cudaStream_t stream) {
  using namespace gemv_impl;
  switch (t8) {
    case 1:
      if (ks == 4) return launch_s<1, 4>(tmP, tmS, tmZ, p, x_bf16, sc_tma, stream);
      if (ks == 2) return launch_s<1, 2>(tmP, tmS, tmZ, p, x_bf16, sc_tma, stream);
      return launch_s<1, 1>(tmP, tmS, tmZ, p, x_bf16, sc_tma, stream);
    case 2:
      if (ks == 2) return launch_s<2, 2>(tmP, tmS, tmZ, p, x_bf16, sc_tma, stream);
      return launch_s<2, 1>(tmP, tmS, tmZ, p, x_bf16, sc_tma, stream);
    case 4: return launch_s<4, 1>(tmP, tmS, tmZ, p, x_bf16, sc_tma, stream);
    default: return launch_s<8, 1>(tmP, tmS, tmZ, p, x_bf16, sc_tma, stream);
  }
}

}  // namespace w4
