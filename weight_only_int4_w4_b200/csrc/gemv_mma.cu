// gemv_mma.cu -- K1: decode / small-batch W4A16 matmul, M <= 64 tokens.
//
// Decode is bound by the weight bytes read per token, not by arithmetic
// ("LLM inference acceleration" article, section 1.1; ch. 22 "Advanced
// inference optimisation", section 22.2 table).  The kernel keeps a deep TMA
// ring in flight on every SM and spends about five integer instructions per
// eight weights on dequantization.
//
//   * Grid: (CTAs per k-slice) x (k-slices).  A CTA owns one k-slice of KR
//     quantization groups (KR x 128 input channels).  At start its 4 compute
//     warps stage the activations of that k-slice in shared memory as fp16
//     mma.sync B fragments (see "activation staging" below).
//   * Work unit ("task"): 64 output rows x the CTA's k-slice.  Row tiles are
//     handed out by an atomic counter per k-slice, so faster CTAs take more.
//     Warp 4 (producer) streams each tile's packed codes [64 rows x 128 B =
//     2 groups per stage, 128-byte swizzle] and fp16 scales / zeros [64 rows x
//     8 groups] through an NST-deep shared-memory ring with TMA; a header per
//     stage tells the compute warps which tile and k-chunk it holds.
//   * Warps 0..3 (compute) own 16 rows each.  Dequantization: a 32-bit word
//     holds 8 codes; with the fp16 magic 0x6400 one LOP3 yields the exact fp16
//     pairs 1024 + q for the low nibbles (even k) and 1024 + 16 q for the high
//     nibbles (odd k) in place, and one shift exposes the other byte pair: one
//     SHF + four LOP3 per 8 weights.  The tensor core then computes
//         D = sum_even (1024 + q) x' + sum_odd (1024 + 16 q) (x'/16)
//           = sum_k q x' + 1024 * sum_k B_k          (B = the staged fragment values)
//     exactly up to fp32 accumulation, and per group the result is promoted
//     once:  y' += scale * (D - P - z * S),  P = 1024 * sum B, S = sum x',
//     i.e. scale * sum_k (q - z) x': the dequantize-then-matmul of the
//     weight-only path (ch. 22, section 22.3) without rounding any weight.
//   * Activation staging: x' = x * s (AWQ, ch. 22 section 22.3) * 2^e, with a
//     power of two e per token and k-slice chosen so max|x'| lies in
//     [2^13, 2^14): bf16 and fp16 inputs both convert exactly to fp16 (bar
//     values 2^27 times below the token's maximum), and the result is scaled
//     back by 2^-e exactly.  With AWQ, x' is split into fp16 high + low parts.
//   * Split-K (k-slices > 1): each warp stores its fp32 partials for a tile,
//     then one lane announces them with a release atomic on the tile's 16-row
//     block counter; the ticket is read one task later (hiding the round trip)
//     and the last of the k-slices sums the partials into Y.  No warp ever
//     waits on another CTA.
//
// mma.sync m16n8k16 fragments (g = lane / 4, t = lane % 4):
//   A regs: {row g, k 2t..2t+1}, {row g+8, k 2t..}, {row g, k 2t+8..}, {row g+8, k 2t+8..}
//   B regs: {k 2t..2t+1, col g}, {k 2t+8.., col g};  C: {row g, col 2t..2t+1}, {row g+8, ...}
// The MMA's k order is a permutation of the group's 128 channels: in MMA block
// b = 2i + h, lane (g, t) takes the actual channels 32t + 8i + 2h + {0, 4}
// (even, from the low nibbles) and 32t + 8i + 2h + {1, 5} (odd, high nibbles),
// i.e. exactly the codes in the 16-byte chunk t of its own rows; the staged B
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
  int x_bf16;
  float *ws;           // [kslices][M][N] fp32 partials (split-K only)
  uint32_t *counters;  // [ceil(N/16)] split-K arrival counters
  uint32_t *sched;     // [2 * kslices]: next row tile, CTAs done fetching (per k-slice)
  int kslices;
  int kr;              // groups per k-slice (even)
  int grid_x;          // CTAs per k-slice
  int xs_bytes;        // shared-memory bytes of the staged activations
};

namespace gemv_impl {

constexpr int kRows = 64;     // rows per task (4 compute warps x 16)
constexpr int kSG = 2;        // groups per pipeline stage (128 bytes of codes per row)
constexpr int kNst = 6;       // pipeline stages
constexpr int kPBytes = kRows * kSG * 64;  // 8 KiB of codes per stage
constexpr int kSBytes = kRows * 8 * 2;     // 8-group scale (or zero) box per stage
constexpr int kStage = kPBytes + 2 * kSBytes;
constexpr int kMaxTok = 64;

// Staged activations for KR groups and M tokens: B fragments [g][tok][part][t][16 u32],
// then (P, S) float pairs [g][tok], then the per-token exponents.
__host__ __device__ constexpr int xs_frag_bytes(int kr, int m, bool awq) { return kr * m * (awq ? 2 : 1) * 4 * 64; }
__host__ __device__ constexpr int xs_bytes_for(int kr, int m, bool awq) {
  return xs_frag_bytes(kr, m, awq) + kr * m * 8 + kMaxTok * 4;
}
__host__ __device__ constexpr int smem_bytes_for(int xs_bytes) {
  return 1024 + kNst * kStage + xs_bytes + kNst * 16 + 2 * kNst * 8 + 64;
}

// D (+)= A * B on fp16 operands with fp32 accumulation; `first` starts from zero.
__device__ __forceinline__ void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1, bool first) {
  if (first) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%10,%10,%10};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.0f));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
}

__device__ __forceinline__ void named_bar_compute() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__device__ __forceinline__ void atom_release_add(uint32_t *addr, uint32_t v, uint32_t &old) {
  asm volatile("atom.add.release.gpu.global.u32 %0, [%1], %2;" : "=r"(old) : "l"(addr), "r"(v) : "memory");
}

__device__ __forceinline__ float x_to_f32(uint32_t bits16, bool bf16) {
  return bf16 ? __uint_as_float(bits16 << 16) : __half2float(__ushort_as_half((unsigned short)bits16));
}

__device__ __forceinline__ uint32_t f16_bits(float v) { return (uint32_t)__half_as_ushort(__float2half_rn(v)); }

// 2^e with e an integer in [-126, 127], exact.
__device__ __forceinline__ float exp2i(int e) { return __uint_as_float((uint32_t)(e + 127) << 23); }

template <int T8, bool kAwq, bool kScTma>
__global__ void __launch_bounds__(160) gemv_kernel(const __grid_constant__ CUtensorMap tmP,
                                                   const __grid_constant__ CUtensorMap tmS,
                                                   const __grid_constant__ CUtensorMap tmZ, const GemvParams p) {
  constexpr uint32_t kMagic = 0x64006400u;  // fp16 1024.0 in both halves
  constexpr int kParts = kAwq ? 2 : 1;      // high / low fp16 parts of x'

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int Mi = (int)p.M;
  uint8_t *stages = smem;
  uint32_t *xs = reinterpret_cast<uint32_t *>(smem + kNst * kStage);
  float2 *ps = reinterpret_cast<float2 *>(smem + kNst * kStage + xs_frag_bytes(p.kr, Mi, kAwq));
  int *xexp = reinterpret_cast<int *>(smem + kNst * kStage + xs_frag_bytes(p.kr, Mi, kAwq) + p.kr * Mi * 8);
  int *hdr = reinterpret_cast<int *>(smem + kNst * kStage + p.xs_bytes);  // [kNst][4]
  uint64_t *full = reinterpret_cast<uint64_t *>(hdr + 4 * kNst);
  uint64_t *empty = full + kNst;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t M = p.M, N = p.N, K = p.K;
  const int64_t Kg = K / kGroup;
  const int64_t RT = (N + kRows - 1) / kRows;
  const int64_t RB16 = (N + 15) / 16;
  const int kslice = blockIdx.y;
  const int64_t g_first = (int64_t)kslice * p.kr;
  const int ng = (int)min((int64_t)p.kr, Kg - g_first);  // groups of this k-slice
  const int nst_task = (ng + kSG - 1) / kSG;                 // stages per task

  if (threadIdx.x == 0) {
    for (int s = 0; s < kNst; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 4);
    }
    fence_barrier_init();
  }
  if (threadIdx.x < kMaxTok) xexp[threadIdx.x] = 0;  // max |x'| bits per token (first pass)
  __syncthreads();

  if (warp == 4) {
    // ---------------- producer: fetch row tiles, drive the TMA ring
    if (lane == 0) {
      prefetch_tensormap(&tmP);
      if (kScTma) {
        prefetch_tensormap(&tmS);
        prefetch_tensormap(&tmZ);
      }
      uint32_t *next = p.sched + 2 * kslice;
      uint32_t *fin = next + 1;
      int64_t rt = atomicAdd(next, 1u);
      int64_t it = 0;
      bool ok = true;
      while (ok) {
        const bool have = rt < RT;
        const int64_t rt_next = have ? (int64_t)atomicAdd(next, 1u) : RT;  // overlaps the issue below
        if (!have) {
          const int s = (int)(it % kNst);
          const uint32_t ph = (uint32_t)(it / kNst) & 1u;
          if (mbar_wait(&empty[s], ph ^ 1u, kErrTimeoutTma)) {
            hdr[4 * s] = -1;  // end of work
            mbar_arrive(&full[s]);
          }
          break;
        }
        const int32_t row0 = (int32_t)(rt * kRows);
        for (int c = 0; c < nst_task; ++c, ++it) {
          const int s = (int)(it % kNst);
          const uint32_t ph = (uint32_t)(it / kNst) & 1u;
          if (!mbar_wait(&empty[s], ph ^ 1u, kErrTimeoutTma)) { ok = false; break; }
          hdr[4 * s + 0] = (int)rt;
          hdr[4 * s + 1] = c;
          uint8_t *st = stages + s * kStage;
          mbar_arrive_expect_tx(&full[s], kScTma ? kStage : kPBytes);
          const int64_t gs = g_first + (int64_t)c * kSG;
          tma_load_2d(st, &tmP, &full[s], (int32_t)(gs * 64), row0);
          if constexpr (kScTma) {
            const int32_t gx0 = (int32_t)(gs & ~(int64_t)7);
            tma_load_2d(st + kPBytes, &tmS, &full[s], gx0, row0);
            tma_load_2d(st + kPBytes + kSBytes, &tmZ, &full[s], gx0, row0);
          }
        }
        rt = rt_next;
      }
      // every CTA of this k-slice is done fetching: the last one resets the scheduler
      const uint32_t prev = atomicAdd(fin, 1u);
      if (prev == gridDim.x - 1) {
        atomicExch(next, 0u);
        atomicExch(fin, 0u);
      }
    }
    return;
  }

  // ---------------- compute warps: activation staging
  const uint16_t *xg = static_cast<const uint16_t *>(p.X);
  const int units = ng * Mi * 4;  // (group, token, t): 32 channels each
  // pass 1: per-token max |x * s| over the k-slice -> power-of-two exponent
  for (int u = threadIdx.x; u < units; u += 128) {
    const int tt = u & 3;
    const int tok = (u >> 2) % Mi;
    const int gl = (u >> 2) / Mi;
    const int64_t k0 = (g_first + gl) * kGroup + 32 * tt;
    const uint16_t *src = xg + (int64_t)tok * K + k0;
    float mx = 0.0f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint4 v = __ldg(reinterpret_cast<const uint4 *>(src + 8 * c));
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        float xv = x_to_f32((w[e >> 1] >> (16 * (e & 1))) & 0xFFFFu, p.x_bf16);
        if (kAwq) xv *= __ldg(p.awq_s + k0 + 8 * c + e);
        mx = fmaxf(mx, fabsf(xv));
      }
    }
    atomicMax(&xexp[tok], __float_as_int(mx));  // non-negative floats order like their bits
  }
  named_bar_compute();
  if (threadIdx.x < Mi) {
    const int bits = xexp[threadIdx.x];
    // max|x'| in [2^13, 2^14): e = 13 - floor(log2 max); 0 for an all-zero token
    const int E = (bits >> 23) & 0xFF;  // biased exponent of the max (finite inputs)
    int e = (bits == 0) ? 0 : 13 - (E - 127);
    e = max(-100, min(100, e));
    xexp[threadIdx.x] = e;
  }
  named_bar_compute();
  // pass 2: x' = x * s * 2^e as fp16 fragments (odd channels / 16), group sums P and S.
  // Every lane runs the same number of rounds (the shuffles below need the whole
  // warp); a round's 4-lane (group, token) quads are all valid or all idle
  // because both 128 and the unit count are multiples of 4.
  for (int r0 = 0; r0 < units; r0 += 128) {
    const int u = r0 + threadIdx.x;
    const bool valid = u < units;
    const int tt = u & 3;
    const int tok = valid ? (u >> 2) % Mi : 0;
    const int gl = valid ? (u >> 2) / Mi : 0;
    const int64_t k0 = (g_first + gl) * kGroup + 32 * tt;
    const uint16_t *src = xg + (int64_t)tok * K + k0;
    const float sc2 = exp2i(xexp[tok]);
    uint32_t hbits[kParts][32];
    float sumB = 0.0f, sumX = 0.0f;
    if (valid) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint4 v = __ldg(reinterpret_cast<const uint4 *>(src + 8 * c));
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int j = 8 * c + e;  // channel offset within the 32
        float xv = x_to_f32((w[e >> 1] >> (16 * (e & 1))) & 0xFFFFu, p.x_bf16);
        if (kAwq) xv *= __ldg(p.awq_s + k0 + j);
        float xp = xv * sc2;                   // exact power-of-two scaling
        if (j & 1) xp *= 0.0625f;              // odd channels pair with 1024 + 16 q
        const uint32_t hb = f16_bits(xp);
        const float hv = __half2float(__ushort_as_half((unsigned short)hb));
        hbits[0][j] = hb;
        float used = hv;
        if constexpr (kAwq) {
          const uint32_t lb = f16_bits(xp - hv);
          hbits[kParts - 1][j] = lb;
          used += __half2float(__ushort_as_half((unsigned short)lb));
        }
        sumB += used;
        sumX += (j & 1) ? used * 16.0f : used;
      }
    }
    // B fragments for MMA block b = 2i + h: B0 = (v[8i+2h], v[8i+2h+4]), B1 = (v[8i+2h+1], v[8i+2h+5])
#pragma unroll
    for (int pp = 0; pp < kParts; ++pp) {
      uint32_t o16[16];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int base = 8 * i + 2 * h;
          o16[4 * i + 2 * h + 0] = hbits[pp][base] | (hbits[pp][base + 4] << 16);
          o16[4 * i + 2 * h + 1] = hbits[pp][base + 1] | (hbits[pp][base + 5] << 16);
        }
      uint4 *dst = reinterpret_cast<uint4 *>(xs + ((((gl * Mi + tok) * kParts + pp) * 4 + tt) * 16));
#pragma unroll
      for (int c = 0; c < 4; ++c) dst[c] = make_uint4(o16[4 * c], o16[4 * c + 1], o16[4 * c + 2], o16[4 * c + 3]);
    }
    }  // valid
    // sums over the 4 t-units of (group, token): lanes 4q..4q+3 hold them
    sumB += __shfl_xor_sync(0xffffffffu, sumB, 1);
    sumB += __shfl_xor_sync(0xffffffffu, sumB, 2);
    sumX += __shfl_xor_sync(0xffffffffu, sumX, 1);
    sumX += __shfl_xor_sync(0xffffffffu, sumX, 2);
    if (valid && tt == 0) ps[gl * Mi + tok] = make_float2(1024.0f * sumB, sumX);
  }
  named_bar_compute();

  // ---------------- stream row tiles
  const int g = lane >> 2;
  const int t = lane & 3;
  const int ra = warp * 16 + g;  // smem rows of this lane's A fragments
  const int rb = ra + 8;
  const bool split = p.kslices > 1;
  const uint32_t stage_base = smem_u32(stages);
  const uint32_t xs_base = smem_u32(xs);
  const uint32_t ps_base = smem_u32(ps);

  float acc[T8][4];
#pragma unroll
  for (int o = 0; o < T8; ++o) acc[o][0] = acc[o][1] = acc[o][2] = acc[o][3] = 0.0f;
  int64_t pend_row0 = -1;  // split-K arrival of the previous tile, read one tile later
  uint32_t pend_ticket = 0;

  auto finish_pending = [&]() {
    if (pend_row0 < 0) return;
    const uint32_t prev = __shfl_sync(0xffffffffu, pend_ticket, 0);
    if (prev == (uint32_t)(p.kslices - 1)) {
      __threadfence();
      const int64_t blk = pend_row0 / 16 + warp;
#pragma unroll
      for (int o = 0; o < T8; ++o)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int64_t row = pend_row0 + ((c < 2) ? ra : rb);
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
    pend_row0 = -1;
  };

  // per-lane constant parts of the shared-memory addresses
  const uint32_t a_off0 = (uint32_t)(ra * 128), b_off0 = (uint32_t)(rb * 128);
  const uint32_t sw_a = (uint32_t)(ra & 7), sw_b = (uint32_t)(rb & 7);

  for (int64_t it = 0;; ++it) {
    const int s = (int)(it % kNst);
    const uint32_t ph = (uint32_t)(it / kNst) & 1u;
    if (!mbar_wait(&full[s], ph, kErrTimeoutDequant)) break;
    const int rt = hdr[4 * s + 0];
    if (rt < 0) break;
    const int c = hdr[4 * s + 1];
    const uint32_t st = stage_base + (uint32_t)(s * kStage);
    const int64_t row0 = (int64_t)rt * kRows;
    const int ngs = min(kSG, ng - c * kSG);  // groups in this stage (warp-uniform)

#pragma unroll
    for (int gl2 = 0; gl2 < kSG; ++gl2) {
      if (gl2 >= ngs) break;
      const int gl = c * kSG + gl2;  // group within the k-slice
      const uint32_t chunk = (uint32_t)(gl2 * 4 + t);
      const uint4 pa = lds128(st + a_off0 + ((chunk ^ sw_a) << 4));
      const uint4 pb = lds128(st + b_off0 + ((chunk ^ sw_b) << 4));
      uint32_t sa, sb, za, zb;
      const int64_t kg = g_first + gl;
      if constexpr (kScTma) {
        const uint32_t off = (uint32_t)(kg & 7) * 2;
        sa = lds_u16(st + kPBytes + ra * 16 + off);
        sb = lds_u16(st + kPBytes + rb * 16 + off);
        za = lds_u16(st + kPBytes + kSBytes + ra * 16 + off);
        zb = lds_u16(st + kPBytes + kSBytes + rb * 16 + off);
      } else {
        const int64_t na = row0 + ra, nb = row0 + rb;
        sa = na < N ? __ldg(p.scales + na * Kg + kg) : 0u;
        sb = nb < N ? __ldg(p.scales + nb * Kg + kg) : 0u;
        za = na < N ? __ldg(p.zeros + na * Kg + kg) : 0u;
        zb = nb < N ? __ldg(p.zeros + nb * Kg + kg) : 0u;
      }
      // A fragments: one SHF + four LOP3 per 32-bit word (8 codes)
      uint32_t A[8][4];
      const uint32_t wa[4] = {pa.x, pa.y, pa.z, pa.w};
      const uint32_t wb[4] = {pb.x, pb.y, pb.z, pb.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t wa8 = wa[i] >> 8, wb8 = wb[i] >> 8;
        A[2 * i][0] = lop3_and_or(wa[i], 0x000F000Fu, kMagic);
        A[2 * i][2] = lop3_and_or(wa[i], 0x00F000F0u, kMagic);
        A[2 * i][1] = lop3_and_or(wb[i], 0x000F000Fu, kMagic);
        A[2 * i][3] = lop3_and_or(wb[i], 0x00F000F0u, kMagic);
        A[2 * i + 1][0] = lop3_and_or(wa8, 0x000F000Fu, kMagic);
        A[2 * i + 1][2] = lop3_and_or(wa8, 0x00F000F0u, kMagic);
        A[2 * i + 1][1] = lop3_and_or(wb8, 0x000F000Fu, kMagic);
        A[2 * i + 1][3] = lop3_and_or(wb8, 0x00F000F0u, kMagic);
      }
      const float sca = half_bits_to_float((uint16_t)sa);
      const float scb = half_bits_to_float((uint16_t)sb);
      const float zfa = half_bits_to_float((uint16_t)za);
      const float zfb = half_bits_to_float((uint16_t)zb);
#pragma unroll
      for (int o = 0; o < T8; ++o) {
        if (o * 8 >= Mi) break;  // octet without real tokens (warp-uniform)
        const int tok = o * 8 + g;
        float d0[4], d1[4];
#pragma unroll
        for (int pp = 0; pp < kParts; ++pp) {
          uint32_t Bv[16];
          if (tok < Mi) {
            const uint32_t bad = xs_base + (uint32_t)(((((gl * Mi + tok) * kParts + pp) * 4 + t) * 16) * 4);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint4 v = lds128(bad + 16 * q);
              Bv[4 * q] = v.x; Bv[4 * q + 1] = v.y; Bv[4 * q + 2] = v.z; Bv[4 * q + 3] = v.w;
            }
          } else {
#pragma unroll
            for (int q = 0; q < 16; ++q) Bv[q] = 0u;
          }
#pragma unroll
          for (int b = 0; b < 8; ++b) {
            if (b & 1) mma_f16(d1, A[b], Bv[2 * b], Bv[2 * b + 1], pp == 0 && b == 1);
            else mma_f16(d0, A[b], Bv[2 * b], Bv[2 * b + 1], pp == 0 && b == 0);
          }
        }
        // promotion: y' += scale * (D - P - z S) for tokens 2t, 2t+1 of this octet
        const int t0 = o * 8 + 2 * t;
        float2 q0 = make_float2(0.f, 0.f), q1 = make_float2(0.f, 0.f);
        if (t0 < Mi) q0 = lds_f2(ps_base + (uint32_t)((gl * Mi + t0) * 8));
        if (t0 + 1 < Mi) q1 = lds_f2(ps_base + (uint32_t)((gl * Mi + t0 + 1) * 8));
        acc[o][0] = fmaf(-sca, fmaf(zfa, q0.y, q0.x), fmaf(sca, d0[0] + d1[0], acc[o][0]));
        acc[o][1] = fmaf(-sca, fmaf(zfa, q1.y, q1.x), fmaf(sca, d0[1] + d1[1], acc[o][1]));
        acc[o][2] = fmaf(-scb, fmaf(zfb, q0.y, q0.x), fmaf(scb, d0[2] + d1[2], acc[o][2]));
        acc[o][3] = fmaf(-scb, fmaf(zfb, q1.y, q1.x), fmaf(scb, d0[3] + d1[3], acc[o][3]));
      }
    }
    // release the stage (all lanes' shared-memory reads are consumed above)
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    if (c != nst_task - 1) continue;

    // ---------------- tile done: outputs of this warp's 16 rows (scaled back by 2^-e)
    finish_pending();
    const int64_t blk = row0 / 16 + warp;
    if (blk < RB16) {
      const int64_t rowa = row0 + ra, rowb = row0 + rb;
#pragma unroll
      for (int o = 0; o < T8; ++o)
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const int64_t row = (cc < 2) ? rowa : rowb;
          const int tok = o * 8 + 2 * t + (cc & 1);
          if (row < N && tok < Mi) {
            const float v = acc[o][cc] * exp2i(-xexp[tok]);
            if (!split) {
              if (p.y_bf16) static_cast<__nv_bfloat16 *>(p.Y)[(int64_t)tok * N + row] = __float2bfloat16_rn(v);
              else static_cast<float *>(p.Y)[(int64_t)tok * N + row] = v;
            } else {
              p.ws[((int64_t)kslice * M + tok) * N + row] = v;
            }
          }
        }
      if (split) {
        // announce the partials: warp barrier, then one release atomic (read one tile later)
        __syncwarp();
        if (lane == 0) atom_release_add(&p.counters[blk], 1u, pend_ticket);
        pend_row0 = row0;
      }
    }
#pragma unroll
    for (int o = 0; o < T8; ++o) acc[o][0] = acc[o][1] = acc[o][2] = acc[o][3] = 0.0f;
  }
  finish_pending();
}

template <int T8, bool kAwq, bool kScTma>
cudaError_t launch_t(const CUtensorMap &tmP, const CUtensorMap &tmS, const CUtensorMap &tmZ, const GemvParams &p,
                     cudaStream_t stream) {
  auto kern = gemv_kernel<T8, kAwq, kScTma>;
  const int smem = smem_bytes_for(p.xs_bytes);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)p.grid_x, (unsigned)p.kslices);
  kern<<<grid, 160, smem, stream>>>(tmP, tmS, tmZ, p);
  return cudaGetLastError();
}

template <int T8>
cudaError_t launch_s(const CUtensorMap &tmP, const CUtensorMap &tmS, const CUtensorMap &tmZ, const GemvParams &p,
                     bool sc_tma, cudaStream_t stream) {
  if (p.awq_s)
    return sc_tma ? launch_t<T8, true, true>(tmP, tmS, tmZ, p, stream) : launch_t<T8, true, false>(tmP, tmS, tmZ, p, stream);
  return sc_tma ? launch_t<T8, false, true>(tmP, tmS, tmZ, p, stream) : launch_t<T8, false, false>(tmP, tmS, tmZ, p, stream);
}

}  // namespace gemv_impl

bool gemv_supports(int64_t M, bool awq) { return M <= 64 && !(awq && M > 32); }

// Shared-memory bytes of the staged activations for a k-slice of kr groups.
int gemv_xs_bytes(int kr, int64_t M, bool awq) { return gemv_impl::xs_bytes_for(kr, (int)M, awq); }
int gemv_smem_bytes(int xs_bytes) { return gemv_impl::smem_bytes_for(xs_bytes); }

cudaError_t launch_gemv(const CUtensorMap &tmP, const CUtensorMap &tmS, const CUtensorMap &tmZ, const GemvParams &p,
                        int t8, bool sc_tma, cudaStream_t stream) {
  using namespace gemv_impl;
  switch (t8) {
    case 1: return launch_s<1>(tmP, tmS, tmZ, p, sc_tma, stream);
    case 2: return launch_s<2>(tmP, tmS, tmZ, p, sc_tma, stream);
    case 4: return launch_s<4>(tmP, tmS, tmZ, p, sc_tma, stream);
    default: return launch_s<8>(tmP, tmS, tmZ, p, sc_tma, stream);
  }
}

}  // namespace w4
