// gemv_mma.cu -- K1: decode / small-batch W4A16 matmul, M <= 64 tokens.
//
// Decode is bound by the weight bytes read per token, not by arithmetic
// ("LLM inference acceleration" article, section 1.1; ch. 22 "Advanced
// inference optimisation", section 22.2 table).  The kernel keeps a deep TMA
// ring in flight on every SM and spends about nine instructions per eight
// weights on dequantization.
//
//   * Grid: (CTAs per k-slice) x (k-slices).  A CTA owns one k-slice of KR
//     quantization groups (KR x 128 input channels).  At start its compute
//     warps stage the activations of that k-slice in shared memory as fp16
//     mma.sync B fragments (see "activation staging" below).
//   * Work: the iterations of a k-slice are its (64-row tile, 4-group stage)
//     pairs in tile-major order; CTA c of the slice's C CTAs takes a fixed,
//     contiguous, balanced range of them (no scheduling atomics).  Warp 8
//     (producer) streams each stage's packed codes [64 rows x 256 B = 4 groups,
//     two 128-byte-swizzled boxes] and fp16 scales / zeros [64 rows x 8 groups]
//     through an NST-deep shared-memory ring with TMA; a header per stage tells
//     the compute warps which tile and stage it holds.
//   * Warps 0..7 (compute): warp (b, h) owns rows 16b..16b+15 of the tile and
//     groups 2h, 2h+1 of every stage (two independent MMA streams).  A 32-bit
//     word holds 8 codes; with the fp16 magic 0x6400 one LOP3 yields the exact
//     fp16 pairs 1024 + q for the low nibbles (even k) and 1024 + 16 q for the
//     high nibbles (odd k) in place, one shift exposes the other byte pair, and
//     one fp16x2 subtraction of 1024 + z (low) or 1024 + 16 z (high) leaves the
//     exact integers q - z and 16 (q - z): one SHF + four LOP3 + four HSUB2 per
//     8 weights.  The tensor core then computes, per group,
//         D = sum_even (q - z) x' + sum_odd 16 (q - z) (x'/16) = sum_k (q - z) x'
//     from exact products with fp32 accumulation, and the group is promoted
//     once:  y' += scale * D -- the dequantize-then-matmul of the weight-only
//     path (ch. 22, section 22.3) without rounding any weight.  A row whose
//     codes equal its zero point contributes exactly 0.
//     At the end of a tile the two warps of a row block add their halves
//     through shared memory (bounded mbarrier hand-off).
//   * Activation staging: x' = x * s (AWQ, ch. 22 section 22.3) * 2^e, with a
//     power of two e per token and k-slice chosen so max|x'| lies in
//     [2^13, 2^14): bf16 and fp16 inputs both convert exactly to fp16 (bar
//     values 2^27 times below the token's maximum), and the result is scaled
//     back by 2^-e exactly.  With AWQ, x * s is rounded to fp16 (at most 2^-11
//     relative per product).
//   * Shared row tiles and split-K: a CTA that holds only part of a row tile
//     (or a k-slice of it) stores its fp32 partials, then one lane announces
//     them with a release atomic on the 16-row block's counter; the ticket is
//     read one tile later (hiding the round trip) and the last contributor sums
//     every partial in a fixed order into Y.  No warp ever waits on another CTA.
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
  float *ws;           // [kslices][slots][M][N] fp32 partials (row tiles shared by CTAs)
  uint32_t *counters;  // [ceil(N/16)] split-K arrival counters
  int kslices;
  int slots;           // partial slots per k-slice and row tile (see the static partition)
  int kr;              // groups per k-slice (multiple of 4)
  int grid_x;          // CTAs per k-slice
  int xs_bytes;        // shared-memory bytes of the staged activations
};

namespace gemv_impl {

constexpr int kRows = 64;      // rows per task
constexpr int kSG = 4;         // groups per pipeline stage (256 bytes of codes per row)
constexpr int kNst = 5;        // pipeline stages (5 x 18 KiB in flight per CTA)
constexpr int kBox = kRows * 128;          // one 128-byte-swizzled box: 2 groups x 64 rows
constexpr int kPBytes = 2 * kBox;          // 16 KiB of codes per stage
constexpr int kSBytes = kRows * 8 * 2;     // 8-group scale (or zero) box per stage
constexpr int kStage = kPBytes + 2 * kSBytes;
constexpr int kMaxTok = 64;
constexpr int kComputeWarps = 8;
constexpr int kComputeThreads = kComputeWarps * 32;

// Staged activations for KR groups and M tokens: B fragments [g][tok][part][t][16 u32],
// then the per-token exponents.
__host__ __device__ constexpr int xs_frag_bytes(int kr, int m, bool) { return kr * m * 4 * 64; }
__host__ __device__ constexpr int xs_bytes_for(int kr, int m, bool awq) {
  return xs_frag_bytes(kr, m, awq) + kMaxTok * 4;
}
// pair-reduction buffer: [4 row blocks][32 lanes][T8 octets][4] floats
__host__ __device__ constexpr int pair_bytes_for(int t8) { return 4 * 32 * t8 * 4 * 4; }
__host__ __device__ constexpr int smem_bytes_for(int xs_bytes, int t8) {
  return 1024 + kNst * kStage + xs_bytes + pair_bytes_for(t8) + kNst * 16 + 2 * kNst * 8 + 8 * 8 + 64;
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

__device__ __forceinline__ void named_bar_compute() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

__device__ __forceinline__ void atom_release_add(uint32_t *addr, uint32_t v, uint32_t &old) {
  asm volatile("atom.add.release.gpu.global.u32 %0, [%1], %2;" : "=r"(old) : "l"(addr), "r"(v) : "memory");
}

// Two 16-bit inputs of a 32-bit word (channel 2j in the low half) -> two floats.
template <bool kBf16>
__device__ __forceinline__ float2 pair_to_f32(uint32_t w) {
  if constexpr (kBf16) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
  } else {
    return __half22float2(*reinterpret_cast<const __half2 *>(&w));
  }
}

// fp32 pair -> fp16x2 word (round to nearest even), low half = first.
__device__ __forceinline__ uint32_t f16x2_bits(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t *>(&h);
}

// fp16x2 a - b.  Used on exact small integers only (1024 + q minus 1024 + z),
// so the result is exact whatever the rounding mode.
__device__ __forceinline__ uint32_t hsub2_bits(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("sub.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// Exact fp16 pair (q - z) (low nibbles: mask 0x000F000F, zc = 1024 + z in both
// halves) or 16 (q - z) (high nibbles: mask 0x00F000F0, zc = 1024 + 16 z).
__device__ __forceinline__ uint32_t dq_pair(uint32_t w, uint32_t mask, uint32_t zc) {
  return hsub2_bits(lop3_and_or(w, mask, 0x64006400u), zc);
}

// 2^e with e an integer in [-126, 127], exact.
__device__ __forceinline__ float exp2i(int e) { return __uint_as_float((uint32_t)(e + 127) << 23); }

// Static balanced partition of a k-slice's work.  The iterations of a k-slice
// are its (row tile, stage) pairs in tile-major order, T = RT * S of them; CTA
// c of the slice's C CTAs takes iterations [floor(c T / C), floor((c+1) T / C)).
// The planner keeps C <= T, so every range is non-empty.
// (32-bit arithmetic whenever the products fit, which is every realistic layer.)
__device__ __forceinline__ int64_t part_begin(int64_t c, int64_t T, int64_t C) {
  if (T * C < (int64_t(1) << 32)) return (int64_t)((uint32_t)(c * T) / (uint32_t)C);
  return (c * T) / C;
}
// The CTA whose range holds iteration i.
__device__ __forceinline__ int64_t part_owner(int64_t i, int64_t T, int64_t C) {
  if (T * C < (int64_t(1) << 32)) return (int64_t)((uint32_t)((i + 1) * C - 1) / (uint32_t)T);
  return ((i + 1) * C - 1) / T;
}
// Stages of k-slice ks (the last slice may hold fewer groups).
__device__ __forceinline__ int64_t slice_stages(int ks, int kr, int64_t Kg) {
  const int64_t ng = min((int64_t)kr, Kg - (int64_t)ks * kr);
  return (ng + kSG - 1) / kSG;
}
// CTAs of k-slice ks that hold part of row tile rt, and the first of them.
__device__ __forceinline__ void tile_owners(int64_t rt, int64_t RT, int64_t C, int ks, int kr, int64_t Kg,
                                            int64_t &first, int64_t &count) {
  const int64_t S = slice_stages(ks, kr, Kg);
  const int64_t T = RT * S;
  first = part_owner(rt * S, T, C);
  count = part_owner(rt * S + S - 1, T, C) - first + 1;
}

template <int T8, bool kBf16, bool kAwq, bool kScTma>
__global__ void __launch_bounds__(288, (T8 <= 2 ? 2 : 1)) gemv_kernel(const __grid_constant__ CUtensorMap tmP,
                                                   const __grid_constant__ CUtensorMap tmS,
                                                   const __grid_constant__ CUtensorMap tmZ, const GemvParams p) {
  constexpr int kParts = 1;  // x' (x * s with AWQ) staged as one fp16 value per channel

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int Mi = (int)p.M;
  uint8_t *stages = smem;
  uint32_t *xs = reinterpret_cast<uint32_t *>(smem + kNst * kStage);
  int *xexp = reinterpret_cast<int *>(smem + kNst * kStage + xs_frag_bytes(p.kr, Mi, kAwq));
  float *pairbuf = reinterpret_cast<float *>(smem + kNst * kStage + p.xs_bytes);  // [4][32][T8][4]
  int *hdr = reinterpret_cast<int *>(smem + kNst * kStage + p.xs_bytes + pair_bytes_for(T8));  // [kNst][4]
  uint64_t *full = reinterpret_cast<uint64_t *>(hdr + 4 * kNst);
  uint64_t *empty = full + kNst;
  uint64_t *pair_full = empty + kNst;    // [4]
  uint64_t *pair_empty = pair_full + 4;  // [4]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t M = p.M, N = p.N, K = p.K;
  const int64_t Kg = K / kGroup;
  const int64_t RT = (N + kRows - 1) / kRows;
  const int64_t RB16 = (N + 15) / 16;
  const int kslice = blockIdx.y;
  const int64_t g_first = (int64_t)kslice * p.kr;
  const int ng = (int)min((int64_t)p.kr, Kg - g_first);  // groups of this k-slice
  const int S = (ng + kSG - 1) / kSG;                       // stages per row tile
  const int ng_pad = S * kSG;                               // staged groups (zero beyond ng)

  if (threadIdx.x == 0) {
    for (int s = 0; s < kNst; ++s) {
      mbar_init(&full[s], 2);  // the expect-tx arrival, then the header's
      mbar_init(&empty[s], kComputeWarps);
    }
    for (int b = 0; b < 4; ++b) {
      mbar_init(&pair_full[b], 1);
      mbar_init(&pair_empty[b], 1);
    }
    fence_barrier_init();
  }
  if (threadIdx.x < kMaxTok) xexp[threadIdx.x] = 0;  // max |x'| bits per token (first pass)
  __syncthreads();

  if (warp == kComputeWarps) {
    // ---------------- producer: walk this CTA's iteration range, drive the TMA ring.
    // Lanes 0..3 each issue one box of every stage (the two code boxes, then the
    // scale and zero boxes) in the same instruction: a CTA whose boxes come from
    // one issuing thread streams at well under the HBM rate on B200, while boxes
    // issued by separate lanes are in flight together.
    // Weights are never written by a preceding kernel, so nothing here waits for it.
    if (lane < 4) {
      if (lane == 0) {
        prefetch_tensormap(&tmP);
        if (kScTma) {
          prefetch_tensormap(&tmS);
          prefetch_tensormap(&tmZ);
        }
      }
      const int64_t C = gridDim.x;
      const int64_t T = RT * S;
      const int64_t it1 = part_begin((int64_t)blockIdx.x + 1, T, C);
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int64_t it = part_begin(blockIdx.x, T, C); ok && it < it1;) {
        const int64_t rt = it / S;
        const int c0 = (int)(it - rt * S);
        const int64_t frag_end = min(it1, (rt + 1) * (int64_t)S);
        const int c1 = (int)(frag_end - rt * S);
        const bool direct = c0 == 0 && c1 == S && p.kslices == 1;
        const int32_t row0 = (int32_t)(rt * kRows);
        for (int c = c0; c < c1; ++c) {
          // every issuing lane waits for the free slot itself; the vote keeps the
          // four lanes on one path if a wait ever gives up
          const bool w_ok = mbar_wait(&empty[s], ph ^ 1u, kErrTimeoutTma);
          if (!__all_sync(0xFu, w_ok)) { ok = false; break; }
          uint8_t *st = stages + s * kStage;
          if (lane == 0) mbar_arrive_expect_tx(&full[s], kScTma ? kStage : kPBytes);
          __syncwarp(0xFu);
          const int64_t gs = g_first + (int64_t)c * kSG;
          if (lane < 2) {
            tma_load_2d(st + lane * kBox, &tmP, &full[s], (int32_t)(gs * 64 + 128 * lane), row0);
          } else if (kScTma) {
            const int32_t gx0 = (int32_t)(gs & ~(int64_t)7);
            tma_load_2d(st + kPBytes + (lane - 2) * kSBytes, lane == 2 ? &tmS : &tmZ, &full[s], gx0, row0);
          }
          if (lane == 0) {
            // Header: the fragment's place among the row tile's contributors is only
            // read at its last stage, so it is worked out after that stage's loads.
            int slot = 0, ntotal = 0;
            if (c == c1 - 1 && !direct) {
              int64_t first, count;
              tile_owners(rt, RT, C, kslice, p.kr, Kg, first, count);
              slot = (int)((int64_t)blockIdx.x - first);
              for (int ks = 0; ks < p.kslices; ++ks) {
                tile_owners(rt, RT, C, ks, p.kr, Kg, first, count);
                ntotal += (int)count;
              }
            }
            hdr[4 * s + 0] = (int)rt;
            hdr[4 * s + 1] = c | ((c == c1 - 1) ? (1 << 16) : 0);
            hdr[4 * s + 2] = slot | (direct ? (1 << 16) : 0);
            hdr[4 * s + 3] = ntotal;
            mbar_arrive(&full[s]);
          }
          if (++s == kNst) {
            s = 0;
            ph ^= 1u;
          }
        }
        it = frag_end;
      }
      if (lane == 0 && ok && mbar_wait(&empty[s], ph ^ 1u, kErrTimeoutTma)) {
        hdr[4 * s] = -1;  // end of work (no loads: both arrivals here)
        mbar_arrive(&full[s]);
        mbar_arrive(&full[s]);
      }
      // All of this CTA's loads are issued: let the next kernel in the stream start
      // launching.  (Triggering at CTA start measured slower on B200: consecutive
      // kernels then pile their CTAs onto the same SMs and compete for issue slots.)
      if (lane == 0) grid_launch_dependents();
    }
    return;
  }

  // ---------------- compute warps: activation staging.  A unit is 32 channels
  // (group gl, token tok, quarter tt); every lane runs the same number of rounds
  // (the shuffles need whole warps) and a round's 4-lane quads are all valid or
  // all idle, since the thread count and the unit count are multiples of 4.
  // Groups ng..ng_pad-1 (past the end of the k-slice) are staged as zeros, so a
  // stage always holds whole groups that contribute exactly 0.
  grid_dependency_wait();  // X (and Y, the workspace) may come from the preceding kernel
  const uint16_t *xg = static_cast<const uint16_t *>(p.X);
  const int units = ng * Mi * 4;
  const int units_pad = ng_pad * Mi * 4;
  // Unit u -> (group gl, token tok, quarter tt); its 32 channels start at k0.
  auto unit_src = [&](int u) -> const uint4 * {
    const int tt = u & 3, tok = (u >> 2) % Mi, gl = (u >> 2) / Mi;
    return reinterpret_cast<const uint4 *>(xg + (int64_t)tok * K + (g_first + gl) * kGroup + 32 * tt);
  };
  auto unit_max = [&](int u, const uint32_t (&w)[16]) {  // max |x * s| of the unit -> its token's running max
    const int tt = u & 3, tok = (u >> 2) % Mi, gl = (u >> 2) / Mi;
    const int64_t k0 = (g_first + gl) * kGroup + 32 * tt;
    float mx = 0.0f;
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      float2 f = pair_to_f32<kBf16>(w[e]);
      if constexpr (kAwq) {
        const float2 s2 = __ldg(reinterpret_cast<const float2 *>(p.awq_s + k0 + 2 * e));
        f.x *= s2.x;
        f.y *= s2.y;
      }
      mx = fmaxf(mx, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
    atomicMax(&xexp[tok], __float_as_int(mx));  // non-negative floats order like their bits
  };
  // x' = x * s * 2^e as fp16 B fragments (odd channels / 16).  Units past units_pad
  // are idle, and units of the zero padding (gl >= ng) write zeros.
  auto unit_convert = [&](int u, const uint32_t (&w)[16]) {
    const bool valid = u < units_pad;
    const int tt = u & 3;
    const int tok = valid ? (u >> 2) % Mi : 0;
    const int gl = valid ? (u >> 2) / Mi : 0;
    const bool real = valid && gl < ng;
    if (valid) {
      uint32_t hw[kParts][16];  // fp16 pairs (channels 2j, 2j+1) of the 32
#pragma unroll
      for (int pp = 0; pp < kParts; ++pp)
#pragma unroll
        for (int j = 0; j < 16; ++j) hw[pp][j] = 0u;
      if (real) {
        const int64_t k0 = (g_first + gl) * kGroup + 32 * tt;
        const int e = xexp[tok];
        const float se = exp2i(e), so = exp2i(e - 4);  // even channels x 2^e, odd x 2^(e-4)
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          float2 f = pair_to_f32<kBf16>(w[j]);
          if constexpr (kAwq) {
            const float2 s2 = __ldg(reinterpret_cast<const float2 *>(p.awq_s + k0 + 2 * j));
            f.x *= s2.x;
            f.y *= s2.y;
          }
          f.x *= se;  // exact power-of-two scaling
          f.y *= so;
          // With AWQ, x * s is rounded to fp16 here (at most 2^-11 relative per
          // product, well inside the accuracy bound).
          hw[0][j] = f16x2_bits(f.x, f.y);
        }
      }
      // B fragments for MMA block b = 2i + h: B0 = (v[8i+2h], v[8i+2h+4]), B1 = (v[8i+2h+1], v[8i+2h+5]);
      // word 4i + h holds channels (8i+2h, 8i+2h+1) and word 4i + h + 2 holds (8i+2h+4, 8i+2h+5)
#pragma unroll
      for (int pp = 0; pp < kParts; ++pp) {
        uint32_t o16[16];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint32_t wa = hw[pp][4 * i + h], wb = hw[pp][4 * i + h + 2];
            o16[4 * i + 2 * h + 0] = __byte_perm(wa, wb, 0x5410);
            o16[4 * i + 2 * h + 1] = __byte_perm(wa, wb, 0x7632);
          }
        uint4 *dst = reinterpret_cast<uint4 *>(xs + ((((gl * Mi + tok) * kParts + pp) * 4 + tt) * 16));
#pragma unroll
        for (int c = 0; c < 4; ++c) dst[c] = make_uint4(o16[4 * c], o16[4 * c + 1], o16[4 * c + 2], o16[4 * c + 3]);
      }
    }
  };
  auto load_unit = [&](int u, uint32_t (&w)[16]) {
    const uint4 *src = unit_src(u);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint4 v = __ldg(src + c);
      w[4 * c] = v.x; w[4 * c + 1] = v.y; w[4 * c + 2] = v.z; w[4 * c + 3] = v.w;
    }
  };
  auto set_exponents = [&]() {
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
  };
  if (!kAwq && units_pad <= 2 * kComputeThreads) {
    // one read of X: both rounds' words stay in registers across the exponent step
    uint32_t w0[16], w1[16];
    const int u0 = threadIdx.x, u1 = kComputeThreads + threadIdx.x;
    if (u0 < units) { load_unit(u0, w0); unit_max(u0, w0); }
    if (u1 < units) { load_unit(u1, w1); unit_max(u1, w1); }
    set_exponents();
    unit_convert(u0, w0);
    if (units_pad > kComputeThreads) unit_convert(u1, w1);
  } else {
    // pass 1: per-token max over the k-slice; pass 2 reads X again and converts
    for (int r0 = 0; r0 < units; r0 += kComputeThreads) {
      const int u = r0 + threadIdx.x;
      if (u < units) {
        uint32_t w[16];
        load_unit(u, w);
        unit_max(u, w);
      }
    }
    set_exponents();
    for (int r0 = 0; r0 < units_pad; r0 += kComputeThreads) {
      const int u = r0 + threadIdx.x;
      uint32_t w[16];
      if (u < units) load_unit(u, w);
      else {
#pragma unroll
        for (int j = 0; j < 16; ++j) w[j] = 0u;
      }
      unit_convert(u, w);
    }
  }
  named_bar_compute();

  // ---------------- consume stages
  const int g = lane >> 2;
  const int t = lane & 3;
  const int blk4 = warp & 3;     // 16-row block of the tile
  const int half = warp >> 2;    // this warp takes groups 2*half, 2*half+1 of every stage
  const int ra = blk4 * 16 + g;  // smem rows of this lane's A fragments
  const int rb = ra + 8;
  const int kslices = p.kslices;
  const uint32_t stage_base = smem_u32(stages);
  const uint32_t xs_base = smem_u32(xs);

  float acc[T8][4];
#pragma unroll
  for (int o = 0; o < T8; ++o) acc[o][0] = acc[o][1] = acc[o][2] = acc[o][3] = 0.0f;
  int64_t frags_done = 0;
  int64_t pend_row0 = -1;  // arrival of the previous fragment's partials, read one fragment later
  int pend_total = 0;
  uint32_t pend_ticket = 0;

  // The last contributor of a row block sums every k-slice's and every
  // fragment's partials in a fixed order (slice-major, then fragment), so the
  // result does not depend on which CTA finishes last.
  auto finish_pending = [&]() {
    if (pend_row0 < 0) return;
    const uint32_t prev = __shfl_sync(0xffffffffu, pend_ticket, 0);
    if (prev == (uint32_t)(pend_total - 1)) {
      __threadfence();
      const int64_t blk = pend_row0 / 16 + blk4;
      const int64_t rt = pend_row0 / kRows;
      float v[T8][4];
#pragma unroll
      for (int o = 0; o < T8; ++o) v[o][0] = v[o][1] = v[o][2] = v[o][3] = 0.0f;
      for (int ks = 0; ks < kslices; ++ks) {
        int64_t first, count;
        tile_owners(rt, RT, (int64_t)gridDim.x, ks, p.kr, Kg, first, count);
        for (int64_t sl = 0; sl < count; ++sl) {
          const float *base = p.ws + ((int64_t)ks * p.slots + sl) * M * N;
#pragma unroll
          for (int o = 0; o < T8; ++o)
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const int64_t row = pend_row0 + ((c < 2) ? ra : rb);
              const int64_t tok = o * 8 + 2 * t + (c & 1);
              if (row < N && tok < M) v[o][c] += __ldcg(base + tok * N + row);
            }
        }
      }
#pragma unroll
      for (int o = 0; o < T8; ++o)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int64_t row = pend_row0 + ((c < 2) ? ra : rb);
          const int64_t tok = o * 8 + 2 * t + (c & 1);
          if (row < N && tok < M) {
            if (p.y_bf16) static_cast<__nv_bfloat16 *>(p.Y)[tok * N + row] = __float2bfloat16_rn(v[o][c]);
            else static_cast<float *>(p.Y)[tok * N + row] = v[o][c];
          }
        }
      __syncwarp();
      if (lane == 0) atomicExch(&p.counters[blk], 0u);
    }
    pend_row0 = -1;
  };

  // per-lane constants: every shared-memory address below is one of these plus a
  // per-stage or per-group increment (no index arithmetic in the hot loop)
  const int Mi1 = Mi - 1;
  const int g_first_i = (int)g_first;
  const uint32_t box_off = (uint32_t)(half * kBox);
  const uint32_t a_off0 = box_off + (uint32_t)(ra * 128) + (((uint32_t)t ^ (uint32_t)(ra & 7)) << 4);
  const uint32_t a_off1 = box_off + (uint32_t)(ra * 128) + (((uint32_t)(4 + t) ^ (uint32_t)(ra & 7)) << 4);
  const uint32_t b_off0 = box_off + (uint32_t)(rb * 128) + (((uint32_t)t ^ (uint32_t)(rb & 7)) << 4);
  const uint32_t b_off1 = box_off + (uint32_t)(rb * 128) + (((uint32_t)(4 + t) ^ (uint32_t)(rb & 7)) << 4);
  const uint32_t sa_off = (uint32_t)(kPBytes + ra * 16), sb_off = (uint32_t)(kPBytes + rb * 16);
  const uint32_t gstride_x = (uint32_t)(Mi * kParts * 256);  // staged-fragment bytes per group
  // Token columns beyond M read a real token's data (clamped): a B column only
  // feeds its own D column, and those columns are never stored.
  uint32_t bofs[T8];
#pragma unroll
  for (int o = 0; o < T8; ++o) {
    const int tb = min(o * 8 + g, Mi1);
    bofs[o] = xs_base + (uint32_t)(tb * kParts * 256 + t * 64);
  }
  const uint32_t hdr_base = smem_u32(hdr);

  int s = 0;
  uint32_t ph = 0;
  for (;;) {
    if (!mbar_wait(&full[s], ph, kErrTimeoutDequant)) break;
    int rt, cw, sw, ntotal;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(rt), "=r"(cw), "=r"(sw), "=r"(ntotal)
                 : "r"(hdr_base + (uint32_t)(s * 16)));
    if (rt < 0) break;
    const int c = cw & 0xFFFF;
    const bool last = (cw >> 16) != 0;
    const uint32_t st = stage_base + (uint32_t)(s * kStage);
    const int gl0 = c * kSG + 2 * half;  // first of this warp's two groups (both < ng_pad)

    // packed codes: one 16-byte chunk per row and group
    const uint4 pa0 = lds128(st + a_off0), pb0 = lds128(st + b_off0);
    const uint4 pa1 = lds128(st + a_off1), pb1 = lds128(st + b_off1);
    // scales and zeros of both groups (adjacent fp16 in one 32-bit word)
    uint32_t sa2, sb2, za2, zb2;
    if constexpr (kScTma) {
      const uint32_t off = (uint32_t)((g_first_i + gl0) & 7) * 2;
      asm volatile("ld.shared.u32 %0, [%1];" : "=r"(sa2) : "r"(st + sa_off + off));
      asm volatile("ld.shared.u32 %0, [%1];" : "=r"(sb2) : "r"(st + sb_off + off));
      asm volatile("ld.shared.u32 %0, [%1];" : "=r"(za2) : "r"(st + sa_off + kSBytes + off));
      asm volatile("ld.shared.u32 %0, [%1];" : "=r"(zb2) : "r"(st + sb_off + kSBytes + off));
    } else {
      const int64_t row0 = (int64_t)rt * kRows;
      const int64_t kg = g_first + gl0;
      const bool two = gl0 + 1 < ng;
      const bool one = gl0 < ng;
      const int64_t na = row0 + ra, nb = row0 + rb;
      const uint32_t a0 = (one && na < N) ? __ldg(p.scales + na * Kg + kg) : 0u;
      const uint32_t b0 = (one && nb < N) ? __ldg(p.scales + nb * Kg + kg) : 0u;
      const uint32_t c0 = (one && na < N) ? __ldg(p.zeros + na * Kg + kg) : 0u;
      const uint32_t d0 = (one && nb < N) ? __ldg(p.zeros + nb * Kg + kg) : 0u;
      const uint32_t a1 = (two && na < N) ? __ldg(p.scales + na * Kg + kg + 1) : 0u;
      const uint32_t b1 = (two && nb < N) ? __ldg(p.scales + nb * Kg + kg + 1) : 0u;
      const uint32_t c1 = (two && na < N) ? __ldg(p.zeros + na * Kg + kg + 1) : 0u;
      const uint32_t d1 = (two && nb < N) ? __ldg(p.zeros + nb * Kg + kg + 1) : 0u;
      sa2 = a0 | (a1 << 16);
      sb2 = b0 | (b1 << 16);
      za2 = c0 | (c1 << 16);
      zb2 = d0 | (d1 << 16);
    }
    const float2 sca = __half22float2(*reinterpret_cast<const __half2 *>(&sa2));
    const float2 scb = __half22float2(*reinterpret_cast<const __half2 *>(&sb2));
    // Per group and row, the fp16 constants 1024 + z (low nibbles) and 1024 + 16 z
    // (high nibbles) in both halves; z is an integer 0..15, so both are exact.
    uint32_t zlo_a[2], zhi_a[2], zlo_b[2], zhi_b[2];
    {
      const __half2 k1024 = __float2half2_rn(1024.0f), k16 = __float2half2_rn(16.0f);
      const __half2 za = *reinterpret_cast<const __half2 *>(&za2);  // (z of group gl0, gl0 + 1), row a
      const __half2 zb = *reinterpret_cast<const __half2 *>(&zb2);
      const __half2 la = __hadd2(za, k1024), ha = __hfma2(za, k16, k1024);
      const __half2 lb = __hadd2(zb, k1024), hb = __hfma2(zb, k16, k1024);
      const __half2 v[8] = {__low2half2(la), __high2half2(la), __low2half2(ha), __high2half2(ha),
                            __low2half2(lb), __high2half2(lb), __low2half2(hb), __high2half2(hb)};
      const uint32_t *u = reinterpret_cast<const uint32_t *>(v);
      zlo_a[0] = u[0]; zlo_a[1] = u[1]; zhi_a[0] = u[2]; zhi_a[1] = u[3];
      zlo_b[0] = u[4]; zlo_b[1] = u[5]; zhi_b[0] = u[6]; zhi_b[1] = u[7];
    }
    const uint32_t xg_off0 = (uint32_t)gl0 * gstride_x, xg_off1 = xg_off0 + gstride_x;

    if constexpr (T8 <= 2) {
      // Both groups at once, k-block by k-block: four independent accumulator chains
      // per token octet (group x even/odd k-block), A fragments built just in time.
      float d[T8][2][2][4];
      const uint32_t wa0[4] = {pa0.x, pa0.y, pa0.z, pa0.w}, wb0[4] = {pb0.x, pb0.y, pb0.z, pb0.w};
      const uint32_t wa1[4] = {pa1.x, pa1.y, pa1.z, pa1.w}, wb1[4] = {pb1.x, pb1.y, pb1.z, pb1.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint32_t A[2][2][4];  // [group][k-block parity][fragment reg]
        {
          const uint32_t a8 = wa0[i] >> 8, b8 = wb0[i] >> 8, a18 = wa1[i] >> 8, b18 = wb1[i] >> 8;
          A[0][0][0] = dq_pair(wa0[i], 0x000F000Fu, zlo_a[0]);
          A[0][0][2] = dq_pair(wa0[i], 0x00F000F0u, zhi_a[0]);
          A[0][0][1] = dq_pair(wb0[i], 0x000F000Fu, zlo_b[0]);
          A[0][0][3] = dq_pair(wb0[i], 0x00F000F0u, zhi_b[0]);
          A[0][1][0] = dq_pair(a8, 0x000F000Fu, zlo_a[0]);
          A[0][1][2] = dq_pair(a8, 0x00F000F0u, zhi_a[0]);
          A[0][1][1] = dq_pair(b8, 0x000F000Fu, zlo_b[0]);
          A[0][1][3] = dq_pair(b8, 0x00F000F0u, zhi_b[0]);
          A[1][0][0] = dq_pair(wa1[i], 0x000F000Fu, zlo_a[1]);
          A[1][0][2] = dq_pair(wa1[i], 0x00F000F0u, zhi_a[1]);
          A[1][0][1] = dq_pair(wb1[i], 0x000F000Fu, zlo_b[1]);
          A[1][0][3] = dq_pair(wb1[i], 0x00F000F0u, zhi_b[1]);
          A[1][1][0] = dq_pair(a18, 0x000F000Fu, zlo_a[1]);
          A[1][1][2] = dq_pair(a18, 0x00F000F0u, zhi_a[1]);
          A[1][1][1] = dq_pair(b18, 0x000F000Fu, zlo_b[1]);
          A[1][1][3] = dq_pair(b18, 0x00F000F0u, zhi_b[1]);
        }
#pragma unroll
        for (int o = 0; o < T8; ++o)
#pragma unroll
          for (int pp = 0; pp < kParts; ++pp) {
            // B words 4i..4i+3 of each group: (x, y) feed k-block 2i, (z, w) feed 2i+1
            const uint4 B0 = lds128(bofs[o] + xg_off0 + (uint32_t)(pp * 256 + 16 * i));
            const uint4 B1 = lds128(bofs[o] + xg_off1 + (uint32_t)(pp * 256 + 16 * i));
            const bool first = i == 0 && pp == 0;
            mma_f16(d[o][0][0], A[0][0], B0.x, B0.y, first);
            mma_f16(d[o][1][0], A[1][0], B1.x, B1.y, first);
            mma_f16(d[o][0][1], A[0][1], B0.z, B0.w, first);
            mma_f16(d[o][1][1], A[1][1], B1.z, B1.w, first);
          }
      }
      // promotion: y' += scale * D per group, tokens 2t, 2t+1 of each octet
#pragma unroll
      for (int o = 0; o < T8; ++o)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const float sa = j ? sca.y : sca.x, sb = j ? scb.y : scb.x;
          acc[o][0] = fmaf(sa, d[o][j][0][0] + d[o][j][1][0], acc[o][0]);
          acc[o][1] = fmaf(sa, d[o][j][0][1] + d[o][j][1][1], acc[o][1]);
          acc[o][2] = fmaf(sb, d[o][j][0][2] + d[o][j][1][2], acc[o][2]);
          acc[o][3] = fmaf(sb, d[o][j][0][3] + d[o][j][1][3], acc[o][3]);
        }
    } else {
      // Many token octets: one group at a time, its A fragments reused across octets.
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const uint4 pa = j ? pa1 : pa0, pb = j ? pb1 : pb0;
        // A fragments: one SHF + four LOP3 + four HSUB2 per 32-bit word (8 codes)
        uint32_t A[8][4];
        const uint32_t wa[4] = {pa.x, pa.y, pa.z, pa.w};
        const uint32_t wb[4] = {pb.x, pb.y, pb.z, pb.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t wa8 = wa[i] >> 8, wb8 = wb[i] >> 8;
          A[2 * i][0] = dq_pair(wa[i], 0x000F000Fu, zlo_a[j]);
          A[2 * i][2] = dq_pair(wa[i], 0x00F000F0u, zhi_a[j]);
          A[2 * i][1] = dq_pair(wb[i], 0x000F000Fu, zlo_b[j]);
          A[2 * i][3] = dq_pair(wb[i], 0x00F000F0u, zhi_b[j]);
          A[2 * i + 1][0] = dq_pair(wa8, 0x000F000Fu, zlo_a[j]);
          A[2 * i + 1][2] = dq_pair(wa8, 0x00F000F0u, zhi_a[j]);
          A[2 * i + 1][1] = dq_pair(wb8, 0x000F000Fu, zlo_b[j]);
          A[2 * i + 1][3] = dq_pair(wb8, 0x00F000F0u, zhi_b[j]);
        }
        const float sa = j ? sca.y : sca.x, sb = j ? scb.y : scb.x;
        const uint32_t xg_off = j ? xg_off1 : xg_off0;
#pragma unroll
        for (int o = 0; o < T8; ++o) {
          if (o * 8 >= Mi) break;  // octet without real tokens (warp-uniform)
          float d0[4], d1[4];
#pragma unroll
          for (int pp = 0; pp < kParts; ++pp) {
            uint32_t Bv[16];
            const uint32_t bad = bofs[o] + xg_off + (uint32_t)(pp * 256);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint4 v = lds128(bad + 16 * q);
              Bv[4 * q] = v.x; Bv[4 * q + 1] = v.y; Bv[4 * q + 2] = v.z; Bv[4 * q + 3] = v.w;
            }
#pragma unroll
            for (int b = 0; b < 8; ++b) {
              if (b & 1) mma_f16(d1, A[b], Bv[2 * b], Bv[2 * b + 1], pp == 0 && b == 1);
              else mma_f16(d0, A[b], Bv[2 * b], Bv[2 * b + 1], pp == 0 && b == 0);
            }
          }
          acc[o][0] = fmaf(sa, d0[0] + d1[0], acc[o][0]);
          acc[o][1] = fmaf(sa, d0[1] + d1[1], acc[o][1]);
          acc[o][2] = fmaf(sb, d0[2] + d1[2], acc[o][2]);
          acc[o][3] = fmaf(sb, d0[3] + d1[3], acc[o][3]);
        }
      }
    }
    // release the stage (all lanes' shared-memory reads are consumed above)
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    if (++s == kNst) {
      s = 0;
      ph ^= 1u;
    }
    if (!last) continue;

    // ---------------- fragment done: the two warps of a row block combine their groups
    // through shared memory, handing off with (bounded) mbarrier waits
    {
      const uint32_t pph = (uint32_t)(frags_done & 1);
      if (half == 1) {
        if (!mbar_wait(&pair_empty[blk4], pph ^ 1u, kErrTimeoutDequant)) break;
#pragma unroll
        for (int o = 0; o < T8; ++o)
          *reinterpret_cast<float4 *>(pairbuf + ((blk4 * 32 + lane) * T8 + o) * 4) =
              make_float4(acc[o][0], acc[o][1], acc[o][2], acc[o][3]);
        __syncwarp();
        if (lane == 0) mbar_arrive(&pair_full[blk4]);
      } else {
        if (!mbar_wait(&pair_full[blk4], pph, kErrTimeoutDequant)) break;
#pragma unroll
        for (int o = 0; o < T8; ++o) {
          const float4 v = *reinterpret_cast<const float4 *>(pairbuf + ((blk4 * 32 + lane) * T8 + o) * 4);
          acc[o][0] += v.x; acc[o][1] += v.y; acc[o][2] += v.z; acc[o][3] += v.w;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&pair_empty[blk4]);
      }
      ++frags_done;
    }
    // outputs of this row block (scaled back by 2^-e), written by the half-0 warp
    const int64_t row0 = (int64_t)rt * kRows;
    const int64_t blk = row0 / 16 + blk4;
    if (half == 0) finish_pending();
    if (half == 0 && blk < RB16) {
      const bool direct = (sw >> 16) != 0;
      const int slot = sw & 0xFFFF;
      const int64_t rowa = row0 + ra, rowb = row0 + rb;
      float *part = p.ws + ((int64_t)kslice * p.slots + slot) * M * N;
#pragma unroll
      for (int o = 0; o < T8; ++o)
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const int64_t row = (cc < 2) ? rowa : rowb;
          const int tok = o * 8 + 2 * t + (cc & 1);
          if (row < N && tok < Mi) {
            const float v = acc[o][cc] * exp2i(-xexp[tok]);
            if (direct) {
              if (p.y_bf16) static_cast<__nv_bfloat16 *>(p.Y)[(int64_t)tok * N + row] = __float2bfloat16_rn(v);
              else static_cast<float *>(p.Y)[(int64_t)tok * N + row] = v;
            } else {
              part[(int64_t)tok * N + row] = v;
            }
          }
        }
      if (!direct) {
        // announce the partials: warp barrier, then one release atomic (read one fragment later)
        __syncwarp();
        if (lane == 0) atom_release_add(&p.counters[blk], 1u, pend_ticket);
        pend_row0 = row0;
        pend_total = ntotal;
      }
    }
#pragma unroll
    for (int o = 0; o < T8; ++o) acc[o][0] = acc[o][1] = acc[o][2] = acc[o][3] = 0.0f;
  }
  if (half == 0) finish_pending();
}

// Programmatic dependent launch is on by default; W4_PDL=0 launches without it
// (for tools that replay kernels one at a time).
inline bool pdl_enabled() {
  static const bool on = [] {
    const char *e = getenv("W4_PDL");
    return !(e && e[0] == '0');
  }();
  return on;
}

template <int T8, bool kBf16, bool kAwq, bool kScTma>
cudaError_t launch_t(const CUtensorMap &tmP, const CUtensorMap &tmS, const CUtensorMap &tmZ, const GemvParams &p,
                     cudaStream_t stream) {
  auto kern = gemv_kernel<T8, kBf16, kAwq, kScTma>;
  const int smem = smem_bytes_for(p.xs_bytes, T8);
  static std::atomic<int> smem_set[kAttrDevices];  // largest size already set, per device
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void *>(kern), smem, smem_set);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)p.grid_x, (unsigned)p.kslices);
  cfg.blockDim = dim3(kComputeThreads + 32);
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, tmP, tmS, tmZ, p);
}

template <int T8, bool kBf16>
cudaError_t launch_x(const CUtensorMap &tmP, const CUtensorMap &tmS, const CUtensorMap &tmZ, const GemvParams &p,
                     bool sc_tma, cudaStream_t stream) {
  if (p.awq_s)
    return sc_tma ? launch_t<T8, kBf16, true, true>(tmP, tmS, tmZ, p, stream)
                  : launch_t<T8, kBf16, true, false>(tmP, tmS, tmZ, p, stream);
  return sc_tma ? launch_t<T8, kBf16, false, true>(tmP, tmS, tmZ, p, stream)
                : launch_t<T8, kBf16, false, false>(tmP, tmS, tmZ, p, stream);
}

template <int T8>
cudaError_t launch_s(const CUtensorMap &tmP, const CUtensorMap &tmS, const CUtensorMap &tmZ, const GemvParams &p,
                     bool x_bf16, bool sc_tma, cudaStream_t stream) {
  return x_bf16 ? launch_x<T8, true>(tmP, tmS, tmZ, p, sc_tma, stream)
                : launch_x<T8, false>(tmP, tmS, tmZ, p, sc_tma, stream);
}

}  // namespace gemv_impl

bool gemv_supports(int64_t M, bool) { return M <= 64; }

// Shared-memory bytes of the staged activations for a k-slice of kr groups.
int gemv_xs_bytes(int kr, int64_t M, bool awq) { return gemv_impl::xs_bytes_for(kr, (int)M, awq); }
int gemv_smem_bytes(int xs_bytes, int t8) { return gemv_impl::smem_bytes_for(xs_bytes, t8); }

cudaError_t launch_gemv(const CUtensorMap &tmP, const CUtensorMap &tmS, const CUtensorMap &tmZ, const GemvParams &p,
                        int t8, bool x_bf16, bool sc_tma, cudaStream_t stream) {
  using namespace gemv_impl;
  switch (t8) {
    case 1: return launch_s<1>(tmP, tmS, tmZ, p, x_bf16, sc_tma, stream);
    case 2: return launch_s<2>(tmP, tmS, tmZ, p, x_bf16, sc_tma, stream);
    case 4: return launch_s<4>(tmP, tmS, tmZ, p, x_bf16, sc_tma, stream);
    default: return launch_s<8>(tmP, tmS, tmZ, p, x_bf16, sc_tma, stream);
  }
}

}  // namespace w4
