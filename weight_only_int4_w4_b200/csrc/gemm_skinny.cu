// gemm_skinny.cu -- K3: W4A16 matmul for small token counts (8 < M <= 64) on the
// 5th-generation tensor cores, with exact integer weights and per-group promotion.
//
// Speculative verification and small-batch decode multiply every weight by a
// handful of tokens: the call still reads each weight once, so it should stay
// bound by the weight bytes ("LLM inference acceleration" article, section
// 1.1; ch. 22 "Advanced inference optimisation", section 22.1: verifying K
// draft tokens costs about one decode step, and section 22.2: decode is
// memory-bound).  That needs dequantization at well under two instructions per
// weight and the tensor cores for the M-fold product.  The weight-only path of
// ch. 22 section 22.3 (dequantize back to 16 bits, then matmul) is computed as
//
//   y[m][n] = 2^-e[m] * sum_g scale[n][g] * sum_{k in g} (q[n][k] - z[n][g]) * x'[m][k]
//
// with (q - z) an exact small integer and x' = x * s[k] * 2^e[m] in fp16:
//
//   * stage_x_kernel (one CTA per token) writes x' into the workspace: a power of
//     two e per token puts max |x'| in [2^13, 2^14), so bf16 and fp16 inputs
//     convert exactly (values more than 2^27 below the maximum excepted); with
//     AWQ, x * s is rounded to fp16 once (at most 2^-11 relative per product).
//     Within every 8 channels the values are stored in the order the weight
//     dequantization produces them: k = 0, 4, 1, 5, 2, 6, 3, 7, with the odd
//     channels divided by 16.
//   * skinny_kernel: one CTA per SM walks a balanced, contiguous range of
//     (128-row tile, 256-channel stage) iterations in tile-major order.
//       warp 0      TMA producer: the stage's packed codes [128 rows x 128 B,
//                   128-byte swizzle] and x' [4 boxes of BN tokens x 64 channels].
//       warp 1      TMEM owner and MMA issuer: per group, eight
//                   tcgen05.mma.kind::f16 (A = codes from TMEM, B = x' from shared
//                   memory) into one of two per-group fp32 accumulators.
//       warps 4..7  thread r owns weight row r: per group it turns 64 bytes of
//                   codes into the exact fp16 pairs (q - z) / 16 (q - z) with one
//                   LOP3 against the fp16 magic 0x6400 and one HSUB2 of 1024 + z
//                   (or 1024 + 16 z) per pair -- nine instructions per eight
//                   weights -- and stores them into TMEM with tcgen05.st; then it
//                   promotes the previous group, y[t] += scale * D[t] from
//                   tcgen05.ld, and at the end of a tile writes y * 2^-e.
//     A tile split between CTAs is finished by its last contributor: every piece
//     stores its fp32 partials and takes a ticket from the tile's counter, and
//     the last one sums all pieces in a fixed order (tickets are read at the end
//     of the CTA's range, so no warp waits on another CTA).
// All waits are bounded (common.cuh).  No TMA multicast.
#include "common.cuh"

namespace w4 {

struct SkinnyParams {
  int64_t M, N, K;
  const uint16_t *scales;
  const uint16_t *zeros;
  void *Y;
  int y_bf16;
  const int *xexp;     // [M] per-token exponents e (written by stage_x_kernel)
  float *ws;           // [slots][M][N] fp32 partials of split tiles
  uint32_t *counters;  // [row tiles] arrival counters
  int slots;           // partial slots per tile
};

namespace sk_impl {

constexpr int kRows = 128;             // weight rows per tile = TMEM lanes
constexpr int kWStage = kRows * 128;   // 16 KiB of codes per stage (2 groups)


// ------------------------------------------------------------------ staging of x'
// One CTA of 512 threads per token of the BN-token tile: max |x * s| over K,
// then x' in the permuted order (see the file head).  Channels
// k = 8j + c (c = 0..7).  Layout: x'[k / 64][token][k % 64] (64-channel blocks,
// BN tokens each), so one stage's 4 blocks x BN tokens are consecutive rows of
// 128 bytes and arrive in one TMA box.  Tokens M..BN-1 are zeros.
constexpr int kStageThreads = 512;  // threads per token
constexpr int kStageChunks = 8;     // 8-channel chunks a thread holds in the one-pass form

template <bool kBf16, bool kAwq>
__global__ void __launch_bounds__(kStageThreads) stage_x_kernel(const uint16_t *__restrict__ X,
                                                                const float *__restrict__ s, int64_t M, int64_t K,
                                                                int bn, uint16_t *__restrict__ Xp,
                                                                int *__restrict__ xexp) {
  __shared__ float red[kStageThreads / 32];
  // The activations may be written by the preceding kernel, and x' may still be
  // read by the preceding matmul: wait for it, then let the matmul launch.
  grid_dependency_wait();
  if (threadIdx.x == 0) grid_launch_dependents();
  const int64_t m = blockIdx.x;
  const int64_t nb = K / 8;
  // chunk j (channels 8j .. 8j + 7) of this token in the blocked layout
  auto out_at = [&](int64_t j) { return Xp + ((j >> 3) * bn + m) * 64 + (j & 7) * 8; };
  if (m >= M) {  // padding token of the tile
    if (threadIdx.x == 0) xexp[m] = 0;
    for (int64_t j = threadIdx.x; j < nb; j += blockDim.x) *reinterpret_cast<uint4 *>(out_at(j)) = make_uint4(0, 0, 0, 0);
    return;
  }
  const uint16_t *xr = X + m * K;
  auto load_raw = [&](int64_t j) { return __ldg(reinterpret_cast<const uint4 *>(xr + 8 * j)); };
  // x (times s with AWQ) of chunk j from its raw 16 bytes
  auto decode = [&](int64_t j, const uint4 &u, float (&v)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if constexpr (kBf16) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
      } else {
        const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w[i]));
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
      }
    }
    if constexpr (kAwq) {
      const float4 s0 = __ldg(reinterpret_cast<const float4 *>(s + 8 * j));
      const float4 s1 = __ldg(reinterpret_cast<const float4 *>(s + 8 * j + 4));
      v[0] *= s0.x; v[1] *= s0.y; v[2] *= s0.z; v[3] *= s0.w;
      v[4] *= s1.x; v[5] *= s1.y; v[6] *= s1.z; v[7] *= s1.w;
    }
  };
  // One pass when the token fits the registers (every shape up to K = 32768): all
  // of a thread's loads are in flight at once and X is read once.  Otherwise two
  // passes (max, then convert), each reading X.
  const bool one_pass = nb <= (int64_t)kStageChunks * blockDim.x;
  uint4 raw[kStageChunks];
  float mx = 0.0f;
  if (one_pass) {
#pragma unroll
    for (int c = 0; c < kStageChunks; ++c) {
      const int64_t j = threadIdx.x + (int64_t)c * blockDim.x;
      raw[c] = j < nb ? load_raw(j) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int c = 0; c < kStageChunks; ++c) {
      const int64_t j = threadIdx.x + (int64_t)c * blockDim.x;
      if (j < nb) {
        float v[8];
        decode(j, raw[c], v);
#pragma unroll
        for (int i = 0; i < 8; ++i) mx = fmaxf(mx, fabsf(v[i]));
      }
    }
  } else {
    for (int64_t j = threadIdx.x; j < nb; j += blockDim.x) {
      float v[8];
      decode(j, load_raw(j), v);
#pragma unroll
      for (int i = 0; i < 8; ++i) mx = fmaxf(mx, fabsf(v[i]));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
  __syncthreads();
  mx = red[0];
  for (int i = 1; i < (int)(blockDim.x >> 5); ++i) mx = fmaxf(mx, red[i]);
  // max |x'| in [2^13, 2^14): e = 13 - floor(log2 max); 0 for an all-zero token
  const int bits = __float_as_int(mx);
  int e = bits == 0 ? 0 : 13 - (((bits >> 23) & 0xFF) - 127);
  e = max(-100, min(100, e));
  if (threadIdx.x == 0) xexp[m] = e;
  const float se = __uint_as_float((uint32_t)(e + 127) << 23);      // 2^e
  const float so = __uint_as_float((uint32_t)(e - 4 + 127) << 23);  // 2^(e-4): odd channels / 16
  auto convert_store = [&](int64_t j, const uint4 &u) {
    float v[8];
    decode(j, u, v);
    // slots 0..7 hold channels 0, 4, 1, 5, 2, 6, 3, 7; odd channels carry 1/16
    const __half2 h0 = __floats2half2_rn(v[0] * se, v[4] * se);
    const __half2 h1 = __floats2half2_rn(v[1] * so, v[5] * so);
    const __half2 h2 = __floats2half2_rn(v[2] * se, v[6] * se);
    const __half2 h3 = __floats2half2_rn(v[3] * so, v[7] * so);
    uint4 o;
    o.x = *reinterpret_cast<const uint32_t *>(&h0);
    o.y = *reinterpret_cast<const uint32_t *>(&h1);
    o.z = *reinterpret_cast<const uint32_t *>(&h2);
    o.w = *reinterpret_cast<const uint32_t *>(&h3);
    *reinterpret_cast<uint4 *>(out_at(j)) = o;
  };
  if (one_pass) {
#pragma unroll
    for (int c = 0; c < kStageChunks; ++c) {
      const int64_t j = threadIdx.x + (int64_t)c * blockDim.x;
      if (j < nb) convert_store(j, raw[c]);
    }
  } else {
    for (int64_t j = threadIdx.x; j < nb; j += blockDim.x) convert_store(j, load_raw(j));
  }
}

// ------------------------------------------------------------------ helpers
__device__ __forceinline__ uint32_t hsub2_u32(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("sub.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// 4-byte asynchronous copy global -> shared (both 4-byte aligned); completion is
// tracked per thread with commit / wait groups.
__device__ __forceinline__ void cp_async4(uint32_t saddr, const void *gaddr) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(saddr), "l"(gaddr) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int kPending>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(kPending) : "memory"); }

// Exact fp16 pair: (w & mask) | 1024.0 minus zc (1024 + z, or 1024 + 16 z for the high nibbles).
__device__ __forceinline__ uint32_t dq2(uint32_t w, uint32_t mask, uint32_t zc) {
  return hsub2_u32(lop3_and_or(w, mask, 0x64006400u), zc);
}

// ------------------------------------------------------------------ main kernel
// Warp roles (512 threads for BN <= 32, 640 above):
//   warps 0..3    TMA producers: warp k issues the stages i = k (mod 4), lane 0
//                 the codes box, lane 1 the x' box.  The boxes one thread issues
//                 are in flight roughly one after another, so stages issued by
//                 different warps are what overlaps.
//   warps 4..7    MMA issuers: issuer j = w - 4 owns TMEM A buffer j and
//                 accumulator j, i.e. every 4th group (warp 4 also owns TMEM).
//                 A tcgen05.mma costs its issuing thread about 0.1 us on B200
//                 whatever N is, so one issuer caps a 128-row x 16-channel MMA
//                 stream far below the HBM rate; four issuers overlap.
//   warps 8..11   dequantization: warp w serves TMEM lane quadrant w % 4, one
//                 weight row per thread, all 128 channels of every group
//   warps 12..    promotion and epilogue, one warp per quadrant (two for BN > 32):
//                 warp w serves quadrant w % 4, one weight row and tokens
//                 hp kTB .. hp kTB + kTB - 1 per thread, hp = (w - 12) / 4
// TMEM holds kNA A buffers (64 columns, one group, each) then kNR accumulators of
// BN columns; kNA is as many as fit (7 at BN = 16 down to 4 at BN = 64).  A buffer
// goes round dequantization, hand-off, eight MMA issues and their completion
// (about 1.2 us), so the buffer count sets how many groups are in flight.  Groups
// take buffers g mod kNA; dequantization fills them in group order and each issuer
// takes its groups in order, so no waiter runs two barrier phases ahead.
// The two sets run decoupled: dequantization runs up to kNA groups ahead of the
// tensor core, promotion up to kNR groups behind it, and each set pays its TMEM
// store (or load) wait once per two groups.
constexpr int kIssuers = 4;                   // MMA issuer warps (see the role list)
// Scales and zeros are copied kPf stages ahead of use into a per-thread ring in
// shared memory (cp.async): under a full HBM stream a global load takes about a
// microsecond, several stages.  (A register queue does not work: rotating it
// copies the register of the most recent load and waits for that load.)
constexpr int kPf = 8;
constexpr int kProdWarps = 4;                 // warps 0..3
constexpr int kMma0 = kProdWarps;             // first MMA warp (TMEM owner)
constexpr int kMmaWarps = 4;                  // warps 4..7
constexpr int kDq0 = 32 * (kProdWarps + kMmaWarps);  // first dequantization thread (warp 8)
constexpr int kDqThreads = 128;               // warps 8..11
constexpr int kPr0 = kDq0 + kDqThreads;       // first promotion thread (warp 12)

// Ticket of a split tile: acquire-release at GPU scope.  After a CTA barrier, one
// thread's release publishes the whole CTA's partial stores (no full fence); the
// last ticket's acquire, followed by a CTA barrier, orders the loads of the
// threads that sum every piece after all contributors' stores.
__device__ __forceinline__ uint32_t atom_add_acq_rel_gpu(uint32_t *addr, uint32_t v) {
  uint32_t old;
  asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], %2;" : "=r"(old) : "l"(addr), "r"(v) : "memory");
  return old;
}
__device__ __forceinline__ uint32_t ld_shared_u32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
  return v;
}

// Walks the stages of a CTA's range in order and copies, for weight row rr of
// each stage's tile, the adjacent fp16 pair of the stage's two groups (scales or
// zero points) into ring slot (stage mod kPf) at `slot0 + slot * slot_stride`
// bytes.  One cp.async group is committed per stage, so cp.async.wait_group
// kPf - 1 makes the oldest stage's copy visible.  Rows past N, stages past the
// range and a group past Kg give 0; a pair that is not 4-byte aligned (Kg odd)
// is read with plain loads.
struct PairFetcher {
  const uint16_t *base;
  int N, Kg, S, n_it, i, rr;  // N < 2^31 and Kg < 2^31 (the planner's limits)
  int rt, st;                 // tile and stage of fetch i
  uint32_t slot0, stride;
  __device__ PairFetcher(const uint16_t *b, int64_t it0, int n, int64_t S_, int64_t N_, int64_t Kg_, int r,
                         uint32_t s0, uint32_t str)
      : base(b), N((int)N_), Kg((int)Kg_), S((int)S_), n_it(n), i(0), rr(r), slot0(s0), stride(str) {
    rt = (int)(it0 / S_);
    st = (int)(it0 - (int64_t)rt * S_);
  }
  __device__ __forceinline__ void next() {
    const uint32_t dst = slot0 + (uint32_t)(i % kPf) * stride;
    if (i < n_it) {
      const int n = rt * kRows + rr, kg = 2 * st;
      const int64_t off = (int64_t)n * Kg + kg;
      if (n < N && kg + 1 < Kg && (off & 1) == 0) {
        cp_async4(dst, base + off);
      } else {
        uint32_t v = 0u;
        if (n < N) v = (uint32_t)__ldg(base + off) | (kg + 1 < Kg ? (uint32_t)__ldg(base + off + 1) << 16 : 0u);
        asm volatile("st.shared.u32 [%0], %1;" ::"r"(dst), "r"(v) : "memory");
      }
      if (++st == S) {
        st = 0;
        ++rt;
      }
    }
    cp_async_commit();  // one group per stage, empty past the range
    ++i;
  }
};

template <int BN>
struct Cfg {
  static constexpr int kXStage = 4 * BN * 128;  // 4 blocks [BN tokens x 64 channels] fp16, one box
  static constexpr int kStage = kWStage + kXStage;
  // ring depth: a multiple of the producer warps (each owns the stages i = k mod 4)
  static constexpr int kNS = (229376 / kStage) >= 8 ? 8 : 4;
  static constexpr int kPW = BN > 32 ? 2 : 1;  // promotion warps per lane quadrant
  static constexpr int kTB = BN / kPW;         // tokens promoted by each promotion thread
  static constexpr int kPrThreads = 128 * kPW;
  // rings of zero-point pairs [kPf][dequantization threads] and scale pairs [kPf][promotion threads]
  static constexpr int kRingBytes = kPf * kDqThreads * 4 + kPf * kPrThreads * 4;
  // Per-group accumulators: two per issuer where TMEM has room (BN <= 32), so an
  // issuer's next group never waits for the promotion of its previous one -- that
  // round trip (commit, promotion, arrival, wake-up) is longer than the MMAs.
  static constexpr int kNR = BN <= 32 ? 2 * kIssuers : kIssuers;
  static constexpr int kNA = (512 - kNR * BN) / 64;  // TMEM A buffers
  static constexpr int kAccCol = 64 * kNA;          // first accumulator column
  static constexpr int kSmem =
      1024 + kNS * kStage + (3 * kNS + 2 * kNA + 2 * kNR) * 8 + 16 + 64 * 4 + kRingBytes + 16 + 64;
  static constexpr int kThreads = kPr0 + kPrThreads;
  static_assert(kAccCol + kNR * BN <= 512, "TMEM columns");
  static_assert(kSmem <= 232448, "shared memory");
};

__device__ __forceinline__ void tmem_ld_32x32b_x8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr)
               : "memory");
}

__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
      "%14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

template <int kCount>
__device__ __forceinline__ void named_bar_pr() { asm volatile("bar.sync 1, %0;" ::"n"(kCount) : "memory"); }

// Balanced partition of T iterations over C CTAs: CTA c takes [floor(cT/C), floor((c+1)T/C)).
__device__ __forceinline__ int64_t sk_begin(int64_t c, int64_t T, int64_t C) { return (c * T) / C; }
__device__ __forceinline__ int64_t sk_owner(int64_t i, int64_t T, int64_t C) { return ((i + 1) * C - 1) / T; }

template <int BN>
__global__ void __launch_bounds__(Cfg<BN>::kThreads, 1)
    skinny_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                  const SkinnyParams p) {
  using C_ = Cfg<BN>;
  constexpr int kNR = C_::kNR;
  constexpr int kNA = C_::kNA;
  constexpr int kAccCol = C_::kAccCol;
  constexpr int kNS = C_::kNS;
  constexpr int kTB = C_::kTB;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sW = smem;
  uint8_t *sX = smem + kNS * kWStage;
  // A stage's codes and its x' complete separate barriers: the dequantization needs
  // only the codes, so it runs ahead while x' (which waits for the staging kernel)
  // is still on its way; the MMA issuers wait for x'.
  uint64_t *full = reinterpret_cast<uint64_t *>(sX + kNS * C_::kXStage);  // codes
  uint64_t *xfull = full + kNS;                                            // x'
  uint64_t *empty = xfull + kNS;
  uint64_t *afull = empty + kNS;
  uint64_t *aempty = afull + kNA;
  uint64_t *accfull = aempty + kNA;    // [kNR]
  uint64_t *accempty = accfull + kNR;  // [kNR]
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(accempty + kNR);
  int *s_ticket = reinterpret_cast<int *>(tmem_holder + 1);       // [2]
  float *s_escale = reinterpret_cast<float *>(tmem_holder + 4);  // [64] 2^-e per token
  uint32_t *zring = reinterpret_cast<uint32_t *>(s_escale + 64);  // [kPf][kDqThreads]
  uint32_t *sring = zring + kPf * kDqThreads;                     // [kPf][kPrThreads]
  int *s_pend = reinterpret_cast<int *>(sring + kPf * C_::kPrThreads);  // split tiles: rt0, count0, rt1, count1
  int *s_npend = reinterpret_cast<int *>(tmem_holder + 3);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t M = p.M, N = p.N, K = p.K;
  const int64_t Kg = K / kGroup;
  const int64_t S = (Kg + 1) / 2;  // stages (2 groups each) per tile
  const int64_t RT = (N + kRows - 1) / kRows;
  const int64_t T = RT * S;
  const int64_t CT = gridDim.x;
  const int64_t it0 = sk_begin(blockIdx.x, T, CT), it1 = sk_begin((int64_t)blockIdx.x + 1, T, CT);
  const int n_it = (int)(it1 - it0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kNS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&xfull[s], 1);
      mbar_init(&empty[s], 2);  // one commit per group, from that group's issuer
    }
    for (int a = 0; a < kNA; ++a) {
      mbar_init(&afull[a], kDqThreads);
      mbar_init(&aempty[a], 1);
    }
    for (int r = 0; r < kNR; ++r) {
      mbar_init(&accfull[r], 1);
      mbar_init(&accempty[r], C_::kPrThreads);
    }
    fence_barrier_init();
  }
  if (warp == kMma0) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp < kProdWarps && lane < 2) {
    // ---------------- TMA producer k = w: the stages i = k (mod 4) of the range;
    // lane 0 the codes (one box of 128 rows x 128 bytes), lane 1 the x' of the
    // stage (one box of 4 BN rows).  On B200 the TMA unit works through small
    // boxes one after another at a fixed cost each, so a stage is two boxes.
    // Scales and zeros are not staged: the warps that use them copy 4-byte pairs
    // ahead of use.
    const int k = warp;
    if (lane == 0 && k == 0) {
      prefetch_tensormap(&tmW);
      prefetch_tensormap(&tmX);
    }
    const bool x_lane = lane == 1;
    // (tile, stage) of the lane's last stage: each lane asks for its stages in
    // increasing order, so they advance without a division per stage
    int last_i = -1;
    int64_t rt = 0, st = 0;
    auto load_lane = [&](int i) {
      if (last_i < 0) {
        rt = (it0 + i) / S;
        st = it0 + i - rt * S;
      } else {
        st += i - last_i;
        while (st >= S) {
          st -= S;
          ++rt;
        }
      }
      last_i = i;
      const int s = i % kNS;
      if (!x_lane) {
        tma_load_2d(sW + s * kWStage, &tmW, &full[s], (int32_t)(st * 128), (int32_t)(rt * kRows));
      } else {
        tma_load_2d(sX + s * C_::kXStage, &tmX, &xfull[s], 0, (int32_t)(st * 4 * BN));
      }
    };
    // Weights never come from a preceding kernel: the first ring's codes are
    // requested before waiting for the staged activations.
    const int pre = n_it < kNS ? n_it : kNS;
    for (int i = k; i < pre; i += kProdWarps) {
      if (!x_lane) {
        mbar_arrive_expect_tx(&full[i % kNS], kWStage);
        load_lane(i);
      }
    }
    grid_dependency_wait();
    for (int i = k; i < pre; i += kProdWarps) {
      if (x_lane) {
        mbar_arrive_expect_tx(&xfull[i % kNS], C_::kXStage);
        load_lane(i);
      }
    }
    for (int i = pre + ((k - pre % kProdWarps + kProdWarps) % kProdWarps); i < n_it; i += kProdWarps) {
      const int s = i % kNS;
      // both lanes wait for the free slot; the vote keeps them on one path if a
      // wait ever gives up
      const bool w_ok = mbar_wait(&empty[s], ((uint32_t)(i / kNS) & 1u) ^ 1u, kErrTimeoutTma);
      if (!__all_sync(0x3u, w_ok)) break;
      mbar_arrive_expect_tx(x_lane ? &xfull[s] : &full[s], x_lane ? C_::kXStage : kWStage);
      load_lane(i);
    }
    // every load of this CTA is issued: the next kernel in the stream may launch
    if (!x_lane) grid_launch_dependents();
  } else if (warp >= kMma0 && warp < kMma0 + kMmaWarps && lane == 0) {
    // ---------------- MMA issuer j = w - 4: the groups g = j (mod 4) of the range
    // (CTA-local group index g = 2 * stage + gi), from A buffer g mod kNA into
    // accumulator g mod kNR (always one of this issuer's, as kNR is a multiple of 4).
    const int j = warp - kMma0;
    const uint32_t idesc = idesc_f16(false, BN);
    for (int g = j; g < 2 * n_it; g += kIssuers) {
      const int i = g >> 1, gi = g & 1;
      const int s = i % kNS;
      const int a = g % kNA;
      const int r = g % kNR;
      const uint32_t a_tmem = tmem + (uint32_t)(64 * a);
      const uint32_t d_tmem = tmem + (uint32_t)(kAccCol + BN * r);
      if (!mbar_wait(&xfull[s], (uint32_t)(i / kNS) & 1u, kErrTimeoutMma)) break;
      if (!mbar_wait(&afull[a], (uint32_t)(g / kNA) & 1u, kErrTimeoutMma)) break;
      if (!mbar_wait(&accempty[r], ((uint32_t)(g / kNR) & 1u) ^ 1u, kErrTimeoutMma)) break;
      tc_fence_after();
      const uint32_t xs = smem_u32(sX + s * C_::kXStage);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const int b = 2 * gi + (kk >> 2);
        const uint64_t bdesc = smem_desc_k_sw128(xs + (uint32_t)(b * BN * 128)) + (uint64_t)(2 * (kk & 3));
        tc_mma_ts(d_tmem, a_tmem + 8 * kk, bdesc, idesc, kk > 0 ? 1u : 0u);
      }
      tc_commit(&aempty[a]);
      tc_commit(&accfull[r]);
      tc_commit(&empty[s]);
    }
  } else if (warp >= kDq0 / 32 && warp < kPr0 / 32) {
    // ---------------- dequantization: all 128 channels of every group for one weight row
    const int q = warp & 3;
    const int rr = q * 32 + lane;
    const int dt = threadIdx.x - kDq0;
    const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
    // the zero points of both groups of a stage (adjacent fp16) go to this
    // thread's ring slot (stage mod kPf), kPf stages ahead of use
    PairFetcher zf(p.zeros, it0, n_it, S, N, Kg, rr, smem_u32(zring) + 4u * (uint32_t)dt, kDqThreads * 4);
    for (int d = 0; d < kPf; ++d) zf.next();
    int g = 0;
    for (int i = 0; i < n_it; ++i) {
      cp_async_wait<kPf - 1>();  // this thread's copies for stage i have landed
      const uint32_t zpair = ld_shared_u32(smem_u32(zring) + 4u * (uint32_t)((i % kPf) * kDqThreads + dt));
      const int s = i % kNS;
      // A wait that gives up raises the device error word (later waits then give up
      // quickly); the loop runs to the end all the same.
      mbar_wait(&full[s], (uint32_t)(i / kNS) & 1u, kErrTimeoutDequant);
      const uint32_t wrow = smem_u32(sW + s * kWStage + rr * 128);
#pragma unroll
      for (int gi = 0; gi < 2; ++gi) {
        const uint32_t z_bits = gi ? (zpair >> 16) : (zpair & 0xFFFFu);
        const int a = (g + gi) % kNA;
        mbar_wait(&aempty[a], ((uint32_t)((g + gi) / kNA) & 1u) ^ 1u, kErrTimeoutDequant);
        // zero-point constants 1024 + z (low nibbles) and 1024 + 16 z (high), both halves
        const __half zh = __ushort_as_half((unsigned short)z_bits);
        const __half2 z2 = __halves2half2(zh, zh);
        const __half2 lo2 = __hadd2(z2, __float2half2_rn(1024.0f));
        const __half2 hi2 = __hfma2(z2, __float2half2_rn(16.0f), __float2half2_rn(1024.0f));
        const uint32_t zlo = *reinterpret_cast<const uint32_t *>(&lo2);
        const uint32_t zhi = *reinterpret_cast<const uint32_t *>(&hi2);
        if (gi == 1) zf.next();  // stage i's pair is consumed: its slot takes stage i + kPf
        // the group's 64 bytes of codes: logical chunks 4 gi .. 4 gi + 3 (128-byte
        // swizzle), 32 bytes (64 channels, 32 TMEM columns) per store
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const uint4 u0 = lds128(wrow + (uint32_t)(((4 * gi + 2 * hh) ^ (rr & 7)) << 4));
          const uint4 u1 = lds128(wrow + (uint32_t)(((4 * gi + 2 * hh + 1) ^ (rr & 7)) << 4));
          const uint32_t wv[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
          uint32_t out[32];
#pragma unroll
          for (int wi = 0; wi < 8; ++wi) {
            const uint32_t w = wv[wi], w8 = w >> 8;
            out[4 * wi + 0] = dq2(w, 0x000F000Fu, zlo);
            out[4 * wi + 1] = dq2(w, 0x00F000F0u, zhi);
            out[4 * wi + 2] = dq2(w8, 0x000F000Fu, zlo);
            out[4 * wi + 3] = dq2(w8, 0x00F000F0u, zhi);
          }
          tmem_st_32x32b_x32(lane_base + (uint32_t)(64 * a + 32 * hh), out);
        }
      }
      // one store wait for both groups of the stage
      tc_wait_st();
      tc_fence_before();
      mbar_arrive(&afull[g % kNA]);
      mbar_arrive(&afull[(g + 1) % kNA]);
      g += 2;
    }
  } else if (warp >= kPr0 / 32) {
    // ---------------- promotion and epilogue: kTB tokens of one weight row
    const int q = warp & 3;
    const int hp = (warp - kPr0 / 32) >> 2;
    const int rr = q * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
    const int tok0 = hp * kTB;
    grid_dependency_wait();  // exponents, Y and the workspace may belong to preceding kernels
    if (threadIdx.x - kPr0 < 64) {
      const int t = threadIdx.x - kPr0;
      s_escale[t] = t < M ? __uint_as_float((uint32_t)(127 - p.xexp[t]) << 23) : 0.0f;
    }
    named_bar_pr<C_::kPrThreads>();

    float y[kTB];
#pragma unroll
    for (int j = 0; j < kTB; ++j) y[j] = 0.0f;
    // The scales of both groups of a stage (adjacent fp16) go to this thread's
    // ring slot (stage mod kPf), kPf stages ahead of use.
    const int pt = threadIdx.x - kPr0;
    PairFetcher sf(p.scales, it0, n_it, S, N, Kg, rr, smem_u32(sring) + 4u * (uint32_t)pt, C_::kPrThreads * 4);
    for (int d = 0; d < kPf; ++d) sf.next();

    // Split-tile bookkeeping: at most two pieces of a CTA's range are partial
    // (its first and its last tile); their tickets are resolved at the end.
    int npend = 0;
    int64_t pend_rt0 = -1, pend_rt1 = -1;
    int pend_cnt0 = 0, pend_cnt1 = 0;
    auto finish_piece = [&](int64_t rt) {
      const int64_t n = rt * kRows + rr;
      const bool whole = it0 <= rt * S && it1 >= (rt + 1) * S;
      if (whole) {
        if (n < N) {
#pragma unroll
          for (int j = 0; j < kTB; ++j) {
            const int t = tok0 + j;
            if (t < M) {
              const float v = y[j] * s_escale[t];
              if (p.y_bf16) static_cast<__nv_bfloat16 *>(p.Y)[(int64_t)t * N + n] = __float2bfloat16_rn(v);
              else static_cast<float *>(p.Y)[(int64_t)t * N + n] = v;
            }
          }
        }
      } else {
        const int64_t first = sk_owner(rt * S, T, CT);
        const int64_t last = sk_owner(rt * S + S - 1, T, CT);
        const int slot = (int)((int64_t)blockIdx.x - first);
        float *part = p.ws + (int64_t)slot * M * N;
        if (n < N) {
#pragma unroll
          for (int j = 0; j < kTB; ++j) {
            const int t = tok0 + j;
            if (t < M) __stcg(part + (int64_t)t * N + n, y[j] * s_escale[t]);
          }
        }
        named_bar_pr<C_::kPrThreads>();  // every thread's partials, then one release
        if (threadIdx.x == kPr0) s_ticket[npend] = (int)atom_add_acq_rel_gpu(&p.counters[rt], 1u);
        if (npend == 0) {
          pend_rt0 = rt;
          pend_cnt0 = (int)(last - first + 1);
        } else {
          pend_rt1 = rt;
          pend_cnt1 = (int)(last - first + 1);
        }
        ++npend;
      }
#pragma unroll
      for (int j = 0; j < kTB; ++j) y[j] = 0.0f;
    };

    int g = 0;
    int64_t cur_rt = -1;
    // tile and stage of iteration i, advanced without a division per stage
    int64_t it_rt = it0 / S, it_st = it0 - it_rt * S;
    for (int i = 0; i < n_it; ++i) {
      const int64_t rt = it_rt;
      if (++it_st == S) {
        it_st = 0;
        ++it_rt;
      }
      if (rt != cur_rt) {
        if (cur_rt >= 0) finish_piece(cur_rt);
        cur_rt = rt;
      }
      cp_async_wait<kPf - 1>();  // this thread's copies for stage i have landed
      const uint32_t scb = ld_shared_u32(smem_u32(sring) + 4u * (uint32_t)((i % kPf) * C_::kPrThreads + pt));
      const float sc0 = __half2float(__ushort_as_half((unsigned short)(scb & 0xFFFFu)));
      const float sc1 = __half2float(__ushort_as_half((unsigned short)(scb >> 16)));
      sf.next();  // stage i's pair is consumed: its slot takes stage i + kPf
      // both groups' accumulators, one load wait
      const int r0 = g % kNR, r1 = (g + 1) % kNR;
      const bool ok0 = mbar_wait(&accfull[r0], (uint32_t)(g / kNR) & 1u, kErrTimeoutEpilogue);
      const bool ok1 = mbar_wait(&accfull[r1], (uint32_t)((g + 1) / kNR) & 1u, kErrTimeoutEpilogue);
      tc_fence_after();
      // 16 tokens at a time (8 when the thread has 8): both groups' columns in one
      // load each, one wait -- a TMEM load costs its warp about the same at any width
      constexpr int kW = kTB % 16 == 0 ? 16 : 8;
#pragma unroll
      for (int c0 = 0; c0 < kTB; c0 += kW) {
        const uint32_t col = (uint32_t)(kAccCol + tok0 + c0);
        uint32_t v0[kW], v1[kW];
        if constexpr (kW == 16) {
          tmem_ld_32x32b_x16(lane_base + col + (uint32_t)(BN * r0), v0);
          tmem_ld_32x32b_x16(lane_base + col + (uint32_t)(BN * r1), v1);
        } else {
          tmem_ld_32x32b_x8(lane_base + col + (uint32_t)(BN * r0), v0);
          tmem_ld_32x32b_x8(lane_base + col + (uint32_t)(BN * r1), v1);
        }
        tc_wait_ld();
        if (ok0 && ok1) {
#pragma unroll
          for (int j = 0; j < kW; ++j)
            y[c0 + j] = fmaf(sc1, __uint_as_float(v1[j]), fmaf(sc0, __uint_as_float(v0[j]), y[c0 + j]));
        }
      }
      tc_fence_before();
      mbar_arrive(&accempty[r0]);
      mbar_arrive(&accempty[r1]);
      g += 2;
    }
    if (cur_rt >= 0) finish_piece(cur_rt);
    // the split tiles of this range and their tickets, for the whole CTA's fix-up below
    if (threadIdx.x == kPr0) {
      *s_npend = npend;
      s_pend[0] = (int)pend_rt0;
      s_pend[1] = pend_cnt0;
      s_pend[2] = (int)pend_rt1;
      s_pend[3] = pend_cnt1;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMma0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }

  // Split tiles whose last ticket this CTA took: every thread of the CTA sums
  // (row, token) elements of the tile over its pieces, in increasing slot order.
  // (The ticket's acquire by one promotion thread and the barrier above order these
  // loads after every contributor's partial stores.)
  const int npend_all = *s_npend;
  for (int j = 0; j < npend_all; ++j) {
    const int cnt = s_pend[2 * j + 1];
    const int64_t rt = s_pend[2 * j];
    if (s_ticket[j] != cnt - 1) continue;
    const int64_t elems = (int64_t)kRows * M;
#pragma unroll 2
    for (int64_t e = threadIdx.x; e < elems; e += blockDim.x) {
      const int row = (int)(e % kRows);
      const int64_t t = e / kRows;
      const int64_t n = rt * kRows + row;
      if (n >= N) continue;
      float v[8];
#pragma unroll
      for (int sl = 0; sl < 8; ++sl) v[sl] = sl < cnt ? __ldcg(p.ws + ((int64_t)sl * M + t) * N + n) : 0.0f;
      float acc = 0.0f;
#pragma unroll
      for (int sl = 0; sl < 8; ++sl)
        if (sl < cnt) acc += v[sl];
      for (int sl = 8; sl < cnt; ++sl) acc += __ldcg(p.ws + ((int64_t)sl * M + t) * N + n);
      if (p.y_bf16) static_cast<__nv_bfloat16 *>(p.Y)[t * N + n] = __float2bfloat16_rn(acc);
      else static_cast<float *>(p.Y)[t * N + n] = acc;
    }
    if (threadIdx.x == 0) atomicExch(&p.counters[rt], 0u);
  }
}

// Programmatic dependent launch (W4_PDL=0 turns it off) for both kernels.
inline cudaError_t launch_pdl(const void *func, dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              void **args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  const char *e = getenv("W4_PDL");
  cfg.numAttrs = (e && e[0] == '0') ? 0 : 1;
  return cudaLaunchKernelExC(&cfg, func, args);
}

template <int BN>
cudaError_t launch_main(const CUtensorMap &tmW, const CUtensorMap &tmX, const SkinnyParams &p, int grid,
                        cudaStream_t stream) {
  auto kern = skinny_kernel<BN>;
  static std::atomic<int> smem_set[kAttrDevices];
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void *>(kern), Cfg<BN>::kSmem, smem_set);
  if (e != cudaSuccess) return e;
  CUtensorMap w = tmW, x = tmX;
  SkinnyParams pp = p;
  void *args[] = {&w, &x, &pp};
  return launch_pdl(reinterpret_cast<const void *>(kern), dim3((unsigned)grid), dim3(Cfg<BN>::kThreads),
                    Cfg<BN>::kSmem, stream, args);
}

}  // namespace sk_impl

// Token tile of the skinny kernel for M tokens (a multiple of 16, at least M).
inline int skinny_bn(int64_t M) { return M <= 16 ? 16 : M <= 32 ? 32 : M <= 48 ? 48 : 64; }

cudaError_t launch_stage_x(const void *X, bool x_bf16, const float *awq_s, int64_t M, int64_t K, uint16_t *Xp,
                           int *xexp, cudaStream_t stream) {
  const int bn = skinny_bn(M);
  using namespace sk_impl;
  const void *func = x_bf16 ? (awq_s ? reinterpret_cast<const void *>(stage_x_kernel<true, true>)
                                     : reinterpret_cast<const void *>(stage_x_kernel<true, false>))
                            : (awq_s ? reinterpret_cast<const void *>(stage_x_kernel<false, true>)
                                     : reinterpret_cast<const void *>(stage_x_kernel<false, false>));
  const uint16_t *xp = static_cast<const uint16_t *>(X);
  const float *sp = awq_s;
  int64_t m = M, k = K;
  int b = bn;
  void *args[] = {&xp, &sp, &m, &k, &b, &Xp, &xexp};
  return launch_pdl(func, dim3((unsigned)bn), dim3(kStageThreads), 0, stream, args);
}

cudaError_t launch_skinny(const CUtensorMap &tmW, const CUtensorMap &tmX, const SkinnyParams &p, int grid,
                          cudaStream_t stream) {
  switch (skinny_bn(p.M)) {
    case 16: return sk_impl::launch_main<16>(tmW, tmX, p, grid, stream);
    case 32: return sk_impl::launch_main<32>(tmW, tmX, p, grid, stream);
    case 48: return sk_impl::launch_main<48>(tmW, tmX, p, grid, stream);
    default: return sk_impl::launch_main<64>(tmW, tmX, p, grid, stream);
  }
}

}  // namespace w4
