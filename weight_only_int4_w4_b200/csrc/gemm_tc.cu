// gemm_tc.cu -- K2: prefill W4A16 matmul on the 5th-generation tensor cores.
//
// Prefill is compute-bound (ch. 22 "Advanced inference optimisation", section
// 22.2 table; "LLM inference acceleration" article, section 1.1), so the
// dequantized weights go through tcgen05.mma.  The weight-only path of ch. 22
// section 22.3 (dequantize back to 16 bits, then matmul, fused in one kernel):
//
//   D[n][m] = sum_k W^[n][k] * X[m][k]      (swap-AB: weights are the MMA's M side)
//
// One CTA computes a tile of 128 weight rows x BN tokens over a k-range:
//   warp 0      TMA producer: X tile [BN x 64] (128-byte swizzle) and the packed
//               weight tile [128 rows x 32 bytes] into a ring of NS stages.
//   warps 4..7  dequantize: thread r converts row r's 64 codes of the stage
//               into 16-bit (q - z) * scale (* s[k] for AWQ), rounded once,
//               and stores them with tcgen05.st straight into TMEM, where they
//               are the A operand (TMEM lane = weight row, 2 values per column).
//               With AWQ, warps 4..11: two warps per row, 32 codes each
//               (measured: 8 warps speed up the AWQ kernel at M = 16..64 by
//               6-22% and slow plain weights by 9-15%, so plain keeps 4).
//   warp 1      one thread issues tcgen05.mma (A from TMEM, B = X from shared
//               memory, fp32 accumulator in TMEM) and tcgen05.commit.
//   warps 4..7  epilogue: tcgen05.ld of the accumulator; 32 x 32 chunks staged
//   (..11)      in the idle X ring and written by TMA stores (per-thread stores
//               where Y's rows are not 16-byte multiples, and for split-K).
// TMEM columns: [0, BN) accumulator, then NS stages of 32 columns of A.
// Output tiles that leave a last wave at most half full are cut along K into
// pieces (tail mode, see TcParams), summed by tail_reduce_kernel.
// All waits are bounded (see common.cuh).  No TMA multicast anywhere.
#include "common.cuh"

namespace w4 {

struct TcParams {
  int64_t M, N, K;
  const uint16_t *scales;
  const uint16_t *zeros;
  const float *awq_s;
  void *Y;
  int y_bf16;
  float *ws;           // [splits][M][N] partials (split-K only)
  uint32_t *counters;  // [tiles] arrival counters (split-K only)
  int splits;
  int kb_per_split;  // k-blocks of 64 per split (per tail piece in tail mode)
  int group;         // quantization group: 32, 64 or 128 input channels
  // Tail mode (tail_pieces > 0; splits is then 1): tiles t = y * n-tiles + x
  // below head_tiles are computed whole; each later tile is cut into
  // tail_pieces k-ranges.  Piece 0 runs at the tile's own grid position, pieces
  // 1.. in extra grid rows after the tiles (so they are dispatched last), and
  // piece z of tail tile i writes its fp32 partial tile to
  // ws[i * tail_pieces + z][BN][128]; tail_reduce_kernel sums the pieces.
  int64_t head_tiles;
  int tail_pieces;
  int64_t ntx;  // output tiles along N
  // 1: whole tiles write Y through the tmY tensor map (N * element size is a
  // multiple of 16 bytes and M, N >= 32); tail pieces always use tmT.
  int y_tma;
};

namespace tc_impl {

// Untiled bulk copy, global -> this CTA's shared memory (no multicast).  Both
// addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// tcgen05.st of 16 consecutive 32-bit columns into each thread's own TMEM lane.
__device__ __forceinline__ void tmem_st_32x32b_x16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
      "%13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

constexpr int kBK = 64;   // k per pipeline stage
constexpr int kPStage = 128 * 32;

template <int BN>
struct TcCfg {
  // Pipeline stages.  Measured: 6 ran 10-15% slower than 4 at M = 512..8192;
  // with BN = 64, 12 stages (148 KB) ran up to 50% slower than 4 on plain
  // weights, where 4 stages (50 KB, 256 TMEM columns) let two CTAs share an SM,
  // and 8 or 12 stages changed the AWQ kernel (one CTA per SM) by under 2%.
  static constexpr int kNS = 4;
  static constexpr int kXStage = BN * 128;
  static_assert(BN + 32 * kNS <= 512, "accumulator + A stages exceed TMEM");
  static_assert(kNS * kXStage >= BN * 128 * 4, "the epilogue stages a BN x 128 fp32 tile in the X ring");
  static constexpr uint32_t kTmemCols = (BN + 32 * kNS <= 256) ? 256u : 512u;
  static constexpr int kSStage = kBK * 4;  // AWQ s of the stage's 64 channels (fp32)
  static constexpr int kSmem = 1024 /*align slack*/ + kNS * (kXStage + kPStage + kSStage) + (3 * kNS + 2) * 8;
};

// 64 codes of one row (32 bytes) -> 32 columns of 16-bit pairs (k even in the low half).
// Each byte is moved to bits 15..22 of a word; OR-ing 256.0f (0x43800000) then
// gives the exact fp32 values 256 + q_lo (nibble at bits 15..18) and
// 256 + 16 q_hi (bits 19..22), both inside the 23-bit mantissa.  One FFMA per
// weight turns them into (q - z) * scale: the offsets -(256 + z) * scale and
// -(16 + z) * scale are exact in fp32 (9 + 11 significant bits), so the only
// rounding is that of the final 16-bit conversion.
// (sc0, z0) serve channels 0..31 of the k-block (w0) and (sc1, z1) channels
// 32..63 (w1): the same pair for groups of 64 and 128, two pairs for groups of 32.
template <bool kBf16, bool kAwq>
__device__ __forceinline__ void dequant_row64(const uint4 &w0, const uint4 &w1, float sc0, float z0, float sc1,
                                              float z1, const float *__restrict__ sk, uint32_t (&out)[32]) {
  const uint32_t words[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
  for (int wi = 0; wi < 8; ++wi) {
    const float sc = wi < 4 ? sc0 : sc1, z = wi < 4 ? z0 : z1;
    const float off_lo = -(256.0f + z) * sc;
    const float sc16 = sc * 0.0625f;
    const float off_hi = -(16.0f + z) * sc;
    const uint32_t w = words[wi];
    const uint32_t tb[4] = {w << 15, w << 7, w >> 1, w >> 9};  // byte b at bits 15..22
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const float flo = __uint_as_float(lop3_and_or(tb[b], 0x00078000u, 0x43800000u));
      const float fhi = __uint_as_float(lop3_and_or(tb[b], 0x00780000u, 0x43800000u));
      float vlo = fmaf(flo, sc, off_lo);
      float vhi = fmaf(fhi, sc16, off_hi);
      const int col = wi * 4 + b;
      if constexpr (kAwq) {
        const float2 s2 = *reinterpret_cast<const float2 *>(sk + 2 * col);
        vlo *= s2.x;
        vhi *= s2.y;
      }
      if constexpr (kBf16) {
        const __nv_bfloat162 v = __floats2bfloat162_rn(vlo, vhi);
        out[col] = *reinterpret_cast<const uint32_t *>(&v);
      } else {
        const __half2 v = __floats2half2_rn(vlo, vhi);
        out[col] = *reinterpret_cast<const uint32_t *>(&v);
      }
    }
  }
}

// Half of a row's k-block: 32 codes (16 bytes) -> 16 columns of 16-bit pairs, one (sc, z).
template <bool kBf16, bool kAwq>
__device__ __forceinline__ void dequant_row32(const uint4 &w4v, float sc, float z, const float *__restrict__ sk,
                                              uint32_t (&out)[16]) {
  const uint32_t words[4] = {w4v.x, w4v.y, w4v.z, w4v.w};
  const float off_lo = -(256.0f + z) * sc;
  const float sc16 = sc * 0.0625f;
  const float off_hi = -(16.0f + z) * sc;
#pragma unroll
  for (int wi = 0; wi < 4; ++wi) {
    const uint32_t w = words[wi];
    const uint32_t tb[4] = {w << 15, w << 7, w >> 1, w >> 9};  // byte b at bits 15..22
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const float flo = __uint_as_float(lop3_and_or(tb[b], 0x00078000u, 0x43800000u));
      const float fhi = __uint_as_float(lop3_and_or(tb[b], 0x00780000u, 0x43800000u));
      float vlo = fmaf(flo, sc, off_lo);
      float vhi = fmaf(fhi, sc16, off_hi);
      const int col = wi * 4 + b;
      if constexpr (kAwq) {
        const float2 s2 = *reinterpret_cast<const float2 *>(sk + 2 * col);
        vlo *= s2.x;
        vhi *= s2.y;
      }
      if constexpr (kBf16) {
        const __nv_bfloat162 v = __floats2bfloat162_rn(vlo, vhi);
        out[col] = *reinterpret_cast<const uint32_t *>(&v);
      } else {
        const __half2 v = __floats2half2_rn(vlo, vhi);
        out[col] = *reinterpret_cast<const uint32_t *>(&v);
      }
    }
  }
}

// Dequant / epilogue warps: 4 (warps 4..7) for plain weights; 8 (warps 4..11) with
// AWQ scales, whose extra multiply per weight makes the dequant the longer stage.
template <bool kAwq>
struct TcWarps {
  static constexpr int kHalves = kAwq ? 2 : 1;      // warps per TMEM lane quadrant
  static constexpr int kEpi = 128 * kHalves;        // dequant / epilogue threads
  static constexpr int kThreads = 128 + kEpi;
};

// AND of a predicate over the kEpi dequant/epilogue threads (named barrier 1).
template <int kEpi>
__device__ __forceinline__ bool epilogue_vote(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "barrier.cta.red.and.pred q, 1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "n"(kEpi)
      : "memory");
  return r != 0;
}

template <int BN, bool kBf16, bool kAwq, bool kTail>
__global__ void __launch_bounds__(TcWarps<kAwq>::kThreads, kAwq ? 1 : 2)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmP,
                   const __grid_constant__ CUtensorMap tmY, const __grid_constant__ CUtensorMap tmT,
                   const TcParams p) {
  using Cfg = TcCfg<BN>;
  constexpr int kNS = Cfg::kNS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sX = smem;
  uint8_t *sP = sX + kNS * Cfg::kXStage;
  float *sS = reinterpret_cast<float *>(sP + kNS * kPStage);
  uint64_t *full = reinterpret_cast<uint64_t *>(sS + kNS * kBK);
  uint64_t *empty = full + kNS;
  uint64_t *afull = empty + kNS;
  uint64_t *accfull = afull + kNS;
  uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(accfull + 1);
  int *s_last = reinterpret_cast<int *>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t M = p.M, N = p.N, K = p.K;
  const int total_kb = (int)(K / kBK);
  int64_t tile_n = blockIdx.x, tile_m = blockIdx.y;
  int split = blockIdx.z, kbps = p.kb_per_split;
  int64_t tail_unit = -1;  // tail mode: this CTA's partial slot, -1 for a whole tile
  // (A separate instantiation: compiled into every launch, the tail mapping
  // made the plain kernel 15-18 % slower on B200.)
  if constexpr (kTail) {
    const int64_t tiles_m = (M + BN - 1) / BN;
    const int64_t t = (int64_t)blockIdx.y * gridDim.x + blockIdx.x;
    if (blockIdx.y < tiles_m) {
      if (t < p.head_tiles) kbps = total_kb;                   // a whole tile
      else tail_unit = (t - p.head_tiles) * p.tail_pieces;  // piece 0 of a tail tile
    } else {  // rows past the tiles: pieces 1.. of the tail tiles, then idle CTAs
      const int pm1 = p.tail_pieces - 1;
      const int e = (int)(t - tiles_m * gridDim.x);
      const int64_t rest = tiles_m * gridDim.x - p.head_tiles;
      if (e >= rest * pm1) return;
      const int tt = e / pm1;
      split = 1 + e % pm1;
      tail_unit = (int64_t)tt * p.tail_pieces + split;
      const int64_t tile = p.head_tiles + tt;
      tile_n = tile % gridDim.x;
      tile_m = tile / gridDim.x;
    }
  }
  const int64_t n0 = tile_n * 128;
  const int64_t m0 = tile_m * BN;
  const int kb0 = split * kbps;
  const int kb1 = min(kb0 + kbps, total_kb);
  const int nkb = max(kb1 - kb0, 0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kNS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&afull[s], TcWarps<kAwq>::kEpi);
    }
    mbar_init(accfull, 1);
    fence_barrier_init();
    prefetch_tensormap(&tmX);
    prefetch_tensormap(&tmP);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    if (lane == 0) {
      for (int i = 0; i < nkb; ++i) {
        const int s = i % kNS;
        const uint32_t ph = (uint32_t)(i / kNS) & 1u;
        if (!mbar_wait(&empty[s], ph ^ 1u, kErrTimeoutTma)) break;
        mbar_arrive_expect_tx(&full[s], Cfg::kXStage + kPStage + (kAwq ? Cfg::kSStage : 0));
        const int kb = kb0 + i;
        tma_load_2d(sX + s * Cfg::kXStage, &tmX, &full[s], kb * kBK, (int32_t)m0);
        tma_load_2d(sP + s * kPStage, &tmP, &full[s], kb * (kBK / 2), (int32_t)n0);
        if constexpr (kAwq) bulk_load(sS + s * kBK, p.awq_s + (int64_t)kb * kBK, Cfg::kSStage, &full[s]);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_f16(kBf16, BN);
      for (int i = 0; i < nkb; ++i) {
        const int s = i % kNS;
        const uint32_t ph = (uint32_t)(i / kNS) & 1u;
        if (!mbar_wait(&full[s], ph, kErrTimeoutMma)) break;
        if (!mbar_wait(&afull[s], ph, kErrTimeoutMma)) break;
        tc_fence_after();
        const uint32_t a_tmem = tmem + (uint32_t)(BN + s * 32);
        const uint64_t bdesc = smem_desc_k_sw128(smem_u32(sX + s * Cfg::kXStage));
#pragma unroll
        for (int j = 0; j < kBK / 16; ++j)
          tc_mma_ts(tmem, a_tmem + 8 * j, bdesc + (uint64_t)(2 * j), idesc, (i > 0 || j > 0) ? 1u : 0u);
        tc_commit(&empty[s]);
      }
      tc_commit(accfull);
    }
  } else if (warp >= 4) {
    constexpr int kHalves = TcWarps<kAwq>::kHalves;
    constexpr int kEpi = TcWarps<kAwq>::kEpi;
    // Warp w serves TMEM lane quadrant w % 4 (rows 32 (w % 4) ..+32).  With two
    // warps per quadrant (w and w + 4), the first takes channels 0..31 of every
    // k-block and the second 32..63.
    const int q = warp & 3;
    const int h = kHalves == 2 ? (warp - 4) >> 2 : 0;
    const int r = q * 32 + lane;
    const int64_t n = n0 + r;
    const bool row_ok = n < N;
    const int G = p.group;
    const int64_t Kg = K / G;
    const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
    // This row's scales and zeros.  When rows start on 16-byte boundaries
    // (Kg % 8 == 0) they are read 8 groups at a time, one 16-byte chunk ahead of
    // use, so the load latency overlaps the dequantization of earlier groups
    // instead of stalling the stage that needs them.
    const uint16_t *sc_row = p.scales + (row_ok ? n : 0) * Kg;
    const uint16_t *z_row = p.zeros + (row_ok ? n : 0) * Kg;
    const bool vec = (Kg & 7) == 0;
    const int64_t nch = Kg >> 3;
    uint4 scv = make_uint4(0, 0, 0, 0), zv = scv, scn = scv, zn = scv;
    auto fetch = [&](int64_t c, uint4 &a, uint4 &b) {
      if (row_ok && c < nch) {
        a = __ldg(reinterpret_cast<const uint4 *>(sc_row) + c);
        b = __ldg(reinterpret_cast<const uint4 *>(z_row) + c);
      } else {
        a = make_uint4(0, 0, 0, 0);
        b = a;
      }
    };
    // first group of this thread's k-range; its chunk is fetched before the loop
    const int64_t g_first = G == 32 ? 2 * (int64_t)kb0 + h : (int64_t)kb0 / (G / 64);
    int64_t cur = (g_first >> 3) - 1;  // chunk held in (scv, zv); the next one is in (scn, zn)
    if (vec) fetch(cur + 1, scn, zn);
    auto group_params = [&](int64_t g, float &gs, float &gz) {
      if (vec) {
        const int64_t c = g >> 3;  // groups advance by at most one chunk at a time
        if (c != cur) {
          scv = scn;
          zv = zn;
          cur = c;
          fetch(c + 1, scn, zn);
        }
        const int e = (int)(g & 7), wsel = e >> 1, sh = 16 * (e & 1);
        const uint32_t a = wsel == 0 ? scv.x : wsel == 1 ? scv.y : wsel == 2 ? scv.z : scv.w;
        const uint32_t b = wsel == 0 ? zv.x : wsel == 1 ? zv.y : wsel == 2 ? zv.z : zv.w;
        gs = half_bits_to_float((uint16_t)(a >> sh));
        gz = half_bits_to_float((uint16_t)(b >> sh));
      } else {
        gs = row_ok ? half_bits_to_float(__ldg(sc_row + g)) : 0.0f;
        gz = row_ok ? half_bits_to_float(__ldg(z_row + g)) : 0.0f;
      }
    };
    float sc = 0.0f, z = 0.0f, sc1 = 0.0f, z1 = 0.0f;
    bool ok = true;
    for (int i = 0; i < nkb; ++i) {
      const int s = i % kNS;
      const uint32_t ph = (uint32_t)(i / kNS) & 1u;
      const int kb = kb0 + i;
      if (G == 32) {  // two groups per 64-channel k-block
        group_params(2 * (int64_t)kb + h, sc, z);
        if (kHalves == 1) group_params(2 * (int64_t)kb + 1, sc1, z1);
      } else if (i == 0 || (kb & (G / 64 - 1)) == 0) {  // a group spans G / 64 k-blocks
        group_params((int64_t)kb / (G / 64), sc, z);
        sc1 = sc;
        z1 = z;
      }
      if (!mbar_wait(&full[s], ph, kErrTimeoutDequant)) { ok = false; break; }
      const uint4 *src = reinterpret_cast<const uint4 *>(sP + s * kPStage + r * 32);
      if constexpr (kHalves == 2) {
        uint32_t out[16];
        dequant_row32<kBf16, kAwq>(src[h], sc, z, sS + s * kBK + 32 * h, out);
        tmem_st_32x32b_x16(lane_base + (uint32_t)(BN + s * 32 + 16 * h), out);
      } else {
        uint32_t out[32];
        dequant_row64<kBf16, kAwq>(src[0], src[1], sc, z, sc1, z1, sS + s * kBK, out);
        tmem_st_32x32b_x32(lane_base + (uint32_t)(BN + s * 32), out);
      }
      // (Deferring this wait until the next stage is dequantized measured 5-10% slower.)
      tc_wait_st();
      tc_fence_before();
      mbar_arrive(&afull[s]);
    }

    // ---- epilogue (the decision to run it is made uniform over the kEpi threads,
    // so the named barriers below are reached by all of them or by none)
    bool go = ok && nkb > 0 && mbar_wait(accfull, 0, kErrTimeoutEpilogue);
    go = epilogue_vote<kEpi>(go);
    if (go) {
      tc_fence_after();
      const bool direct = p.splits == 1 && tail_unit < 0;
      if (tail_unit >= 0 || (direct && p.y_tma)) {
        // Each warp stages its 32 rows x 32 tokens of a chunk in the X ring (idle
        // once the accumulator is complete) as [token][row] and writes the chunk
        // with one TMA store, which clips rows >= M and columns >= N.  Measured on
        // B200: per-thread stores of the same tile took 5-13 us per CTA.
        const bool out16 = tail_unit < 0 && p.y_bf16;
        const int esz = out16 ? 2 : 4;
        uint8_t *stage = sX + (size_t)q * (BN / 32) * (32 * 32 * esz);
#pragma unroll 1
        for (int c = h * (BN / 32 / kHalves); c < (h + 1) * (BN / 32 / kHalves); ++c) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(lane_base + (uint32_t)(c * 32), v);
          tc_wait_ld();
          if (m0 + c * 32 >= M) continue;
          uint8_t *chunk = stage + (size_t)c * (32 * 32 * esz);
          if (out16) {
            __nv_bfloat16 *c16 = reinterpret_cast<__nv_bfloat16 *>(chunk);
#pragma unroll
            for (int j = 0; j < 32; ++j) c16[j * 32 + lane] = __float2bfloat16_rn(__uint_as_float(v[j]));
          } else {
            float *c32 = reinterpret_cast<float *>(chunk);
#pragma unroll
            for (int j = 0; j < 32; ++j) c32[j * 32 + lane] = __uint_as_float(v[j]);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            if (tail_unit >= 0) tma_store_2d(&tmT, chunk, q * 32, (int32_t)(tail_unit * BN + c * 32));
            else if (n0 + q * 32 < N) tma_store_2d(&tmY, chunk, (int32_t)(n0 + q * 32), (int32_t)(m0 + c * 32));
            bulk_commit_group();
          }
        }
        if (lane == 0) bulk_wait_read_all();
        __syncwarp();
      } else {
        // Per-thread stores (Y rows not 16-byte multiples, or split-K partials):
        // this row's fp32 destination, Y or the split's partial rows, with a
        // token stride of N, or the bf16 Y row.
        const bool out16 = direct && p.y_bf16;
        float *dst = direct ? static_cast<float *>(p.Y) + m0 * N + n : p.ws + ((int64_t)split * M + m0) * N + n;
        __nv_bfloat16 *dst16 = static_cast<__nv_bfloat16 *>(p.Y) + m0 * N + n;
#pragma unroll 1
        for (int c = h * (BN / 32 / kHalves); c < (h + 1) * (BN / 32 / kHalves); ++c) {  // this warp's columns
          uint32_t v[32];
          tmem_ld_32x32b_x32(lane_base + (uint32_t)(c * 32), v);
          tc_wait_ld();
          if (!row_ok) continue;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int t = c * 32 + j;
            if (m0 + t < M) {
              const float val = __uint_as_float(v[j]);
              if (out16) dst16[t * N] = __float2bfloat16_rn(val);
              else dst[t * N] = val;
            }
          }
        }
      }
      if (!direct && tail_unit < 0) {
        // last CTA of this output tile to arrive sums the split-K partials
        __threadfence();
        asm volatile("bar.sync 1, %0;" ::"n"(kEpi) : "memory");
        const int64_t tile = tile_m * gridDim.x + tile_n;
        if (r == 0 && h == 0) {
          const uint32_t prev = atomicAdd(&p.counters[tile], 1u);
          *s_last = prev == (uint32_t)(p.splits - 1);
        }
        asm volatile("bar.sync 1, %0;" ::"n"(kEpi) : "memory");
        if (*s_last) {
          __threadfence();
          if (row_ok) {
            // 8 tokens x 4 splits of partials are loaded before they are added, so
            // 32 independent loads are in flight (one token and one split at a
            // time left every step waiting on L2).  The splits are summed in
            // increasing order for every token.
            const int j_begin = h * (BN / kHalves);
            const int64_t rem = M - m0;
            const int j_end = rem < j_begin + BN / kHalves ? (int)rem : j_begin + BN / kHalves;
            for (int j0 = j_begin; j0 < j_end; j0 += 8) {
              float acc[8];
#pragma unroll
              for (int u = 0; u < 8; ++u) acc[u] = 0.0f;
              int s = 0;
              for (; s + 4 <= p.splits; s += 4) {
                float v[4][8];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                  const float *part = p.ws + ((int64_t)(s + c) * M + m0 + j0) * N + n;
#pragma unroll
                  for (int u = 0; u < 8; ++u) v[c][u] = j0 + u < j_end ? __ldcg(part + (int64_t)u * N) : 0.0f;
                }
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                  for (int u = 0; u < 8; ++u) acc[u] += v[c][u];
              }
              for (; s < p.splits; ++s) {
                const float *part = p.ws + ((int64_t)s * M + m0 + j0) * N + n;
#pragma unroll
                for (int u = 0; u < 8; ++u)
                  if (j0 + u < j_end) acc[u] += __ldcg(part + (int64_t)u * N);
              }
#pragma unroll
              for (int u = 0; u < 8; ++u) {
                if (j0 + u >= j_end) break;
                const int64_t m = m0 + j0 + u;
                if (p.y_bf16) static_cast<__nv_bfloat16 *>(p.Y)[m * N + n] = __float2bfloat16_rn(acc[u]);
                else static_cast<float *>(p.Y)[m * N + n] = acc[u];
              }
            }
          }
          if (r == 0 && h == 0) atomicExch(&p.counters[tile], 0u);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg::kTmemCols);
  }
}

template <int BN, bool kBf16, bool kAwq>
cudaError_t launch_t(const CUtensorMap &tmX, const CUtensorMap &tmP, const CUtensorMap &tmY, const CUtensorMap &tmT,
                     const TcParams &p, cudaStream_t stream) {
  using Cfg = TcCfg<BN>;
  auto kern = p.tail_pieces > 0 ? gemm_tc_kernel<BN, kBf16, kAwq, true> : gemm_tc_kernel<BN, kBf16, kAwq, false>;
  static std::atomic<int> smem_set[kAttrDevices][2];  // largest size already set, per device and variant
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void *>(kern), Cfg::kSmem, smem_set[p.tail_pieces > 0]);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((p.N + 127) / 128), (unsigned)((p.M + BN - 1) / BN), (unsigned)p.splits);
  if (p.tail_pieces > 0) {  // extra rows of CTAs for pieces 1.. of the tail tiles
    const int64_t extra = ((int64_t)grid.x * grid.y - p.head_tiles) * (p.tail_pieces - 1);
    grid.y += (unsigned)((extra + grid.x - 1) / grid.x);
  }
  kern<<<grid, TcWarps<kAwq>::kThreads, Cfg::kSmem, stream>>>(tmX, tmP, tmY, tmT, p);
  return cudaGetLastError();
}

// Sums the tail pieces' partial tiles in piece order and writes Y.  One thread
// per 4 output channels of one token of one tail tile; partials [u][BN][128].
template <int BN>
__global__ void __launch_bounds__(256) tail_reduce_kernel(const TcParams p) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t q = idx % 32, j = (idx / 32) % BN, tt = idx / (32 * BN);
  const int64_t tiles = p.ntx * ((p.M + BN - 1) / BN);
  if (tt >= tiles - p.head_tiles) return;
  const int64_t t = p.head_tiles + tt;
  const int64_t m = (t / p.ntx) * BN + j;
  const int64_t n = (t % p.ntx) * 128 + 4 * q;
  if (m >= p.M || n >= p.N) return;
  const float4 *src = reinterpret_cast<const float4 *>(p.ws) + (tt * p.tail_pieces * BN + j) * 32 + q;
  float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  int s = 0;
  for (; s + 4 <= p.tail_pieces; s += 4) {  // 4 loads in flight, summed in piece order
    float4 v[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) v[c] = __ldcg(src + (int64_t)(s + c) * BN * 32);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      acc[0] += v[c].x; acc[1] += v[c].y; acc[2] += v[c].z; acc[3] += v[c].w;
    }
  }
  for (; s < p.tail_pieces; ++s) {
    const float4 v = __ldcg(src + (int64_t)s * BN * 32);
    acc[0] += v.x; acc[1] += v.y; acc[2] += v.z; acc[3] += v.w;
  }
  const int nv = p.N - n < 4 ? (int)(p.N - n) : 4;
  if (p.y_bf16) {
    __nv_bfloat16 *y = static_cast<__nv_bfloat16 *>(p.Y) + m * p.N + n;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (i < nv) y[i] = __float2bfloat16_rn(acc[i]);
  } else {
    float *y = static_cast<float *>(p.Y) + m * p.N + n;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (i < nv) y[i] = acc[i];
  }
}

template <int BN>
cudaError_t launch_tail_reduce_bn(const TcParams &p, cudaStream_t stream) {
  const int64_t tiles = p.ntx * ((p.M + BN - 1) / BN);
  const int64_t threads = (tiles - p.head_tiles) * BN * 32;
  if (threads <= 0) return cudaSuccess;
  tail_reduce_kernel<BN><<<(unsigned)((threads + 255) / 256), 256, 0, stream>>>(p);
  return cudaGetLastError();
}

template <int BN>
cudaError_t launch_bn(const CUtensorMap &tmX, const CUtensorMap &tmP, const CUtensorMap &tmY,
                      const CUtensorMap &tmT, const TcParams &p, bool bf16, cudaStream_t stream) {
  const bool awq = p.awq_s != nullptr;
  if (bf16)
    return awq ? launch_t<BN, true, true>(tmX, tmP, tmY, tmT, p, stream)
               : launch_t<BN, true, false>(tmX, tmP, tmY, tmT, p, stream);
  return awq ? launch_t<BN, false, true>(tmX, tmP, tmY, tmT, p, stream)
             : launch_t<BN, false, false>(tmX, tmP, tmY, tmT, p, stream);
}

}  // namespace tc_impl

cudaError_t launch_gemm_tc(const CUtensorMap &tmX, const CUtensorMap &tmP, const CUtensorMap &tmY,
                           const CUtensorMap &tmT, const TcParams &p, bool x_bf16, int bn,
                           cudaStream_t stream) {
  switch (bn) {
    case 64: return tc_impl::launch_bn<64>(tmX, tmP, tmY, tmT, p, x_bf16, stream);
    case 128: return tc_impl::launch_bn<128>(tmX, tmP, tmY, tmT, p, x_bf16, stream);
    default: return tc_impl::launch_bn<256>(tmX, tmP, tmY, tmT, p, x_bf16, stream);
  }
}

// Tail mode only: the reduction of the tail pieces, enqueued after the GEMM.
cudaError_t launch_tail_reduce(const TcParams &p, int bn, cudaStream_t stream) {
  switch (bn) {
    case 64: return tc_impl::launch_tail_reduce_bn<64>(p, stream);
    case 128: return tc_impl::launch_tail_reduce_bn<128>(p, stream);
    default: return tc_impl::launch_tail_reduce_bn<256>(p, stream);
  }
}

}  // namespace w4
