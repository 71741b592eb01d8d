// libw4.cu -- the C ABI of libw4 (declared in include/w4.h) and the single
// translation unit that holds every kernel of the library.
//
// Host side only: argument validation (before anything is launched), the
// per-call launch plan (which kernel, how many k-slices, grid), TMA
// descriptor encoding, and error reporting.  The arithmetic is in the kernels.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>

#include "common.cuh"
#include "gemm_tc.cu"
#include "gemm_skinny.cu"
#include "gemv_mma.cu"
#include "quantize.cu"
#include "awq_search.cu"
#include "outliers.cu"
#include "gptq.cu"
#include "w4.h"

namespace w4 {
cudaError_t launch_mean_abs(const void *X, bool x_bf16, int64_t Mc, int64_t K, double *m, cudaStream_t stream);
cudaError_t launch_awq_scale(const double *m, int64_t K, double a, float *s, cudaStream_t stream);
cudaError_t launch_dense_ref(const void *X, bool x_bf16, const float *W, int64_t Mc, int64_t N, int64_t K, float *Y,
                             cudaStream_t stream);
cudaError_t launch_sq_err(const float *A, const float *B, int64_t count, double *partial, double *err,
                          cudaStream_t stream);
cudaError_t launch_quantize(const void *W, int dtype, const float *awq_s, int64_t N, int64_t K, int group,
                            bool symmetric, const uint32_t *tau, uint8_t *packed, uint16_t *scales, uint16_t *zeros,
                            uint8_t *codes, int sm_count, cudaStream_t stream);
cudaError_t launch_outlier_threshold(const float *W, int64_t E, int64_t count, uint32_t *state, uint32_t *hist,
                                     int sm_count, cudaStream_t stream);
cudaError_t launch_outlier_csr(const float *W, int64_t N, int64_t K, const uint32_t *state, int32_t *counts,
                               int32_t *row_ptr, int64_t cap, int32_t *col, uint16_t *val, cudaStream_t stream);
cudaError_t launch_gptq_hinv(const void *X, bool x_bf16, int64_t Mc, int64_t K, double damp_frac, double *H,
                             double *Lc, double *Li, int *bad, cudaStream_t stream);
cudaError_t launch_gptq_sweep(const float *W, int64_t N, int64_t K, int group, const double *Li, double *Wd,
                              uint8_t *codes, uint16_t *scales, uint16_t *zeros, cudaStream_t stream);
cudaError_t launch_sparse_add(const void *X, bool x_bf16, int64_t M, int64_t N, int64_t K, const int32_t *row_ptr,
                              const int32_t *col, const uint16_t *val, void *Y, bool y_bf16, cudaStream_t stream);
cudaError_t launch_pack(const uint8_t *codes, int64_t N, int64_t K, uint8_t *packed, int sm_count,
                        cudaStream_t stream);
}  // namespace w4

namespace {

thread_local std::string t_last_error;

w4_status fail(w4_status s, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  t_last_error = buf;
  return s;
}

w4_status cuda_fail(cudaError_t e, const char *what) {
  return fail(W4_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr int kMaxDevices = 64;
int g_sm_count[kMaxDevices];
std::mutex g_mu;

// SM count of the current device (148 on B200); cached per device.
cudaError_t current_sm_count(int *out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_sm_count[dev] == 0) {
    int n = 0;
    e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    g_sm_count[dev] = n;
  }
  *out = g_sm_count[dev];
  return cudaSuccess;
}

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  std::call_once(g_encode_once, [] {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode;
}

int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

// A 2-D tensor map is a pure function of its data type, address, sizes, row
// stride, box, swizzle and L2 promotion, so an encoded map is reused whenever
// the same key comes back (repeated calls on the same layer).  A small
// per-thread cache saves the driver call; entries are replaced round-robin.
struct MapKey {
  int dtype, swizzle, l2;
  const void *addr;
  uint64_t d0, d1, stride;
  uint32_t b0, b1;
  bool operator==(const MapKey &o) const {
    return dtype == o.dtype && swizzle == o.swizzle && l2 == o.l2 && addr == o.addr && d0 == o.d0 && d1 == o.d1 &&
           stride == o.stride && b0 == o.b0 && b1 == o.b1;
  }
};
constexpr int kMapCache = 32;
struct MapCache {
  MapKey key[kMapCache];
  CUtensorMap map[kMapCache];
  int n = 0, next = 0;
};
thread_local MapCache t_maps;

CUresult encode_2d(PFN_cuTensorMapEncodeTiled_v12000 enc, CUtensorMap *out, CUtensorMapDataType dt, const void *addr,
                   uint64_t d0, uint64_t d1, uint64_t stride_bytes, uint32_t b0, uint32_t b1,
                   CUtensorMapSwizzle swz, CUtensorMapL2promotion l2) {
  const MapKey k{(int)dt, (int)swz, (int)l2, addr, d0, d1, stride_bytes, b0, b1};
  for (int i = 0; i < t_maps.n; ++i)
    if (t_maps.key[i] == k) {
      *out = t_maps.map[i];
      return CUDA_SUCCESS;
    }
  const cuuint64_t dims[2] = {d0, d1};
  const cuuint64_t strides[1] = {stride_bytes};
  const cuuint32_t box[2] = {b0, b1};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(out, dt, 2, const_cast<void *>(addr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                   l2, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return r;
  const int slot = t_maps.n < kMapCache ? t_maps.n++ : (t_maps.next++ % kMapCache);
  t_maps.key[slot] = k;
  t_maps.map[slot] = *out;
  return CUDA_SUCCESS;
}


enum Path { kPathGemv = 1, kPathTc = 2, kPathSkinny = 3 };

// Workspace layout: [0, 64 KiB) arrival counters (one per 16-row block),
// [64 KiB, 128 KiB) reserved, then fp32
// partials.  The counter regions are the same for every call, so partials left
// behind by one call never land on the counters of the next; every counter is
// reset to zero by the last CTA (or warp) that uses it.
constexpr size_t kSplitCounterBytes = 65536;
constexpr size_t kSchedBytes = 65536;
constexpr size_t kCounterBytes = kSplitCounterBytes + kSchedBytes;
constexpr int64_t kMaxSplitCounters = kSplitCounterBytes / 4;
constexpr int kGemvXsMax = 40 * 1024;  // staged-activation budget per CTA

struct GemmPlan {
  int path = 0;
  // K1 (and K3: grid_x CTAs, slots partial slots per tile)
  int t8 = 1, kr = 2, kslices = 1, grid_x = 1, xs_bytes = 0, slots = 1;
  bool sc_tma = false;
  // K2
  int bn = 256, splits = 1, kb_per_split = 1;
  int64_t head_tiles = 0;  // tail mode (tail_pieces > 0): tiles computed whole
  int tail_pieces = 0;
  // K3 workspace regions (bytes from the start of the workspace)
  size_t xp_off = 0, xexp_off = 0, part_off = 0;
  size_t ws_bytes = 0;
};

int t8_for(int64_t M) { return M <= 8 ? 1 : M <= 16 ? 2 : M <= 32 ? 4 : 8; }

// Path forced through the environment (W4_FORCE_PATH=gemv|skinny|tc), for tests.
int forced_path() {
  const char *e = getenv("W4_FORCE_PATH");
  if (!e) return 0;
  if (!strcmp(e, "gemv")) return kPathGemv;
  if (!strcmp(e, "tc")) return kPathTc;
  if (!strcmp(e, "skinny")) return kPathSkinny;
  return 0;
}

size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

// CTAs of the decode kernel resident per SM (shared memory, and at most 3 CTAs of
// 288 threads for the register file).
int gemv_ctas_per_sm(int xs_bytes, int t8) {
  const int per = w4::gemv_smem_bytes(xs_bytes, t8) + 1024;
  int n = (228 * 1024) / per;
  return n < 1 ? 1 : (n > 3 ? 3 : n);
}

GemmPlan plan_gemv(int64_t M, int64_t N, int64_t K, bool awq, int sm) {
  GemmPlan p;
  p.path = kPathGemv;
  p.t8 = t8_for(M);
  const int64_t Kg = K / w4::kGroup;
  const int64_t RT = cdiv(N, 64);
  const int64_t RB16 = cdiv(N, 16);
  p.sc_tma = (Kg % 8) == 0;
  // k-slices are whole pipeline stages of 4 groups; the longest one whose
  // activations fit the staging budget (every CTA stages its whole k-slice).
  // The static partition balances the work across CTAs, so K is split only
  // when the activations do not fit.
  int64_t kr_max = std::min<int64_t>(cdiv(Kg, 4) * 4, 4096);
  while (kr_max > 4 && w4::gemv_xs_bytes((int)kr_max, M, awq) > kGemvXsMax) kr_max -= 4;
  const int64_t ks0 = cdiv(Kg, kr_max);
  // balanced slices: the shortest slice length (whole stages) that gives ks slices
  auto kr_for = [&](int64_t ks) { return cdiv(cdiv(Kg, ks), 4) * 4; };
  auto slots_for = [&](int64_t kr_c) {
    return (int64_t)sm * gemv_ctas_per_sm(w4::gemv_xs_bytes((int)kr_c, M, awq), p.t8);
  };
  int64_t kr = kr_for(ks0);
  int64_t C = -1;
  if (RT * ks0 <= slots_for(kr)) {
    // Few row tiles: one whole tile per CTA (no tile is shared, outputs written
    // directly when K is not split), with K split into the most slices that keep
    // RT * slices CTAs resident and at least 6 stages per slice.
    for (int64_t ks = ks0 + 1;; ++ks) {
      const int64_t kr_c = kr_for(ks);
      if (cdiv(Kg, kr_c) != ks) {
        if (kr_c <= 4) break;
        continue;
      }
      if (kr_c / 4 < 6 || RT * ks > slots_for(kr_c)) break;
      kr = kr_c;
    }
    C = RT;
  }
  int64_t ks = cdiv(Kg, kr);
  p.kr = (int)kr;
  p.kslices = (int)ks;
  p.xs_bytes = w4::gemv_xs_bytes(p.kr, M, awq);
  // stages per row tile: S_full for every k-slice but the last, S_last for the last
  const int64_t S_full = kr / 4;
  const int64_t S_last = cdiv(Kg - (ks - 1) * kr, 4);
  const int64_t slots = slots_for(kr);
  if (C < 0) C = std::max<int64_t>(1, slots / ks);  // many row tiles: balanced partition
  C = std::min<int64_t>(C, RT * std::min(S_full, S_last));  // every CTA gets >= 1 iteration
  p.grid_x = (int)C;
  // Partial slots per (k-slice, row tile): a tile's S iterations meet at most
  // floor((S - 2) / L) + 2 CTA ranges, L = the shortest range, floor(S * RT / C).
  auto bound = [&](int64_t S) -> int64_t {
    if (S <= 1) return 1;
    const int64_t L = (S * RT) / C;
    return std::min<int64_t>(C, (S - 2) / L + 2);
  };
  p.slots = (int)std::max(bound(S_full), bound(S_last));
  bool partials = ks > 1 || RT % C != 0;
  if (partials && RB16 > kMaxSplitCounters) {
    // more row blocks than arrival counters: one CTA per row tile (no partials) if
    // K is not split, else not served by this kernel
    if (ks > 1) {
      p.path = 0;
      return p;
    }
    p.grid_x = (int)RT;
    p.slots = 1;
    partials = false;
  }
  p.ws_bytes = kCounterBytes + (partials ? (size_t)ks * p.slots * M * N * 4 : 0);
  return p;
}

// CTAs of the tensor-core kernel resident per SM.  Plain weights with BN <= 128
// fit two (256 threads x at most 128 registers, <= 83 KB of shared memory, 256
// TMEM columns each); the AWQ kernel (384 threads x 128 registers) and BN = 256
// (150 KB of shared memory) fit one.
int tc_ctas_per_sm(int bn, bool awq) { return (awq || bn == 256) ? 1 : 2; }

// ws_cap: the partials must fit this many workspace bytes (fewer K splits otherwise).
GemmPlan plan_tc(int64_t M, int64_t N, int64_t K, bool awq, int sm, size_t ws_cap = SIZE_MAX) {
  GemmPlan p;
  p.path = kPathTc;
  p.bn = M <= 64 ? 64 : (M <= 128 ? 128 : 256);
  const int64_t tiles = cdiv(N, 128) * cdiv(M, p.bn);
  const int64_t total_kb = K / 64;
  // Split K when the output tiles do not fill the SMs (each split keeps >= 8
  // k-blocks), and further toward the second resident CTA per SM where that
  // fits only while each split keeps >= 32 k-blocks.  Measured on B200: the
  // second slot made 70B layers at M = 16..128 up to 30 % faster, while the
  // 4096-deep 8B layers, cut into 8 to 11 k-blocks per split, ran slower.
  int64_t splits = 1;
  if (tiles < sm && tiles <= kMaxSplitCounters)
    splits = std::max<int64_t>(1, std::min<int64_t>(sm / tiles, total_kb / 8));
  const int64_t slots = (int64_t)sm * tc_ctas_per_sm(p.bn, awq);
  if (tiles < slots && tiles <= kMaxSplitCounters)
    splits = std::max<int64_t>(splits, std::min<int64_t>(slots / tiles, total_kb / 32));
  while (splits > 1 && kCounterBytes + (size_t)splits * M * N * 4 > ws_cap) --splits;
  int64_t kbps = cdiv(total_kb, splits);
  splits = cdiv(total_kb, kbps);
  p.splits = (int)splits;
  p.kb_per_split = (int)kbps;
  if (splits > 1) p.ws_bytes = kCounterBytes + (size_t)splits * M * N * 4;
  // Tail split: where the tiles fill whole waves of resident CTAs and leave a
  // last wave at most half full, that wave's tiles are cut along K into pieces
  // (each >= 16 k-blocks) that run on the SMs the full waves free; a reduction
  // kernel sums the pieces.  At the 70B qkv shape, M = 512 (160 tiles of
  // 128 x 256 on 148 SMs), the second wave otherwise costs as much as the first.
  // Measured on B200 at the 70B shapes, with tiles stored by TMA, every call
  // that qualifies ran as fast or faster split (gate_up at M = 512 447 -> 415 us,
  // qkv and o_proj at M = 2048 312 -> 290 and 250 -> 231 us, qkv at M = 8192
  // 1144 -> 1124 us; qkv at M = 512 137 -> 110 us before the TMA stores).
  if (splits == 1 && tiles > slots) {
    const int64_t rest = tiles % slots;
    if (rest > 0 && 2 * rest <= slots) {
      int64_t pieces = std::min<int64_t>(slots / rest, total_kb / 16);
      while (pieces > 1 && kCounterBytes + (size_t)(rest * pieces) * p.bn * 128 * 4 > ws_cap) --pieces;
      if (pieces >= 2) {
        const int64_t kpp = cdiv(total_kb, pieces);
        pieces = cdiv(total_kb, kpp);
        p.head_tiles = tiles - rest;
        p.tail_pieces = (int)pieces;
        p.kb_per_split = (int)kpp;
        p.ws_bytes = kCounterBytes + (size_t)(rest * pieces) * p.bn * 128 * 4;
      }
    }
  }
  return p;
}

// K3 (small token counts, group 128): one CTA per SM over a balanced partition
// of the (128-row tile, 2-group stage) iterations; workspace = counters, the
// staged activations x' (fp16 [K / 64][BN][64], BN = M rounded up to 16), the
// per-token exponents, and fp32 partials [slots][M][N] for tiles split between CTAs.
constexpr int64_t kSkinnyMaxM = 64;

GemmPlan plan_skinny(int64_t M, int64_t N, int64_t K, int sm) {
  GemmPlan p;
  const int64_t Kg = K / w4::kGroup;
  const int64_t RT = cdiv(N, 128), S = cdiv(Kg, 2), T = RT * S;
  if (M > kSkinnyMaxM || RT > kMaxSplitCounters) return p;  // path 0: not served
  p.path = kPathSkinny;
  const int64_t C = std::min<int64_t>(sm, T);
  const int64_t L = T / C;  // shortest range
  p.grid_x = (int)C;
  p.slots = (int)(S <= 1 ? 1 : std::min<int64_t>(C, (S - 2) / L + 2));
  p.xp_off = kCounterBytes;
  p.xexp_off = p.xp_off + align256((size_t)w4::skinny_bn(M) * K * 2);
  p.part_off = p.xexp_off + 256;
  p.ws_bytes = p.part_off + (size_t)p.slots * M * N * 4;
  return p;
}

// Measured on B200 (8B and 70B layer shapes): the decode kernel wins at M = 1..3
// and on the smaller layers up to M = 8; above that the tensor cores take the
// M-fold product: K3 up to 64 tokens (faster than K2 at every 8B and 70B shape
// at M = 16..64), K2 above.  Crossovers measured for K1 against K3: at M = 5..8,
// K3 on every layer with N*K >= 32 M weights (8B gate_up 31 against 42..46 us,
// 8B down 24 against 26..39 us, every 70B layer); at M = 4 only on the largest
// (70B gate_up 92 against 109 us, 70B down 54 against 82 us).
bool gemv_fits(int64_t M, int64_t N, int64_t K, bool awq) {
  if (M > 8 || !w4::gemv_supports(M, awq)) return false;
  const double nk = (double)N * (double)K;
  const bool skinny_wins = (M >= 5 && nk >= 32.0e6) || (M == 4 && nk >= 200.0e6);
  return !skinny_wins;
}

GemmPlan plan_gemm_raw(int64_t M, int64_t N, int64_t K, bool awq, int sm, size_t ws_cap) {
  int f = forced_path();
  if (f == kPathTc) return plan_tc(M, N, K, awq, sm, ws_cap);
  if (f == kPathSkinny) return plan_skinny(M, N, K, sm);
  if (f == kPathGemv || gemv_fits(M, N, K, awq)) {
    const GemmPlan p = plan_gemv(M, N, K, awq, sm);
    if (p.path == kPathGemv || f == kPathGemv) return p;
  }
  if (M <= kSkinnyMaxM) {
    const GemmPlan p = plan_skinny(M, N, K, sm);
    if (p.path == kPathSkinny && p.ws_bytes <= ws_cap) return p;
  }
  return plan_tc(M, N, K, awq, sm, ws_cap);
}

GemmPlan plan_gemm(int64_t M, int64_t N, int64_t K, bool awq, int sm, size_t ws_cap = SIZE_MAX) {
  return plan_gemm_raw(M, N, K, awq, sm, ws_cap);
}

// W4_DEBUG_PLAN=1 prints the launch plan of every GEMM call to stderr (tests read it).
void debug_plan(const GemmPlan &p, int64_t M, int64_t N, int64_t K) {
  if (getenv("W4_DEBUG_PLAN")) {
    if (p.path == kPathSkinny)
      fprintf(stderr, "[w4] M=%lld N=%lld K=%lld skinny: grid=%d slots=%d ws=%zu\n", (long long)M, (long long)N,
              (long long)K, p.grid_x, p.slots, p.ws_bytes);
    else if (p.path == kPathGemv)
      fprintf(stderr,
              "[w4] M=%lld N=%lld K=%lld decode: t8=%d kr=%d kslices=%d grid_x=%d slots=%d xs=%d scale_tma=%d ws=%zu\n",
              (long long)M, (long long)N, (long long)K, p.t8, p.kr, p.kslices, p.grid_x, p.slots, p.xs_bytes,
              (int)p.sc_tma, p.ws_bytes);
    else
      fprintf(stderr,
              "[w4] M=%lld N=%lld K=%lld tensor-core: bn=%d splits=%d kb_per_split=%d head_tiles=%lld "
              "tail_pieces=%d ws=%zu\n",
              (long long)M, (long long)N, (long long)K, p.bn, p.splits, p.kb_per_split, (long long)p.head_tiles,
              p.tail_pieces, p.ws_bytes);
  }
}

size_t ws_size_all(int64_t M, int64_t N, int64_t K, int sm) {
  size_t ws = std::max(plan_tc(M, N, K, false, sm).ws_bytes, plan_tc(M, N, K, true, sm).ws_bytes);
  if (M <= 64) {
    ws = std::max(ws, plan_gemv(M, N, K, false, sm).ws_bytes);
    if (M <= 32) ws = std::max(ws, plan_gemv(M, N, K, true, sm).ws_bytes);
    ws = std::max(ws, plan_skinny(M, N, K, sm).ws_bytes);
  }
  return ws;
}

w4_status check_shape(int64_t M, int64_t N, int64_t K, int group) {
  if (N < 1 || K < 1 || M < 1) return fail(W4_ERR_INVALID_ARG, "sizes must be >= 1 (M=%lld N=%lld K=%lld)",
                                           (long long)M, (long long)N, (long long)K);
  if (group != 32 && group != 64 && group != 128)
    return fail(W4_ERR_UNSUPPORTED, "group=%d: 32, 64 and 128 are served", group);
  if (K % group != 0) return fail(W4_ERR_INVALID_ARG, "K=%lld is not a multiple of the group (%d)", (long long)K, group);
  const int64_t lim = (int64_t)1 << 40;
  if (N > lim || K > lim || M > lim || (double)N * (double)K > 9.0e18 || (double)M * (double)N > 4.0e18 ||
      (double)M * (double)K > 4.0e18)
    return fail(W4_ERR_INVALID_ARG, "sizes overflow 64-bit indexing");
  if (K / 64 > INT32_MAX || N > INT32_MAX || M > INT32_MAX)
    return fail(W4_ERR_INVALID_ARG, "M, N and K/64 must each fit in 31 bits");
  return W4_OK;
}

}  // namespace

extern "C" {

const char *w4_status_string(w4_status s) {
  switch (s) {
    case W4_OK: return "W4_OK";
    case W4_ERR_INVALID_ARG: return "W4_ERR_INVALID_ARG";
    case W4_ERR_UNSUPPORTED: return "W4_ERR_UNSUPPORTED";
    case W4_ERR_CUDA: return "W4_ERR_CUDA";
  }
  return "W4_ERR_UNKNOWN";
}

const char *w4_last_error(void) { return t_last_error.c_str(); }

}  // extern "C"

namespace {

w4_status quantize_common(const void *W, w4_dtype w_dtype, const float *awq_s, int64_t N, int64_t K, int group,
                          bool symmetric, uint8_t *packed, uint16_t *scales, uint16_t *zeros, uint8_t *codes,
                          w4_stream_t stream) {
  t_last_error.clear();
  w4_status st = check_shape(1, N, K, group);
  if (st != W4_OK) return st;
  if (w_dtype != W4_F32 && w_dtype != W4_F16 && w_dtype != W4_BF16)
    return fail(W4_ERR_UNSUPPORTED, "weight dtype %d not served", (int)w_dtype);
  if (!W || !packed || !scales || !zeros) return fail(W4_ERR_INVALID_ARG, "null W, packed, scales or zeros");
  if (!aligned16(W) || !aligned16(packed) || !aligned16(scales) || !aligned16(zeros) ||
      (awq_s && !aligned16(awq_s)) || (codes && !aligned16(codes)))
    return fail(W4_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  int sm = 0;
  cudaError_t e = current_sm_count(&sm);
  if (e != cudaSuccess) return cuda_fail(e, "device query");
  e = w4::launch_quantize(W, (int)w_dtype, awq_s, N, K, group, symmetric, nullptr, packed, scales, zeros, codes, sm,
                          reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "quantize launch");
  return W4_OK;
}

}  // namespace

extern "C" {

w4_status w4_quantize(const void *W, w4_dtype w_dtype, const float *awq_s, int64_t N, int64_t K, int group,
                      uint8_t *packed, uint16_t *scales, uint16_t *zeros, uint8_t *codes, w4_stream_t stream) {
  return quantize_common(W, w_dtype, awq_s, N, K, group, false, packed, scales, zeros, codes, stream);
}

w4_status w4_quantize_symmetric(const void *W, w4_dtype w_dtype, const float *awq_s, int64_t N, int64_t K,
                                int group, uint8_t *packed, uint16_t *scales, uint16_t *zeros, uint8_t *codes,
                                w4_stream_t stream) {
  return quantize_common(W, w_dtype, awq_s, N, K, group, true, packed, scales, zeros, codes, stream);
}

w4_status w4_pack(const uint8_t *codes, int64_t N, int64_t K, uint8_t *packed, w4_stream_t stream) {
  t_last_error.clear();
  if (N < 1 || K < 1) return fail(W4_ERR_INVALID_ARG, "sizes must be >= 1");
  if (K % 32 != 0) return fail(W4_ERR_INVALID_ARG, "K=%lld must be a multiple of 32", (long long)K);
  if ((double)N * (double)K > 9.0e18) return fail(W4_ERR_INVALID_ARG, "sizes overflow");
  if (!codes || !packed) return fail(W4_ERR_INVALID_ARG, "null codes or packed");
  if (!aligned16(codes) || !aligned16(packed)) return fail(W4_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  int sm = 0;
  cudaError_t e = current_sm_count(&sm);
  if (e != cudaSuccess) return cuda_fail(e, "device query");
  e = w4::launch_pack(codes, N, K, packed, sm, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "pack launch");
  return W4_OK;
}

size_t w4a16_gemm_workspace_size(int64_t M, int64_t N, int64_t K) {
  if (M < 1 || N < 1 || K < 1 || K % w4::kGroup != 0) return 0;
  int sm = 0;
  if (current_sm_count(&sm) != cudaSuccess) sm = 148;
  return ws_size_all(M, N, K, sm);
}

}  // extern "C"

namespace {

// The fused dequantize-matmul; with a CSR (row_ptr, col, val) the sparse part of
// a dense + sparse split is added by a separate kernel right after it.  (Fusing
// it into the decode kernel's output writes measured slower on B200: the chain
// of dependent CSR and activation loads lands on every tile's critical path.)
w4_status gemm_common(const void *X, w4_dtype x_dtype, int64_t M, int64_t N, int64_t K, int group,
                      const uint8_t *packed, const uint16_t *scales, const uint16_t *zeros, const float *awq_s,
                      void *Y, w4_dtype y_dtype, void *workspace, size_t workspace_bytes, w4_stream_t stream,
                      const int32_t *row_ptr, const int32_t *col, const uint16_t *val,
                      size_t plan_ws_cap = SIZE_MAX, const GemmPlan *given_plan = nullptr) {
  t_last_error.clear();
  w4_status st = check_shape(M, N, K, group);
  if (st != W4_OK) return st;
  if (x_dtype != W4_F16 && x_dtype != W4_BF16)
    return fail(W4_ERR_UNSUPPORTED, "activation dtype must be F16 or BF16");
  if (y_dtype != W4_F32 && y_dtype != W4_BF16) return fail(W4_ERR_UNSUPPORTED, "output dtype must be F32 or BF16");
  // Groups of 32 or 64 are served by the tensor-core kernel (64-channel k-blocks).
  if (group != w4::kGroup) {
    if (K % 64 != 0) return fail(W4_ERR_UNSUPPORTED, "group=%d needs K a multiple of 64 (K=%lld)", group, (long long)K);
    if (forced_path() == kPathGemv || forced_path() == kPathSkinny)
      return fail(W4_ERR_UNSUPPORTED, "the decode and skinny kernels serve group 128 only");
  }
  if (!X || !packed || !scales || !zeros || !Y) return fail(W4_ERR_INVALID_ARG, "null X, packed, scales, zeros or Y");
  if (!aligned16(X) || !aligned16(packed) || !aligned16(scales) || !aligned16(zeros) || !aligned16(Y) ||
      (awq_s && !aligned16(awq_s)) || (workspace && !aligned16(workspace)))
    return fail(W4_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  int sm = 0;
  cudaError_t e = current_sm_count(&sm);
  if (e != cudaSuccess) return cuda_fail(e, "device query");
  const bool awq = awq_s != nullptr;
  const GemmPlan plan = given_plan ? *given_plan
                                   : group == w4::kGroup ? plan_gemm(M, N, K, awq, sm, plan_ws_cap)
                                                         : plan_tc(M, N, K, awq, sm, plan_ws_cap);
  debug_plan(plan, M, N, K);
  if (plan.path == 0)
    return fail(W4_ERR_UNSUPPORTED, "the forced kernel (W4_FORCE_PATH) cannot serve M=%lld N=%lld K=%lld",
                (long long)M, (long long)N, (long long)K);
  if (plan.path == kPathGemv && !w4::gemv_supports(M, awq))
    return fail(W4_ERR_UNSUPPORTED, "W4_FORCE_PATH=gemv cannot serve M=%lld%s", (long long)M, awq ? " with AWQ" : "");
  if (plan.ws_bytes > 0 && (!workspace || workspace_bytes < plan.ws_bytes))
    return fail(W4_ERR_INVALID_ARG, "workspace too small: need %zu bytes, got %zu", plan.ws_bytes,
                workspace ? workspace_bytes : (size_t)0);
  uint32_t *counters = static_cast<uint32_t *>(workspace);
  float *partials = workspace ? reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + kCounterBytes) : nullptr;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const bool xbf16 = x_dtype == W4_BF16;

  PFN_cuTensorMapEncodeTiled_v12000 enc = encode_fn();
  if (!enc) return fail(W4_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");

  if (plan.path == kPathGemv) {
    CUtensorMap tmP, tmS, tmZ;
    {
      CUresult r = encode_2d(enc, &tmP, CU_TENSOR_MAP_DATA_TYPE_UINT8, packed, (uint64_t)(K / 2), (uint64_t)N,
                             (uint64_t)(K / 2), 128u, 64u, CU_TENSOR_MAP_SWIZZLE_128B,
                             CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
      if (r != CUDA_SUCCESS) return fail(W4_ERR_CUDA, "tensor map for packed weights failed (CUresult %d)", (int)r);
    }
    tmS = tmP;
    tmZ = tmP;
    if (plan.sc_tma) {
      const uint64_t kg = (uint64_t)(K / w4::kGroup);
      CUresult r = encode_2d(enc, &tmS, CU_TENSOR_MAP_DATA_TYPE_UINT16, scales, kg, (uint64_t)N, kg * 2, 8u, 64u,
                             CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE);
      if (r != CUDA_SUCCESS) return fail(W4_ERR_CUDA, "tensor map for scales failed (CUresult %d)", (int)r);
      r = encode_2d(enc, &tmZ, CU_TENSOR_MAP_DATA_TYPE_UINT16, zeros, kg, (uint64_t)N, kg * 2, 8u, 64u,
                    CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE);
      if (r != CUDA_SUCCESS) return fail(W4_ERR_CUDA, "tensor map for zeros failed (CUresult %d)", (int)r);
    }
    w4::GemvParams p{};
    p.X = X; p.M = M; p.N = N; p.K = K;
    p.scales = scales; p.zeros = zeros; p.awq_s = awq_s;
    p.Y = Y; p.y_bf16 = y_dtype == W4_BF16;
    p.ws = partials; p.counters = counters;
    p.kslices = plan.kslices; p.slots = plan.slots; p.kr = plan.kr; p.grid_x = plan.grid_x; p.xs_bytes = plan.xs_bytes;
    e = w4::launch_gemv(tmP, tmS, tmZ, p, plan.t8, xbf16, plan.sc_tma, s);
    if (e != cudaSuccess) return cuda_fail(e, "decode gemm launch");
    if (row_ptr) {
      e = w4::launch_sparse_add(X, xbf16, M, N, K, row_ptr, col, val, Y, y_dtype == W4_BF16, s);
      if (e != cudaSuccess) return cuda_fail(e, "sparse add");
    }
    return W4_OK;
  }

  if (plan.path == kPathSkinny) {
    uint8_t *wsb = static_cast<uint8_t *>(workspace);
    uint16_t *xp = reinterpret_cast<uint16_t *>(wsb + plan.xp_off);
    int *xexp = reinterpret_cast<int *>(wsb + plan.xexp_off);
    CUtensorMap tmW, tmXp;
    CUresult r = encode_2d(enc, &tmW, CU_TENSOR_MAP_DATA_TYPE_UINT8, packed, (uint64_t)(K / 2), (uint64_t)N,
                           (uint64_t)(K / 2), 128u, 128u, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
    if (r != CUDA_SUCCESS) return fail(W4_ERR_CUDA, "tensor map for packed weights failed (CUresult %d)", (int)r);
    // x' blocked as [K / 64][BN][64]: rows of 64 channels, one stage = 4 BN rows
    const uint32_t bn = (uint32_t)w4::skinny_bn(M);
    r = encode_2d(enc, &tmXp, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, xp, 64u, (uint64_t)(K / 64) * bn, 128u, 64u, 4u * bn,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
    if (r != CUDA_SUCCESS) return fail(W4_ERR_CUDA, "tensor map for staged activations failed (CUresult %d)", (int)r);
    e = w4::launch_stage_x(X, xbf16, awq_s, M, K, xp, xexp, s);
    if (e != cudaSuccess) return cuda_fail(e, "activation staging launch");
    w4::SkinnyParams p{};
    p.M = M; p.N = N; p.K = K;
    p.scales = scales; p.zeros = zeros;
    p.Y = Y; p.y_bf16 = y_dtype == W4_BF16;
    p.xexp = xexp; p.ws = reinterpret_cast<float *>(wsb + plan.part_off); p.counters = counters;
    p.slots = plan.slots;
    e = w4::launch_skinny(tmW, tmXp, p, plan.grid_x, s);
    if (e != cudaSuccess) return cuda_fail(e, "skinny gemm launch");
    if (row_ptr) {
      e = w4::launch_sparse_add(X, xbf16, M, N, K, row_ptr, col, val, Y, y_dtype == W4_BF16, s);
      if (e != cudaSuccess) return cuda_fail(e, "sparse add");
    }
    return W4_OK;
  }

  CUtensorMap tmX, tmP;
  {
    CUresult r = encode_2d(enc, &tmX, xbf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, X,
                           (uint64_t)K, (uint64_t)M, (uint64_t)K * 2, 64u, (uint32_t)plan.bn,
                           CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
    if (r != CUDA_SUCCESS) return fail(W4_ERR_CUDA, "tensor map for X failed (CUresult %d)", (int)r);
  }
  {
    CUresult r = encode_2d(enc, &tmP, CU_TENSOR_MAP_DATA_TYPE_UINT8, packed, (uint64_t)(K / 2), (uint64_t)N,
                           (uint64_t)(K / 2), 32u, 128u, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
    if (r != CUDA_SUCCESS) return fail(W4_ERR_CUDA, "tensor map for packed weights failed (CUresult %d)", (int)r);
  }
  w4::TcParams p{};
  p.M = M; p.N = N; p.K = K;
  p.scales = scales; p.zeros = zeros; p.awq_s = awq_s;
  p.Y = Y; p.y_bf16 = y_dtype == W4_BF16;
  p.ws = partials; p.counters = counters; p.splits = plan.splits; p.kb_per_split = plan.kb_per_split;
  p.group = group;
  p.head_tiles = plan.head_tiles; p.tail_pieces = plan.tail_pieces; p.ntx = (N + 127) / 128;
  // Tile stores by TMA (32 x 32 boxes): Y where its rows are 16-byte multiples,
  // and the tail pieces' partial tiles [tail tiles x pieces x BN][128] fp32.
  // Unused maps are copies of tmX and are never read.
  CUtensorMap tmY = tmX, tmT = tmX;
  const int ysz = y_dtype == W4_BF16 ? 2 : 4;
  if ((N * ysz) % 16 == 0 && M >= 32 && N >= 32) {
    CUresult r = encode_2d(enc, &tmY, ysz == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, Y,
                           (uint64_t)N, (uint64_t)M, (uint64_t)N * ysz, 32u, 32u, CU_TENSOR_MAP_SWIZZLE_NONE,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
    if (r != CUDA_SUCCESS) return fail(W4_ERR_CUDA, "tensor map for Y failed (CUresult %d)", (int)r);
    p.y_tma = 1;
  }
  if (plan.tail_pieces > 0) {
    const uint64_t rows = (uint64_t)(cdiv(N, 128) * cdiv(M, plan.bn) - plan.head_tiles) * plan.tail_pieces * plan.bn;
    CUresult r = encode_2d(enc, &tmT, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, partials, 128u, rows, 512u, 32u, 32u,
                           CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B);
    if (r != CUDA_SUCCESS) return fail(W4_ERR_CUDA, "tensor map for tail partials failed (CUresult %d)", (int)r);
  }
  e = w4::launch_gemm_tc(tmX, tmP, tmY, tmT, p, xbf16, plan.bn, s);
  if (e != cudaSuccess) return cuda_fail(e, "tensor-core gemm launch");
  if (plan.tail_pieces > 0) {
    e = w4::launch_tail_reduce(p, plan.bn, s);
    if (e != cudaSuccess) return cuda_fail(e, "tail reduction launch");
  }
  if (row_ptr) {
    e = w4::launch_sparse_add(X, xbf16, M, N, K, row_ptr, col, val, Y, y_dtype == W4_BF16, s);
    if (e != cudaSuccess) return cuda_fail(e, "sparse add");
  }
  return W4_OK;
}

}  // namespace

extern "C" {

w4_status w4a16_gemm(const void *X, w4_dtype x_dtype, int64_t M, int64_t N, int64_t K, int group,
                     const uint8_t *packed, const uint16_t *scales, const uint16_t *zeros, const float *awq_s,
                     void *Y, w4_dtype y_dtype, void *workspace, size_t workspace_bytes, w4_stream_t stream) {
  return gemm_common(X, x_dtype, M, N, K, group, packed, scales, zeros, awq_s, Y, y_dtype, workspace, workspace_bytes,
                     stream, nullptr, nullptr, nullptr);
}

w4_status w4a16_gemm_host_async(const void *X_host, void *X_dev, w4_dtype x_dtype, int64_t M, int64_t N,
                                int64_t K, int group, const uint8_t *packed, const uint16_t *scales,
                                const uint16_t *zeros, const float *awq_s, void *Y_host, void *Y_dev,
                                w4_dtype y_dtype, void *workspace, size_t workspace_bytes, w4_stream_t stream) {
  t_last_error.clear();
  w4_status st = check_shape(M, N, K, group);
  if (st != W4_OK) return st;
  if (!X_host || !Y_host || !X_dev || !Y_dev) return fail(W4_ERR_INVALID_ARG, "null host or staging buffer");
  if (x_dtype != W4_F16 && x_dtype != W4_BF16)
    return fail(W4_ERR_UNSUPPORTED, "activation dtype must be F16 or BF16");
  if (y_dtype != W4_F32 && y_dtype != W4_BF16) return fail(W4_ERR_UNSUPPORTED, "output dtype must be F32 or BF16");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t xb = (size_t)M * K * 2;
  const size_t yb = (size_t)M * N * (y_dtype == W4_F32 ? 4 : 2);
  cudaError_t e = cudaMemcpyAsync(X_dev, X_host, xb, cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return cuda_fail(e, "copy X to device");
  st = w4a16_gemm(X_dev, x_dtype, M, N, K, group, packed, scales, zeros, awq_s, Y_dev, y_dtype, workspace,
                  workspace_bytes, stream);
  if (st != W4_OK) return st;
  e = cudaMemcpyAsync(Y_host, Y_dev, yb, cudaMemcpyDeviceToHost, s);
  if (e != cudaSuccess) return cuda_fail(e, "copy Y to host");
  return W4_OK;
}

w4_status w4a16_gemm_host(const void *X_host, void *X_dev, w4_dtype x_dtype, int64_t M, int64_t N, int64_t K,
                          int group, const uint8_t *packed, const uint16_t *scales, const uint16_t *zeros,
                          const float *awq_s, void *Y_host, void *Y_dev, w4_dtype y_dtype, void *workspace,
                          size_t workspace_bytes, w4_stream_t stream) {
  w4_status st = w4a16_gemm_host_async(X_host, X_dev, x_dtype, M, N, K, group, packed, scales, zeros, awq_s, Y_host,
                                       Y_dev, y_dtype, workspace, workspace_bytes, stream);
  if (st != W4_OK) return st;
  const cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  return W4_OK;
}

w4_status w4a16_gemm_host_batch_async(const w4_gemm_item *items, int count, const void *X_host, void *X_dev,
                                      size_t x_bytes, void *Y_host, void *Y_dev, size_t y_bytes, void *workspace,
                                      size_t workspace_bytes, w4_stream_t stream) {
  t_last_error.clear();
  if (!items || count < 1 || count > 4096) return fail(W4_ERR_INVALID_ARG, "items: need 1..4096, got %d", count);
  if (!X_host || !Y_host || !X_dev || !Y_dev) return fail(W4_ERR_INVALID_ARG, "null host or staging buffer");
  if (!aligned16(X_dev) || !aligned16(Y_dev)) return fail(W4_ERR_INVALID_ARG, "staging buffers must be 16-byte aligned");
  // Everything an item's matmul would reject is checked here, before the copy of
  // X is enqueued, so a bad item leaves nothing half done on the stream.
  for (int i = 0; i < count; ++i) {
    const w4_gemm_item &it = items[i];
    w4_status st = check_shape(it.M, it.N, it.K, it.group);
    if (st != W4_OK) return fail(st, "item %d: %s", i, t_last_error.c_str());
    if (it.x_dtype != W4_F16 && it.x_dtype != W4_BF16)
      return fail(W4_ERR_UNSUPPORTED, "item %d: activation dtype must be F16 or BF16", i);
    if (it.y_dtype != W4_F32 && it.y_dtype != W4_BF16)
      return fail(W4_ERR_UNSUPPORTED, "item %d: output dtype must be F32 or BF16", i);
    if (!it.packed || !it.scales || !it.zeros) return fail(W4_ERR_INVALID_ARG, "item %d: null weights", i);
    if (!aligned16(it.packed) || !aligned16(it.scales) || !aligned16(it.zeros) || (it.awq_s && !aligned16(it.awq_s)))
      return fail(W4_ERR_INVALID_ARG, "item %d: device pointers must be 16-byte aligned", i);
    if (it.x_offset % 16 != 0 || it.y_offset % 16 != 0)
      return fail(W4_ERR_INVALID_ARG, "item %d: offsets must be multiples of 16 bytes", i);
    const size_t xb = (size_t)it.M * it.K * 2, yb = (size_t)it.M * it.N * (it.y_dtype == W4_F32 ? 4 : 2);
    if (it.x_offset > x_bytes || xb > x_bytes - it.x_offset)
      return fail(W4_ERR_INVALID_ARG, "item %d: X [%zu, %zu) is outside the %zu staged bytes", i, it.x_offset,
                  it.x_offset + xb, x_bytes);
    if (it.y_offset > y_bytes || yb > y_bytes - it.y_offset)
      return fail(W4_ERR_INVALID_ARG, "item %d: Y [%zu, %zu) is outside the %zu staged bytes", i, it.y_offset,
                  it.y_offset + yb, y_bytes);
  }
  int sm = 0;
  cudaError_t e = current_sm_count(&sm);
  if (e != cudaSuccess) return cuda_fail(e, "device query");
  for (int i = 0; i < count; ++i) {
    const w4_gemm_item &it = items[i];
    const GemmPlan plan = it.group == w4::kGroup ? plan_gemm(it.M, it.N, it.K, it.awq_s != nullptr, sm)
                                                 : plan_tc(it.M, it.N, it.K, it.awq_s != nullptr, sm);
    if (it.group != w4::kGroup && (it.K % 64 != 0 || forced_path() == kPathGemv || forced_path() == kPathSkinny))
      return fail(W4_ERR_UNSUPPORTED, "item %d: group=%d needs K a multiple of 64 and the tensor-core kernel", i,
                  it.group);
    if (plan.path == 0 || (plan.path == kPathGemv && !w4::gemv_supports(it.M, it.awq_s != nullptr)))
      return fail(W4_ERR_UNSUPPORTED, "item %d: the forced kernel (W4_FORCE_PATH) cannot serve this shape", i);
    if (plan.ws_bytes > 0 && (!workspace || workspace_bytes < plan.ws_bytes))
      return fail(W4_ERR_INVALID_ARG, "item %d: workspace too small: need %zu bytes, got %zu", i, plan.ws_bytes,
                  workspace ? workspace_bytes : (size_t)0);
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  e = cudaMemcpyAsync(X_dev, X_host, x_bytes, cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return cuda_fail(e, "copy X to device");
  for (int i = 0; i < count; ++i) {
    const w4_gemm_item &it = items[i];
    const w4_status st =
        w4a16_gemm(static_cast<uint8_t *>(X_dev) + it.x_offset, it.x_dtype, it.M, it.N, it.K, it.group, it.packed,
                   it.scales, it.zeros, it.awq_s, static_cast<uint8_t *>(Y_dev) + it.y_offset, it.y_dtype, workspace,
                   workspace_bytes, stream);
    if (st != W4_OK) return fail(st, "item %d: %s", i, t_last_error.c_str());
  }
  e = cudaMemcpyAsync(Y_host, Y_dev, y_bytes, cudaMemcpyDeviceToHost, s);
  if (e != cudaSuccess) return cuda_fail(e, "copy Y to host");
  return W4_OK;
}

w4_status w4_device_error(int *flag) {
  t_last_error.clear();
  if (!flag) return fail(W4_ERR_INVALID_ARG, "null flag");
  int v = 0;
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "device synchronize");
  e = cudaMemcpyFromSymbol(&v, w4::g_error_flag, sizeof v);
  if (e != cudaSuccess) return cuda_fail(e, "read error word");
  const int zero = 0;
  e = cudaMemcpyToSymbol(w4::g_error_flag, &zero, sizeof zero);
  if (e != cudaSuccess) return cuda_fail(e, "clear error word");
  *flag = v;
  return W4_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Decode GEMM with library-owned scratch.
//
// Some callers cannot allocate device memory at the point where they run the
// layer: a C plugin inside an engine that has already handed the whole device
// to its own pools (weights, KV cache) and owns no allocator of its own, or a
// latency-bound decode loop that must not take cudaMalloc/cudaFree, which can
// synchronize the whole device.  w4a16_gemm_decode_static serves them with a
// fixed scratch that lives in this module's own device memory: a file-scope
// array loaded with the module, so no call here allocates anything.
//
// What must start at zero: the split-K counters at the front of the scratch.
// Device globals without an initializer are zero-filled when the module is
// loaded, and every completed call leaves the counters at zero again.  The fp32
// partials behind them need no initial value.  A call whose kernel reported a
// device error (w4_device_error) may leave counters non-zero; the scratch has no
// reset, so the process should stop using this entry point then.
//
// All calls on one device share the one scratch: two calls that overlap in time
// (different streams or threads) race on it and give wrong results.  Calls on
// one stream, one after another, are safe.
//
// The scratch's device address belongs to the CUDA context that loaded the
// module.  It is looked up once per context (cudaGetSymbolAddress, with the
// device current) and cached under the context's unique id, so a context that
// is destroyed and created again (cudaDeviceReset) gets a fresh lookup instead
// of a stale address.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kStaticScratchBytes = (size_t)8 << 20;  // 128 KiB counters + ~7.9 MiB partials

static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

struct StaticScratchEntry {
  unsigned long long ctx_id = 0;
  void *ptr = nullptr;
};
StaticScratchEntry g_static_scratch_at[kMaxDevices];

PFN_cuCtxGetCurrent_v4000 g_ctx_current = nullptr;
PFN_cuCtxGetId_v12000 g_ctx_id = nullptr;
std::once_flag g_ctx_once;

// Unique id of the current context (0 if there is none or the driver lacks the call).
unsigned long long current_ctx_id() {
  std::call_once(g_ctx_once, [] {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_ctx_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(fn);
    fn = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_ctx_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(fn);
  });
  if (!g_ctx_current || !g_ctx_id) return 0;
  CUcontext ctx = nullptr;
  if (g_ctx_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
  unsigned long long id = 0;
  if (g_ctx_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Address of the scratch in the current context of the current device.  The
// first call in a context looks it up (which loads the module there if it is
// not loaded yet); later calls in the same context reuse it.
cudaError_t static_scratch(void **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_mu);
  StaticScratchEntry &ent = g_static_scratch_at[dev];
  const unsigned long long id = current_ctx_id();
  if (!ent.ptr || id == 0 || id != ent.ctx_id) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return e;
    ent.ptr = p;
    ent.ctx_id = current_ctx_id();  // the lookup makes the primary context current
  }
  *out = ent.ptr;
  return cudaSuccess;
}

}  // namespace

extern "C" {

size_t w4a16_gemm_decode_static_capacity(void) { return kStaticScratchBytes; }

w4_status w4a16_gemm_decode_static(const void *X, w4_dtype x_dtype, int64_t M, int64_t N, int64_t K, int group,
                                   const uint8_t *packed, const uint16_t *scales, const uint16_t *zeros,
                                   const float *awq_s, void *Y, w4_dtype y_dtype, w4_stream_t stream) {
  t_last_error.clear();
  w4_status st = check_shape(M, N, K, group);
  if (st != W4_OK) return st;
  const bool awq = awq_s != nullptr;
  if (group != w4::kGroup) return fail(W4_ERR_UNSUPPORTED, "the static-scratch decode GEMM serves group 128 only");
  if (!w4::gemv_supports(M, awq))
    return fail(W4_ERR_UNSUPPORTED, "the static-scratch decode GEMM serves M <= 64, got M=%lld", (long long)M);
  int sm = 0;
  cudaError_t e = current_sm_count(&sm);
  if (e != cudaSuccess) return cuda_fail(e, "device query");
  // The tensor-core plan takes fewer K splits where its partials would not fit.
  // A decode-kernel plan whose k-slice partials do not fit gives way to the
  // tensor-core plan under the same cap (unless the decode kernel is forced).
  GemmPlan plan = plan_gemm(M, N, K, awq, sm, kStaticScratchBytes);
  if (plan.ws_bytes > kStaticScratchBytes && forced_path() != kPathGemv)
    plan = plan_tc(M, N, K, awq, sm, kStaticScratchBytes);
  if (plan.ws_bytes > kStaticScratchBytes)
    return fail(W4_ERR_UNSUPPORTED,
                "M=%lld N=%lld K=%lld needs %zu bytes of scratch; the static scratch holds %zu "
                "(call w4a16_gemm with a caller-owned workspace instead)",
                (long long)M, (long long)N, (long long)K, plan.ws_bytes, kStaticScratchBytes);
  void *scratch = nullptr;
  e = static_scratch(&scratch);
  if (e != cudaSuccess) return cuda_fail(e, "static scratch address");
  return gemm_common(X, x_dtype, M, N, K, group, packed, scales, zeros, awq_s, Y, y_dtype, scratch,
                     kStaticScratchBytes, stream, nullptr, nullptr, nullptr, kStaticScratchBytes, &plan);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// AWQ scale search (offline): see awq_search.cu for the method and include/w4.h
// for the contract.
// ---------------------------------------------------------------------------
namespace {

constexpr int kMaxAlphas = 256;

struct SearchLayout {
  size_t gemm_ws, packed, scales, zeros, s, m, yref, yq, partial, errs, total;
};

SearchLayout search_layout(int64_t Mc, int64_t N, int64_t K, int group, int sm) {
  SearchLayout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align256(off + bytes);
    return at;
  };
  const size_t gws = std::max<size_t>(ws_size_all(Mc, N, K, sm), 256);
  L.gemm_ws = take(gws);
  L.packed = take((size_t)N * K / 2);
  L.scales = take((size_t)N * (K / group) * 2);
  L.zeros = take((size_t)N * (K / group) * 2);
  L.s = take((size_t)K * 4);
  L.m = take((size_t)K * 8);
  L.yref = take((size_t)Mc * N * 4);
  L.yq = take((size_t)Mc * N * 4);
  L.partial = take(256 * 8);
  L.errs = take(kMaxAlphas * 8);
  L.total = off;
  return L;
}

}  // namespace

extern "C" {

size_t w4_awq_search_workspace_size(int64_t Mc, int64_t N, int64_t K, int group) {
  if (Mc < 1 || N < 1 || K < 1 || group < 1 || K % group != 0) return 0;
  int sm = 0;
  if (current_sm_count(&sm) != cudaSuccess) sm = 148;
  return search_layout(Mc, N, K, group, sm).total;
}

w4_status w4_awq_search(const float *W, int64_t N, int64_t K, int group, const void *Xcal, w4_dtype x_dtype,
                        int64_t Mc, const float *alphas, int n_alpha, float *awq_s, double *errors, int *best,
                        void *workspace, size_t workspace_bytes, w4_stream_t stream) {
  t_last_error.clear();
  w4_status st = check_shape(Mc, N, K, group);
  if (st != W4_OK) return st;
  if (x_dtype != W4_F16 && x_dtype != W4_BF16) return fail(W4_ERR_UNSUPPORTED, "calibration dtype must be F16 or BF16");
  if (group != w4::kGroup && K % 64 != 0)
    return fail(W4_ERR_UNSUPPORTED, "group=%d needs K a multiple of 64 (K=%lld)", group, (long long)K);
  if (n_alpha < 1 || n_alpha > kMaxAlphas || !alphas)
    return fail(W4_ERR_INVALID_ARG, "need 1..%d exponents (got %d)", kMaxAlphas, n_alpha);
  for (int i = 0; i < n_alpha; ++i)
    if (!std::isfinite(alphas[i])) return fail(W4_ERR_INVALID_ARG, "exponent %d is not finite", i);
  if (!W || !Xcal || !awq_s || !best || !workspace) return fail(W4_ERR_INVALID_ARG, "null W, Xcal, awq_s, best or workspace");
  if (!aligned16(W) || !aligned16(Xcal) || !aligned16(awq_s) || !aligned16(workspace))
    return fail(W4_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  int sm = 0;
  cudaError_t e = current_sm_count(&sm);
  if (e != cudaSuccess) return cuda_fail(e, "device query");
  const SearchLayout L = search_layout(Mc, N, K, group, sm);
  if (workspace_bytes < L.total)
    return fail(W4_ERR_INVALID_ARG, "workspace too small: need %zu bytes, got %zu", L.total, workspace_bytes);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  uint8_t *packed = ws + L.packed;
  uint16_t *scales = reinterpret_cast<uint16_t *>(ws + L.scales);
  uint16_t *zeros = reinterpret_cast<uint16_t *>(ws + L.zeros);
  float *s = reinterpret_cast<float *>(ws + L.s);
  double *m = reinterpret_cast<double *>(ws + L.m);
  float *yref = reinterpret_cast<float *>(ws + L.yref);
  float *yq = reinterpret_cast<float *>(ws + L.yq);
  double *partial = reinterpret_cast<double *>(ws + L.partial);
  double *errs = reinterpret_cast<double *>(ws + L.errs);
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  const bool xbf16 = x_dtype == W4_BF16;

  if ((e = w4::launch_mean_abs(Xcal, xbf16, Mc, K, m, cs)) != cudaSuccess) return cuda_fail(e, "activation magnitude");
  if ((e = w4::launch_dense_ref(Xcal, xbf16, W, Mc, N, K, yref, cs)) != cudaSuccess) return cuda_fail(e, "reference GEMM");
  for (int i = 0; i < n_alpha; ++i) {
    if ((e = w4::launch_awq_scale(m, K, (double)alphas[i], s, cs)) != cudaSuccess) return cuda_fail(e, "scale");
    st = quantize_common(W, W4_F32, s, N, K, group, false, packed, scales, zeros, nullptr, stream);
    if (st != W4_OK) return st;
    st = w4a16_gemm(Xcal, x_dtype, Mc, N, K, group, packed, scales, zeros, s, yq, W4_F32, ws + L.gemm_ws,
                    L.packed - L.gemm_ws, stream);
    if (st != W4_OK) return st;
    if ((e = w4::launch_sq_err(yref, yq, Mc * N, partial, errs + i, cs)) != cudaSuccess) return cuda_fail(e, "error sum");
  }
  double host_errs[kMaxAlphas];
  if ((e = cudaMemcpyAsync(host_errs, errs, sizeof(double) * n_alpha, cudaMemcpyDeviceToHost, cs)) != cudaSuccess)
    return cuda_fail(e, "copy errors");
  if ((e = cudaStreamSynchronize(cs)) != cudaSuccess) return cuda_fail(e, "stream synchronize");
  int arg = 0;
  for (int i = 1; i < n_alpha; ++i)
    if (host_errs[i] < host_errs[arg]) arg = i;
  if ((e = w4::launch_awq_scale(m, K, (double)alphas[arg], awq_s, cs)) != cudaSuccess) return cuda_fail(e, "scale");
  if (errors)
    for (int i = 0; i < n_alpha; ++i) errors[i] = host_errs[i];
  *best = arg;
  return W4_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Dense + sparse split: see outliers.cu for the method, include/w4.h for the contract.
// ---------------------------------------------------------------------------
extern "C" {

size_t w4_outliers_workspace_size(int64_t N) {
  if (N < 1) return 0;
  return 256 + 2048 * 4 + (size_t)((N * 4 + 255) / 256) * 256;
}

// The top 0.1 % of the weights by magnitude stay in fp16 (mhpq.cn practitioner's
// article, section 2.2): ceil(N * K / 1000), at least 1.
int64_t w4_outliers_default_count(int64_t N, int64_t K) {
  if (N < 1 || K < 1 || (double)N * (double)K > 9.0e18) return 0;
  const int64_t nk = N * K;
  return std::max<int64_t>(1, nk / 1000 + (nk % 1000 != 0));
}

w4_status w4_quantize_outliers(const float *W, const float *awq_s, int64_t N, int64_t K, int group, int64_t count,
                               uint8_t *packed, uint16_t *scales, uint16_t *zeros, int32_t *row_ptr, int32_t *col,
                               uint16_t *val, int64_t capacity, int64_t *nnz, void *workspace,
                               size_t workspace_bytes, w4_stream_t stream) {
  t_last_error.clear();
  w4_status st = check_shape(1, N, K, group);
  if (st != W4_OK) return st;
  if (count == 0) count = w4_outliers_default_count(N, K);
  if (count < 1 || count > N * K) return fail(W4_ERR_INVALID_ARG, "outlier count %lld not in [1, N*K]", (long long)count);
  if (N * K > INT32_MAX) return fail(W4_ERR_UNSUPPORTED, "N*K must fit in 31 bits for the CSR indices");
  if (!W || !packed || !scales || !zeros || !row_ptr || !col || !val || !nnz || !workspace)
    return fail(W4_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned16(W) || !aligned16(packed) || !aligned16(scales) || !aligned16(zeros) || !aligned16(row_ptr) ||
      !aligned16(col) || !aligned16(val) || !aligned16(workspace) || (awq_s && !aligned16(awq_s)))
    return fail(W4_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  if (workspace_bytes < w4_outliers_workspace_size(N))
    return fail(W4_ERR_INVALID_ARG, "workspace too small: need %zu bytes", w4_outliers_workspace_size(N));
  int sm = 0;
  cudaError_t e = current_sm_count(&sm);
  if (e != cudaSuccess) return cuda_fail(e, "device query");
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  uint32_t *state = reinterpret_cast<uint32_t *>(ws);
  uint32_t *hist = reinterpret_cast<uint32_t *>(ws + 256);
  int32_t *counts = reinterpret_cast<int32_t *>(ws + 256 + 2048 * 4);
  if ((e = w4::launch_outlier_threshold(W, N * K, count, state, hist, sm, cs)) != cudaSuccess)
    return cuda_fail(e, "outlier threshold");
  if ((e = w4::launch_quantize(W, 0, awq_s, N, K, group, false, state, packed, scales, zeros, nullptr, sm, cs)) !=
      cudaSuccess)
    return cuda_fail(e, "quantize launch");
  if ((e = w4::launch_outlier_csr(W, N, K, state, counts, row_ptr, capacity, col, val, cs)) != cudaSuccess)
    return cuda_fail(e, "outlier CSR");
  int32_t total = 0;
  if ((e = cudaMemcpyAsync(&total, row_ptr + N, sizeof total, cudaMemcpyDeviceToHost, cs)) != cudaSuccess)
    return cuda_fail(e, "copy entry count");
  if ((e = cudaStreamSynchronize(cs)) != cudaSuccess) return cuda_fail(e, "stream synchronize");
  *nnz = total;
  if (total > capacity)
    return fail(W4_ERR_INVALID_ARG, "outlier capacity %lld below the %d entries found (ties at the threshold)",
                (long long)capacity, total);
  return W4_OK;
}

w4_status w4a16_gemm_outliers(const void *X, w4_dtype x_dtype, int64_t M, int64_t N, int64_t K, int group,
                              const uint8_t *packed, const uint16_t *scales, const uint16_t *zeros,
                              const float *awq_s, const int32_t *row_ptr, const int32_t *col, const uint16_t *val,
                              void *Y, w4_dtype y_dtype, void *workspace, size_t workspace_bytes,
                              w4_stream_t stream) {
  if (!row_ptr || !col || !val) {
    t_last_error.clear();
    return fail(W4_ERR_INVALID_ARG, "null CSR pointer");
  }
  return gemm_common(X, x_dtype, M, N, K, group, packed, scales, zeros, awq_s, Y, y_dtype, workspace, workspace_bytes,
                     stream, row_ptr, col, val);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// GPTQ: see gptq.cu for the method, include/w4.h for the contract.
// ---------------------------------------------------------------------------
namespace {

struct GptqLayout {
  size_t h, lc, li, wd, codes, bad, total;
};

GptqLayout gptq_layout(int64_t N, int64_t K) {
  GptqLayout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align256(off + bytes);
    return at;
  };
  L.h = take((size_t)K * K * 8);
  L.lc = take((size_t)K * K * 8);
  L.li = take((size_t)K * K * 8);
  L.wd = take((size_t)N * K * 8);
  L.codes = take((size_t)N * K);
  L.bad = take(256);
  L.total = off;
  return L;
}

}  // namespace

extern "C" {

size_t w4_gptq_workspace_size(int64_t N, int64_t K) {
  if (N < 1 || K < 1) return 0;
  return gptq_layout(N, K).total;
}

w4_status w4_quantize_gptq(const float *W, int64_t N, int64_t K, int group, const void *Xcal, w4_dtype x_dtype,
                           int64_t Mc, double damp_frac, uint8_t *packed, uint16_t *scales, uint16_t *zeros,
                           uint8_t *codes, void *workspace, size_t workspace_bytes, w4_stream_t stream) {
  t_last_error.clear();
  w4_status st = check_shape(Mc, N, K, group);
  if (st != W4_OK) return st;
  if (x_dtype != W4_F16 && x_dtype != W4_BF16) return fail(W4_ERR_UNSUPPORTED, "calibration dtype must be F16 or BF16");
  if (K % 32 != 0) return fail(W4_ERR_INVALID_ARG, "K=%lld must be a multiple of 32", (long long)K);
  if (K > 32768) return fail(W4_ERR_UNSUPPORTED, "K=%lld: the K x K Hessian factors are limited to K <= 32768",
                             (long long)K);
  if (!(damp_frac >= 0.0) || !std::isfinite(damp_frac)) return fail(W4_ERR_INVALID_ARG, "damp_frac must be >= 0");
  if (!W || !Xcal || !packed || !scales || !zeros || !workspace) return fail(W4_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned16(W) || !aligned16(Xcal) || !aligned16(packed) || !aligned16(scales) || !aligned16(zeros) ||
      !aligned16(workspace) || (codes && !aligned16(codes)))
    return fail(W4_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  const GptqLayout L = gptq_layout(N, K);
  if (workspace_bytes < L.total)
    return fail(W4_ERR_INVALID_ARG, "workspace too small: need %zu bytes, got %zu", L.total, workspace_bytes);
  int sm = 0;
  cudaError_t e = current_sm_count(&sm);
  if (e != cudaSuccess) return cuda_fail(e, "device query");
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  double *H = reinterpret_cast<double *>(ws + L.h);
  double *Lc = reinterpret_cast<double *>(ws + L.lc);
  double *Li = reinterpret_cast<double *>(ws + L.li);
  double *Wd = reinterpret_cast<double *>(ws + L.wd);
  uint8_t *cbuf = codes ? codes : ws + L.codes;
  int *bad = reinterpret_cast<int *>(ws + L.bad);
  if ((e = cudaMemsetAsync(bad, 0, sizeof(int), cs)) != cudaSuccess) return cuda_fail(e, "clear flag");
  if ((e = w4::launch_gptq_hinv(Xcal, x_dtype == W4_BF16, Mc, K, damp_frac, H, Lc, Li, bad, cs)) != cudaSuccess)
    return cuda_fail(e, "Hessian factors");
  if ((e = w4::launch_gptq_sweep(W, N, K, group, Li, Wd, cbuf, scales, zeros, cs)) != cudaSuccess)
    return cuda_fail(e, "column sweep");
  if ((e = w4::launch_pack(cbuf, N, K, packed, sm, cs)) != cudaSuccess) return cuda_fail(e, "pack");
  int host_bad = 0;
  if ((e = cudaMemcpyAsync(&host_bad, bad, sizeof host_bad, cudaMemcpyDeviceToHost, cs)) != cudaSuccess)
    return cuda_fail(e, "read flag");
  if ((e = cudaStreamSynchronize(cs)) != cudaSuccess) return cuda_fail(e, "stream synchronize");
  if (host_bad) return fail(W4_ERR_INVALID_ARG, "the damped Hessian 2 X^T X is not positive definite");
  return W4_OK;
}

}  // extern "C"
