// C ABI of the block-scaled FP8 GEMM library: argument checks, plan choice,
// TMA descriptor encoding, split-K workspace, launches and device status.
// The operation and every argument convention are documented in bsgemm.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <iterator>
#include <map>
#include <mutex>
#include <utility>

#include "bsgemm.h"
#include "bsgemm_host.h"
#include "bsgemm_kernel.cuh"

using bsg::Params;
using bsg_host::DeviceInfo;
using bsg_host::Workspace;

namespace {
__device__ int g_device_status;  // BSGEMM_OK or a timeout code (low byte) | where << 8
}  // namespace

namespace bsg_host {
namespace {

// ------------------------------------------------------------------ driver entry point
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

}  // namespace

namespace {
bool encode_2d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint64_t inner, uint64_t outer,
               uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}
}  // namespace

// 2D tensor map with 128-byte swizzle. `inner` is the contiguous extent.
bool make_map_2d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint64_t inner,
                 uint64_t outer, uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer) {
  return encode_2d(m, base, dt, inner, outer, row_stride_bytes, box_inner, box_outer, CU_TENSOR_MAP_SWIZZLE_128B);
}

bool make_out_map(CUtensorMap* m, void* out, int M, int N, bool f32) {
  if (f32)
    return make_map_2d(m, out, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, N, M, static_cast<uint64_t>(N) * 4, 32, 32);
  return make_map_2d(m, out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, N, M, static_cast<uint64_t>(N) * 2, 64, 32);
}

bool make_swap_out_map(CUtensorMap* m, void* out, int M, int N, int bnq) {
  return encode_2d(m, out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, N, M, static_cast<uint64_t>(N) * 2, bsg::BM,
                   static_cast<uint32_t>(bnq), CU_TENSOR_MAP_SWIZZLE_NONE);
}

// ------------------------------------------------------------------ per-device state
std::mutex g_mu;
std::map<int, DeviceInfo> g_dev;
// Split-K workspaces, keyed by (device, the stream's process-unique id from
// cudaStreamGetId).  Ids are never reused, so a stream created later with the
// same handle value gets a workspace of its own.  cudaStreamGetId is not
// called on a stream that is being captured (that would invalidate the
// capture); there the id comes from g_ids, the last id an uncaptured call saw
// for the (device, handle).
std::map<std::pair<int, unsigned long long>, Workspace> g_ws;
std::map<std::pair<int, uintptr_t>, unsigned long long> g_ids;

bsgemm_status device_info(DeviceInfo& out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BSGEMM_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  auto it = g_dev.find(dev);
  if (it == g_dev.end()) {
    DeviceInfo d;
    d.ordinal = dev;
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return BSGEMM_ERR_CUDA;
    d.ok = (major == 10 && minor == 0);
    if (d.ok) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return BSGEMM_ERR_CUDA;
      d.status = static_cast<int*>(p);
    }
    it = g_dev.emplace(dev, d).first;
  }
  out = it->second;
  return out.ok ? BSGEMM_OK : BSGEMM_ERR_UNSUPPORTED_DEVICE;
}

// Workspace of at least `ws_bytes` and `n_counters` zeroed counters for
// (current device, stream).  Growing is stream-ordered on the call's own
// stream: the old buffers are released with cudaFreeAsync after the stream's
// earlier launches and the new ones come from cudaMallocAsync, so a growing
// call never waits for the device or for other streams.  New counters are
// zeroed on the same stream.  A call being captured into a CUDA graph can
// only use the workspace an uncaptured call on the same stream already made
// big enough (the graph would otherwise own the new memory); otherwise it
// fails with BSGEMM_ERR_CUDA before anything is captured.
bsgemm_status get_workspace(cudaStream_t stream, size_t ws_bytes, size_t n_counters, Workspace& out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BSGEMM_ERR_CUDA;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) return BSGEMM_ERR_CUDA;
  const bool capturing = cs != cudaStreamCaptureStatusNone;
  unsigned long long sid = 0;
  if (!capturing && cudaStreamGetId(stream, &sid) != cudaSuccess) return BSGEMM_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  const std::pair<int, uintptr_t> hkey{dev, reinterpret_cast<uintptr_t>(stream)};
  if (capturing) {
    auto id = g_ids.find(hkey);
    if (id == g_ids.end()) return BSGEMM_ERR_CUDA;  // the stream has no workspace yet
    sid = id->second;
  } else {
    g_ids[hkey] = sid;
  }
  Workspace& w = g_ws[{dev, sid}];
  if (w.ws_bytes < ws_bytes || w.n_counters < n_counters) {
    if (capturing) return BSGEMM_ERR_CUDA;
  }
  if (w.ws_bytes < ws_bytes) {
    if (w.ws && cudaFreeAsync(w.ws, stream) != cudaSuccess) return BSGEMM_ERR_CUDA;
    w.ws = nullptr;
    w.ws_bytes = 0;
    size_t want = ws_bytes + ws_bytes / 4;
    void* p = nullptr;
    if (cudaMallocAsync(&p, want, stream) != cudaSuccess) return BSGEMM_ERR_CUDA;
    w.ws = static_cast<float*>(p);
    w.ws_bytes = want;
  }
  if (w.n_counters < n_counters) {
    if (w.counters && cudaFreeAsync(w.counters, stream) != cudaSuccess) return BSGEMM_ERR_CUDA;
    w.counters = nullptr;
    w.n_counters = 0;
    size_t want = n_counters < 1024 ? 1024 : n_counters * 2;
    void* p = nullptr;
    if (cudaMallocAsync(&p, want * sizeof(int), stream) != cudaSuccess) return BSGEMM_ERR_CUDA;
    w.counters = static_cast<int*>(p);
    if (cudaMemsetAsync(w.counters, 0, want * sizeof(int), stream) != cudaSuccess) return BSGEMM_ERR_CUDA;
    w.n_counters = want;
  }
  out = w;
  return BSGEMM_OK;
}

unsigned long long wait_timeout_ns() {
  static unsigned long long t = [] {
    const char* e = std::getenv("BSGEMM_WAIT_TIMEOUT_NS");
    unsigned long long v = e ? std::strtoull(e, nullptr, 10) : 0ull;
    return v ? v : 1000000000ull;  // 1 s
  }();
  return t;
}

bsgemm_status device_status_address(int** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess || p == nullptr) return BSGEMM_ERR_CUDA;
  *out = static_cast<int*>(p);
  return BSGEMM_OK;
}

}  // namespace bsg_host

namespace {
using bsg_host::device_info;

// ------------------------------------------------------------------ checks
bool aligned(const void* p, uintptr_t n) { return (reinterpret_cast<uintptr_t>(p) % n) == 0; }

bsgemm_status check_args(int layout, const void* a, const void* b, const float* sa, const float* sb,
                         const void* out, int64_t M, int64_t N, int64_t K, int gran) {
  if (layout < BSGEMM_LAYOUT_NT || layout > BSGEMM_LAYOUT_TT) return BSGEMM_ERR_INVALID_ARG;
  if (!a || !b || !sa || !sb || !out) return BSGEMM_ERR_INVALID_ARG;
  if (M <= 0 || N <= 0 || K <= 0) return BSGEMM_ERR_INVALID_ARG;
  // TMA coordinates and the kernel's index math are 32-bit
  if (M > (1 << 30) || N > (1 << 30) || K > (1 << 30)) return BSGEMM_ERR_INVALID_ARG;
  if (gran != 64 && gran != 128 && gran != 256) return BSGEMM_ERR_UNSUPPORTED_GRAN;
  if (!aligned(a, 16) || !aligned(b, 16) || !aligned(out, 16) || !aligned(sa, 4) || !aligned(sb, 4))
    return BSGEMM_ERR_MISALIGNED;
  const bool a_mn = (layout == BSGEMM_LAYOUT_TN || layout == BSGEMM_LAYOUT_TT);
  const bool b_mn = (layout == BSGEMM_LAYOUT_TN || layout == BSGEMM_LAYOUT_NN);
  if (a_mn ? (M % 16) : (K % 16)) return BSGEMM_ERR_MISALIGNED;
  if (b_mn ? (N % 16) : (K % 16)) return BSGEMM_ERR_MISALIGNED;
  if (N % 8) return BSGEMM_ERR_MISALIGNED;
  return BSGEMM_OK;
}

int pow2_at_least(int x, int lo) {
  int v = lo;
  while (v < x) v *= 2;
  return v;
}

}  // namespace

// ------------------------------------------------------------------ plan
extern "C" bsgemm_status bsgemm_make_plan(int layout, int64_t M, int64_t N, int64_t K, int gran,
                                          int num_sms, const bsgemm_tuning* t, bsgemm_plan* plan) {
  if (!plan || num_sms <= 0) return BSGEMM_ERR_INVALID_ARG;
  if (layout < BSGEMM_LAYOUT_NT || layout > BSGEMM_LAYOUT_TT) return BSGEMM_ERR_INVALID_ARG;
  if (M <= 0 || N <= 0 || K <= 0) return BSGEMM_ERR_INVALID_ARG;
  if (M > (1 << 30) || N > (1 << 30) || K > (1 << 30)) return BSGEMM_ERR_INVALID_ARG;
  if (gran != 64 && gran != 128 && gran != 256) return BSGEMM_ERR_UNSUPPORTED_GRAN;
  bsgemm_plan pl{};
  const int Kb = static_cast<int>((K + gran - 1) / gran);
  int variant = t ? t->variant : BSGEMM_VARIANT_AUTO;
  if (variant == BSGEMM_VARIANT_AUTO) {
    // Swap-AB up to M = 64 (its 16..64-wide tiles fit the rows); from M = 65
    // the data-parallel 128-wide tile is 3-5 % faster than swap-AB's 128-wide
    // one (same box, M = 72..128 with N = 2048..7168).
    variant = (M <= 64) ? BSGEMM_VARIANT_SWAP_AB : BSGEMM_VARIANT_DATA_PARALLEL;
    // CTA pairs halve each SM's operand traffic and deepen its pipeline
    // (six stages instead of four).  Measured on B200 (same box, back to
    // back) that pays, given at least a full wave of 256 x 256 tiles, where
    // the promotion hand-off is rare (g = 256: one per two stages;
    // 2048 x 4096 x 32768: 224 against 255 us) or where a tile streams a long
    // K (g = 128, K = 32768: 265 against 288 us).  On short K at g = 128 the
    // two are within run-to-run noise of each other (4096^3: 71.6-74.9
    // against 71.9-72.1 us; 6144^2 x 4096: 158 against 145 us), and single
    // CTAs keep stream-K for ragged waves; at g = 64 pairs lose.
    const bool tuned = t && (t->bnq != 0 || t->splits != 0 || t->stream_k != 0);
    const int64_t pair_tiles = ((M + 255) / 256) * ((N + 255) / 256);
    const bool pair_pays = gran == 256 || (gran == 128 && K >= 16384);
    if (!tuned && pair_pays && M > 128 && num_sms >= 2 && pair_tiles >= num_sms / 2)
      variant = BSGEMM_VARIANT_CTA_PAIR;
  }
  if (variant == BSGEMM_VARIANT_CTA_PAIR) {
    // 256 x 256 tiles on CTA pairs, whole tiles walked by persistent pairs
    if ((t && t->bnq != 0 && t->bnq != 256) || (t && t->splits > 1) || (t && t->stream_k > 0))
      return BSGEMM_ERR_INVALID_ARG;
    if (num_sms < 2) return BSGEMM_ERR_INVALID_ARG;
    pl.cta_pair = 1;
    pl.bnq = 256;
    pl.tiles_p = static_cast<int>((M + 255) / 256);
    pl.tiles_q = static_cast<int>((N + 255) / 256);
    const int64_t pair_tiles = static_cast<int64_t>(pl.tiles_p) * pl.tiles_q;
    if (pair_tiles > (1 << 30)) return BSGEMM_ERR_INVALID_ARG;
    const int64_t pairs = pair_tiles < num_sms / 2 ? pair_tiles : num_sms / 2;
    pl.grid = static_cast<int>(2 * pairs);
    pl.splits = 1;
    pl.kb_per_split = Kb;
    pl.sk_units_per_tile = (Kb + (gran == 64 ? 1 : 0)) / (gran == 64 ? 2 : 1);
    pl.group_p = 8;
    pl.layout = layout;
    pl.gran = gran;
    pl.kernels = 1;
    *plan = pl;
    return BSGEMM_OK;
  }
  if (variant != BSGEMM_VARIANT_SWAP_AB && variant != BSGEMM_VARIANT_DATA_PARALLEL) return BSGEMM_ERR_INVALID_ARG;
  pl.swap_ab = (variant == BSGEMM_VARIANT_SWAP_AB);
  const int64_t P = pl.swap_ab ? N : M;
  const int64_t Q = pl.swap_ab ? M : N;
  int bnq = t ? t->bnq : 0;
  if (bnq == 0 && pl.swap_ab) bnq = pow2_at_least(static_cast<int>(Q < 128 ? Q : 128), 16);
  if (bnq == 0) {
    // Data-parallel width: 256, except
    // - where 256-wide tiles are fewer than the SMs and 128-wide ones still
    //   fit in one wave: the narrower tiles halve each stream-K piece and the
    //   fix-up, measured 10-25 % faster (M = 128..256, N = 4096..7168; with
    //   more 128-wide tiles than SMs 256 stayed ahead: M = 320..512);
    // - with whole tiles (short K, no stream-K) where 128-wide tiles waste
    //   less of the last wave: a 128-wide tile takes 0.62 of a 256-wide one
    //   (the square workload: 7 waves of 128 against 4 of 256), and 2 waves
    //   of 256 against 3 of 128 measured 2.5-9 % faster at 128 (seven shapes,
    //   M = 384..2048).  Measured at g = 128 only, so applied there.
    const int64_t tp = (P + bsg::BM - 1) / bsg::BM;
    const int64_t t256 = tp * ((Q + 255) / 256), t128 = tp * ((Q + 127) / 128);
    const int64_t w256 = (t256 + num_sms - 1) / num_sms, w128 = (t128 + num_sms - 1) / num_sms;
    const bool whole = gran == 128 && static_cast<int64_t>(Kb) * gran < 64 * 128;   // no stream-K at 256
    if (Q <= 128 || (t256 < num_sms && t128 <= num_sms)) bnq = 128;
    else if (t256 >= num_sms && whole && 0.62 * static_cast<double>(w128) < 0.97 * static_cast<double>(w256)) bnq = 128;
    else bnq = 256;
  }
  if (pl.swap_ab ? (bnq != 16 && bnq != 32 && bnq != 64 && bnq != 128) : (bnq != 128 && bnq != 256))
    return BSGEMM_ERR_INVALID_ARG;
  pl.bnq = bnq;
  pl.tiles_p = static_cast<int>((P + bsg::BM - 1) / bsg::BM);
  pl.tiles_q = static_cast<int>((Q + bnq - 1) / bnq);
  const int64_t tiles = static_cast<int64_t>(pl.tiles_p) * pl.tiles_q;
  if (tiles > (1 << 30)) return BSGEMM_ERR_INVALID_ARG;
  // K is handed out in units of one 128-deep stage (two K-blocks when g = 64)
  const int unit_kb = (gran == 64) ? 2 : 1;
  const int U = (Kb + unit_kb - 1) / unit_kb;
  auto split_fix = [&](int s, int& per) {
    per = (Kb + s - 1) / s;
    if (gran == 64 && (per & 1)) ++per;  // a split starts on a 128-element stage
    return (Kb + per - 1) / per;
  };
  const int splits_req = t ? t->splits : 0;
  const int sk_req = t ? t->stream_k : 0;
  int splits = 1;
  pl.sk_first_tile = 0;
  pl.sk_units_per_tile = U;
  pl.sk_ctas = 0;
  pl.sk_units = 0;
  if (splits_req > 0) {
    splits = splits_req;
  } else {
    // Stream-K when whole tiles would leave a ragged last wave: the full
    // waves stay whole tiles and the remaining tiles' units are shared out
    // evenly. Compared on the busiest CTA's units, with a partial tile written
    // and re-read counted as (1 + width/128) units.  Measured on B200, the
    // ranges pay off with fewer tiles than SMs (the decode shapes: 5-11 %
    // over split-K at every tile width) and, with more, only when a tile has
    // many units (K >= 64 K-blocks of 128); on short-K problems whole tiles
    // win.  stream_k = 1 forces it wherever a wave is ragged.
    const int64_t full = (tiles / num_sms) * num_sms;
    const int64_t rem = tiles - full;
    const bool sk_pays = tiles < num_sms ? true : U * unit_kb * gran >= 64 * 128;
    bool use_sk = false;
    if (rem > 0 && sk_req >= 0 && (sk_req > 0 || sk_pays)) {
      const int64_t R = rem * U;
      int64_t gp = R / 4;  // at least ~4 units per CTA
      if (gp > num_sms) gp = num_sms;
      if (gp < 1) gp = 1;
      const double piece_cost = 1.0 + bnq / 128.0;
      const double cost_dp = static_cast<double>((tiles + num_sms - 1) / num_sms) * U;
      const double cost_sk = static_cast<double>(full / num_sms) * U +
                             static_cast<double>((R + gp - 1) / gp) + 2.0 * piece_cost;
      if (R < (int64_t(1) << 31) && (sk_req > 0 || cost_sk < cost_dp)) {
        use_sk = true;
        pl.sk_first_tile = static_cast<int>(full);
        pl.sk_ctas = static_cast<int>(gp);
        pl.sk_units = static_cast<int>(R);
      }
    }
    if (!use_sk && tiles < num_sms) {
      // no stream-K: split-K fills the SMs; among the split counts take the
      // least estimated time, waves(tiles * splits) * (K-blocks per split + overhead)
      const double overhead = 1.0 + bnq / 64.0;
      double best = 1e30;
      for (int s = 1; s <= Kb && s <= 64; ++s) {
        int per = 0;
        const int se = split_fix(s, per);
        const int64_t waves = (tiles * se + num_sms - 1) / num_sms;
        const double cost = static_cast<double>(waves) * (per + (se > 1 ? overhead : 0.0));
        if (cost < best - 1e-9) { best = cost; splits = se; }
      }
    }
  }
  if (splits > Kb) splits = Kb;
  int per = 0;
  pl.splits = split_fix(splits, per);
  pl.kb_per_split = per;
  const int64_t whole = pl.sk_ctas > 0 ? pl.sk_first_tile : tiles;
  int64_t work = whole * pl.splits;
  if (work > (1 << 30)) return BSGEMM_ERR_INVALID_ARG;  // work items are counted in 32 bits
  if (work < pl.sk_ctas) work = pl.sk_ctas;
  pl.grid = static_cast<int>(work < num_sms ? work : num_sms);
  // Raster: the persistent CTAs walk group_p row (P) tiles down, then across
  // the Q tiles.  DRAM reads are about P-operand + Q-operand x (tiles_p /
  // group_p): each Q panel is read once per group.  When the whole P operand
  // fits comfortably in L2 (<= 48 MB of the 126 MB), one group spans all the
  // row tiles, P stays resident and every Q panel is read once (FFN
  // 8192 x 14336 x 4096: 265 MB of DRAM reads with groups of 16).
  pl.group_p = (P * K <= (int64_t(48) << 20)) ? pl.tiles_p : 16;
  pl.layout = layout;
  pl.gran = gran;
  pl.kernels = 1;
  *plan = pl;
  return BSGEMM_OK;
}

// ------------------------------------------------------------------ entry points
extern "C" bsgemm_status bsgemm_fp8_gemm_fused(int layout, int a_format, int b_format, const void* a,
                                               const void* b, const float* scale_a, const float* scale_b,
                                               const bsgemm_epilogue* epi, void* out, int64_t M, int64_t N,
                                               int64_t K, int gran, const bsgemm_tuning* tuning,
                                               bsgemm_stream_t stream) {
  if ((a_format != BSGEMM_FP8_E4M3 && a_format != BSGEMM_FP8_E5M2) ||
      (b_format != BSGEMM_FP8_E4M3 && b_format != BSGEMM_FP8_E5M2))
    return BSGEMM_ERR_INVALID_ARG;
  bsg_host::CallOpts opts;
  opts.a_fmt = a_format;
  opts.b_fmt = b_format;
  if (epi) {
    if (epi->activation < BSGEMM_ACT_NONE || epi->activation > BSGEMM_ACT_GELU) return BSGEMM_ERR_INVALID_ARG;
    if (epi->out_dtype != BSGEMM_OUT_BF16 && epi->out_dtype != BSGEMM_OUT_F32) return BSGEMM_ERR_INVALID_ARG;
    if (epi->bias && (reinterpret_cast<uintptr_t>(epi->bias) & 3) != 0) return BSGEMM_ERR_MISALIGNED;
    opts.bias = epi->bias;
    opts.epi = epi->activation | (epi->out_dtype == BSGEMM_OUT_F32 ? bsg::kEpiOutF32 : 0);
  }
  bsgemm_status st = check_args(layout, a, b, scale_a, scale_b, out, M, N, K, gran);
  if (st != BSGEMM_OK) return st;
  DeviceInfo dev;
  st = device_info(dev);
  if (st != BSGEMM_OK) return st;
  bsgemm_plan pl;
  st = bsgemm_make_plan(layout, M, N, K, gran, dev.num_sms, tuning, &pl);
  if (st != BSGEMM_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int m = static_cast<int>(M), n = static_cast<int>(N), k = static_cast<int>(K);
#define BSG_RUN(G, L) bsg_host::run_g##G##_##L(pl, a, b, scale_a, scale_b, out, m, n, k, opts, s, dev)
#define BSG_RUN_LAYOUTS(G)                              \
  switch (layout) {                                     \
    case BSGEMM_LAYOUT_NT: return BSG_RUN(G, nt);       \
    case BSGEMM_LAYOUT_TN: return BSG_RUN(G, tn);       \
    case BSGEMM_LAYOUT_NN: return BSG_RUN(G, nn);       \
    default:               return BSG_RUN(G, tt);       \
  }
  switch (gran) {
    case 64:  BSG_RUN_LAYOUTS(64)
    case 128: BSG_RUN_LAYOUTS(128)
    default:  BSG_RUN_LAYOUTS(256)
  }
#undef BSG_RUN_LAYOUTS
#undef BSG_RUN
}

extern "C" bsgemm_status bsgemm_fp8_grouped_nt(int a_format, int b_format, const void* a, const void* b,
                                               const float* scale_a, const float* scale_b, void* out,
                                               const int32_t* group_m, int num_groups, int64_t max_rows,
                                               int64_t N, int64_t K, int gran, bsgemm_stream_t stream) {
  if ((a_format != BSGEMM_FP8_E4M3 && a_format != BSGEMM_FP8_E5M2) ||
      (b_format != BSGEMM_FP8_E4M3 && b_format != BSGEMM_FP8_E5M2))
    return BSGEMM_ERR_INVALID_ARG;
  if (!group_m || num_groups < 1 || max_rows < 1) return BSGEMM_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(group_m) & 3) != 0) return BSGEMM_ERR_MISALIGNED;
  bsgemm_status st = check_args(BSGEMM_LAYOUT_NT, a, b, scale_a, scale_b, out, max_rows, N, K, gran);
  if (st != BSGEMM_OK) return st;
  if (static_cast<int64_t>(num_groups) * N > (1 << 30)) return BSGEMM_ERR_INVALID_ARG;
  DeviceInfo dev;
  st = device_info(dev);
  if (st != BSGEMM_OK) return st;
  bsgemm_plan pl{};
  pl.layout = BSGEMM_LAYOUT_NT;
  pl.gran = gran;
  pl.grouped = 1;
  pl.bnq = N <= 128 ? 128 : 256;
  pl.tiles_q = static_cast<int>((N + pl.bnq - 1) / pl.bnq);
  pl.splits = 1;
  pl.kb_per_split = static_cast<int>((K + gran - 1) / gran);
  pl.grid = dev.num_sms;
  pl.group_p = 1;
  pl.kernels = 1;
  bsg_host::CallOpts opts;
  opts.a_fmt = a_format;
  opts.b_fmt = b_format;
  opts.group_m = group_m;
  opts.num_groups = num_groups;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int m = static_cast<int>(max_rows), n = static_cast<int>(N), k = static_cast<int>(K);
  switch (gran) {
    case 64:  return bsg_host::run_g64_nt(pl, a, b, scale_a, scale_b, out, m, n, k, opts, s, dev);
    case 128: return bsg_host::run_g128_nt(pl, a, b, scale_a, scale_b, out, m, n, k, opts, s, dev);
    default:  return bsg_host::run_g256_nt(pl, a, b, scale_a, scale_b, out, m, n, k, opts, s, dev);
  }
}

extern "C" bsgemm_status bsgemm_fp8_gemm_fmt(int layout, int a_format, int b_format, const void* a,
                                             const void* b, const float* scale_a, const float* scale_b,
                                             void* out, int64_t M, int64_t N, int64_t K, int gran,
                                             const bsgemm_tuning* tuning, bsgemm_stream_t stream) {
  return bsgemm_fp8_gemm_fused(layout, a_format, b_format, a, b, scale_a, scale_b, nullptr, out, M, N,
                               K, gran, tuning, stream);
}

extern "C" bsgemm_status bsgemm_fp8_gemm_ex(int layout, const void* a, const void* b,
                                            const float* scale_a, const float* scale_b, void* out,
                                            int64_t M, int64_t N, int64_t K, int gran,
                                            const bsgemm_tuning* tuning, bsgemm_stream_t stream) {
  return bsgemm_fp8_gemm_fmt(layout, BSGEMM_FP8_E4M3, BSGEMM_FP8_E4M3, a, b, scale_a, scale_b, out,
                             M, N, K, gran, tuning, stream);
}

extern "C" bsgemm_status bsgemm_fp8_nt(const void* a, const void* b, const float* sa, const float* sb,
                                       void* out, int64_t M, int64_t N, int64_t K, int gran,
                                       bsgemm_stream_t stream) {
  return bsgemm_fp8_gemm_ex(BSGEMM_LAYOUT_NT, a, b, sa, sb, out, M, N, K, gran, nullptr, stream);
}

extern "C" bsgemm_status bsgemm_fp8_tn(const void* a, const void* b, const float* sa, const float* sb,
                                       void* out, int64_t M, int64_t N, int64_t K, int gran,
                                       bsgemm_stream_t stream) {
  return bsgemm_fp8_gemm_ex(BSGEMM_LAYOUT_TN, a, b, sa, sb, out, M, N, K, gran, nullptr, stream);
}

extern "C" bsgemm_status bsgemm_fp8_nn(const void* a, const void* b, const float* sa, const float* sb,
                                       void* out, int64_t M, int64_t N, int64_t K, int gran,
                                       bsgemm_stream_t stream) {
  return bsgemm_fp8_gemm_ex(BSGEMM_LAYOUT_NN, a, b, sa, sb, out, M, N, K, gran, nullptr, stream);
}

extern "C" bsgemm_status bsgemm_fp8_tt(const void* a, const void* b, const float* sa, const float* sb,
                                       void* out, int64_t M, int64_t N, int64_t K, int gran,
                                       bsgemm_stream_t stream) {
  return bsgemm_fp8_gemm_ex(BSGEMM_LAYOUT_TT, a, b, sa, sb, out, M, N, K, gran, nullptr, stream);
}

extern "C" const char* bsgemm_status_string(bsgemm_status s) {
  switch (s) {
    case BSGEMM_OK: return "ok";
    case BSGEMM_ERR_INVALID_ARG: return "invalid argument";
    case BSGEMM_ERR_UNSUPPORTED_GRAN: return "unsupported granularity (use 64, 128 or 256)";
    case BSGEMM_ERR_MISALIGNED: return "misaligned pointer or stride (TMA needs 16-byte rows)";
    case BSGEMM_ERR_UNSUPPORTED_DEVICE: return "current device is not sm_100 (B200)";
    case BSGEMM_ERR_CUDA: return "CUDA runtime or driver call failed";
    case BSGEMM_ERR_DEVICE_TIMEOUT: return "a bounded device-side wait timed out";
    case BSGEMM_ERR_SCRATCH_LIMIT: return "problem needs more split-K scratch than the allocation-free entry point holds";
  }
  return "unknown status";
}

extern "C" bsgemm_status bsgemm_get_last_device_status(bsgemm_stream_t stream) {
  DeviceInfo dev;
  bsgemm_status st = device_info(dev);
  if (st != BSGEMM_OK) return st;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return BSGEMM_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof v) != cudaSuccess) return BSGEMM_ERR_CUDA;
  if (v == 0) return BSGEMM_OK;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof zero) != cudaSuccess) return BSGEMM_ERR_CUDA;
  // an aborted split-K launch may have left tile counters raised: clear them,
  // once no stream of the device still runs (workspaces are stream-ordered
  // allocations of their own streams)
  int cur = 0;
  cudaGetDevice(&cur);
  if (cudaDeviceSynchronize() != cudaSuccess) return BSGEMM_ERR_CUDA;
  {
    std::lock_guard<std::mutex> lk(bsg_host::g_mu);
    for (auto& kv : bsg_host::g_ws)
      if (kv.first.first == cur && kv.second.counters)
        cudaMemset(kv.second.counters, 0, kv.second.n_counters * sizeof(int));
  }
  if (cudaDeviceSynchronize() != cudaSuccess) return BSGEMM_ERR_CUDA;
  return static_cast<bsgemm_status>(v & 0xFF);
}

extern "C" bsgemm_status bsgemm_release_workspaces(void) {
  int cur = 0;
  if (cudaGetDevice(&cur) != cudaSuccess) return BSGEMM_ERR_CUDA;
  // no launch may still use the buffers
  if (cudaDeviceSynchronize() != cudaSuccess) return BSGEMM_ERR_CUDA;
  std::lock_guard<std::mutex> lk(bsg_host::g_mu);
  bsgemm_status st = BSGEMM_OK;
  for (auto it = bsg_host::g_ws.begin(); it != bsg_host::g_ws.end();) {
    if (it->first.first != cur) {
      ++it;
      continue;
    }
    if (it->second.ws && cudaFree(it->second.ws) != cudaSuccess) st = BSGEMM_ERR_CUDA;
    if (it->second.counters && cudaFree(it->second.counters) != cudaSuccess) st = BSGEMM_ERR_CUDA;
    it = bsg_host::g_ws.erase(it);
  }
  for (auto it = bsg_host::g_ids.begin(); it != bsg_host::g_ids.end();)
    it = it->first.first == cur ? bsg_host::g_ids.erase(it) : std::next(it);
  return st;
}

extern "C" int bsgemm_last_device_status_detail(void) {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof v) != cudaSuccess) return -1;
  return v;
}

// ------------------------------------------------------------------ diagnostics
namespace {
// One CTA waits on an mbarrier that nothing ever completes; the bounded wait
// must give up after `timeout_ns`, record the timeout and return.
__global__ void wait_timeout_probe(Params p) {
  __shared__ bsg::Barriers bars;
  if (threadIdx.x == 0) {
    bsg::mbar_init(bsg::smem_addr(&bars.full[0]), 1);
    bars.abort_flag = 0;
    bsg::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) bsg::bounded_wait(bsg::smem_addr(&bars.full[0]), 0, p, &bars, 7);
  __syncwarp();
  __syncthreads();
}
}  // namespace

extern "C" bsgemm_status bsgemm_diag_wait_timeout(unsigned long long timeout_ns, bsgemm_stream_t stream) {
  DeviceInfo dev;
  bsgemm_status st = device_info(dev);
  if (st != BSGEMM_OK) return st;
  if (timeout_ns == 0 || timeout_ns > 10000000000ull) return BSGEMM_ERR_INVALID_ARG;
  Params p{};
  p.status = dev.status;
  p.timeout_ns = timeout_ns;
  wait_timeout_probe<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(p);
  return cudaGetLastError() == cudaSuccess ? BSGEMM_OK : BSGEMM_ERR_CUDA;
}

extern "C" int bsgemm_version(void) { return 100; }
