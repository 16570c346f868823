// bsgemm_fp8_nt_noalloc: the NT block-scaled FP8 GEMM for callers that cannot
// allocate device memory.
//
// Who needs it: code that runs where cudaMalloc is unavailable or forbidden --
// inside a host allocator callback, under a framework that owns all device
// memory and hands out nothing but the tensors it passes in, or in a process
// that must not grow its device footprint after start-up.  The regular entry
// points create a split-K / stream-K workspace on first use with cudaMalloc;
// this one never does.
//
// Instead, that scratch (FP32 partial tiles plus one counter per output tile
// that is cut into pieces) is a fixed array in the library's own device
// memory, declared below.
// Every GPU that loads the library holds one copy of it until the process
// exits.  Its size bounds the plans this entry point takes: where the regular
// plan would need more scratch than the array holds, it takes the largest
// split-K count whose partial tiles fit, down to no split at all, which needs
// no scratch.  A launch whose plan still needed more would be refused with
// BSGEMM_ERR_SCRATCH_LIMIT before anything is launched.
//
// All calls share the array, and it keeps whatever the last call left in it.
// The tile counters must start at zero, so each call clears them
// (cudaMemsetAsync on the caller's stream, which allocates nothing) before its
// kernel.  Two calls whose kernels overlap on the GPU -- different streams, or
// different host threads on one device -- race on the array and corrupt each
// other's results; callers must serialise them.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstring>

#include "bsgemm.h"
#include "bsgemm_host.h"
#include "bsgemm_kernel.cuh"

namespace {

constexpr size_t kPartialBytes = BSGEMM_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxTiles = BSGEMM_NOALLOC_MAX_TILES;

// The scratch: FP32 partial tiles first, then the tile counters.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kPartialBytes + kMaxTiles * sizeof(int)];

// Per-device set-up, done once by the first call on each device: the device
// address of the array (in host code its name is only a host-side stand-in).
// A fixed table, so the set-up itself allocates nothing either.
constexpr int kMaxDevices = 64;
struct DeviceScratch {
  std::atomic<int> state{0};  // 0 not set up, 1 being set up, 2 ready
  unsigned char* base = nullptr;
  int ordinal = 0;
  int num_sms = 0;
  int* status = nullptr;
};
DeviceScratch g_scratch[kMaxDevices];

bsgemm_status setup_current_device(DeviceScratch*& out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BSGEMM_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return BSGEMM_ERR_UNSUPPORTED_DEVICE;
  DeviceScratch& d = g_scratch[dev];
  int st = d.state.load(std::memory_order_acquire);
  while (st != 2) {
    int expect = 0;
    if (st == 0 && d.state.compare_exchange_strong(expect, 1)) {
      int major = 0, minor = 0, sms = 0;
      void* p = nullptr;
      int* status = nullptr;
      bool ok = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) == cudaSuccess &&
                cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) == cudaSuccess &&
                cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess;
      if (ok && !(major == 10 && minor == 0)) {
        d.state.store(0, std::memory_order_release);
        return BSGEMM_ERR_UNSUPPORTED_DEVICE;
      }
      ok = ok && cudaGetSymbolAddress(&p, g_noalloc_scratch) == cudaSuccess && p != nullptr;
      ok = ok && bsg_host::device_status_address(&status) == BSGEMM_OK;
      if (!ok) {
        d.state.store(0, std::memory_order_release);
        return BSGEMM_ERR_CUDA;
      }
      d.base = static_cast<unsigned char*>(p);
      d.ordinal = dev;
      d.num_sms = sms;
      d.status = status;
      d.state.store(2, std::memory_order_release);
    }
    st = d.state.load(std::memory_order_acquire);
  }
  out = &d;
  return BSGEMM_OK;
}

// Partial tiles and tile counters a plan needs: split-K one partial per piece
// and one counter per tile; stream-K two partials per CTA and one counter per
// stream-K tile; none without either.
void scratch_need(const bsgemm_plan& pl, size_t& partials, size_t& counters) {
  const size_t tiles = (size_t)pl.tiles_p * pl.tiles_q;
  if (pl.sk_ctas > 0) {
    partials = 2 * (size_t)pl.sk_ctas;
    counters = tiles - pl.sk_first_tile;
  } else if (pl.splits > 1) {
    partials = tiles * pl.splits;
    counters = tiles;
  } else {
    partials = counters = 0;
  }
}

bool fits(const bsgemm_plan& pl) {
  size_t partials = 0, counters = 0;
  scratch_need(pl, partials, counters);
  return partials * pl.bnq * bsg::BM * sizeof(float) <= kPartialBytes && counters <= (size_t)kMaxTiles;
}

// Same kernel as the regular NT split-K / stream-K path, launched on the fixed scratch.
template <int BNQ, int GRAN, bool SWAP>
bsgemm_status launch_fixed(const bsgemm_plan& plan, const void* a, const void* b, const float* sa,
                           const float* sb, void* out, int M, int N, int K, cudaStream_t stream,
                           const DeviceScratch& d) {
  using SC = bsg::StageCfg<BNQ, false, SWAP>;
  auto kern = bsg::bsgemm_kernel<BNQ, GRAN, SWAP, false, false, true>;
  const void* p_ptr = SWAP ? b : a;
  const void* q_ptr = SWAP ? a : b;
  const int P = SWAP ? N : M;
  const int Q = SWAP ? M : N;
  CUtensorMap tm_p, tm_q;
  if (!bsg_host::make_map_2d(&tm_p, p_ptr, CU_TENSOR_MAP_DATA_TYPE_UINT8, K, P, K, bsg::BK, bsg::BM) ||
      !bsg_host::make_map_2d(&tm_q, q_ptr, CU_TENSOR_MAP_DATA_TYPE_UINT8, K, Q, K, bsg::BK, BNQ))
    return BSGEMM_ERR_CUDA;
  CUtensorMap tm_out;
  std::memset(&tm_out, 0, sizeof tm_out);
  if (SC::kTmaStore && !bsg_host::make_out_map(&tm_out, out, M, N, false)) return BSGEMM_ERR_CUDA;
  if (SC::kSwapTmaStore && !bsg_host::make_swap_out_map(&tm_out, out, M, N, BNQ)) return BSGEMM_ERR_CUDA;

  bsg::Params prm{};
  prm.M = M; prm.N = N; prm.K = K;
  prm.Kb = (K + GRAN - 1) / GRAN;
  prm.Pb = (P + GRAN - 1) / GRAN;
  prm.Qb = (Q + GRAN - 1) / GRAN;
  prm.tiles_p = plan.tiles_p;
  prm.tiles_q = plan.tiles_q;
  const int num_tiles = plan.tiles_p * plan.tiles_q;
  prm.splits = plan.splits;
  prm.kb_per_split = plan.kb_per_split;
  prm.num_work = (plan.sk_ctas > 0 ? plan.sk_first_tile : num_tiles) * plan.splits;
  prm.sk_first_tile = plan.sk_first_tile;
  prm.sk_units_per_tile = plan.sk_units_per_tile;
  prm.sk_ctas = plan.sk_ctas;
  prm.sk_q = plan.sk_ctas > 0 ? plan.sk_units / plan.sk_ctas : 0;
  prm.sk_r = plan.sk_ctas > 0 ? plan.sk_units % plan.sk_ctas : 0;
  prm.group_p = plan.group_p;
  prm.sP = SWAP ? sb : sa;
  prm.sQ = SWAP ? sa : sb;
  prm.out = static_cast<__nv_bfloat16*>(out);
  prm.status = d.status;
  prm.timeout_ns = bsg_host::wait_timeout_ns();
  if (plan.splits > 1 || plan.sk_ctas > 0) {
    size_t partials = 0, counters = 0;
    scratch_need(plan, partials, counters);
    if (partials * BNQ * bsg::BM * sizeof(float) > kPartialBytes || counters > (size_t)kMaxTiles)
      return BSGEMM_ERR_SCRATCH_LIMIT;
    prm.ws = reinterpret_cast<float*>(d.base);
    prm.counters = reinterpret_cast<int*>(d.base + kPartialBytes);
    // the counters must start at zero; the array keeps the previous call's contents
    if (cudaMemsetAsync(prm.counters, 0, counters * sizeof(int), stream) != cudaSuccess)
      return BSGEMM_ERR_CUDA;
  }
  static bsg_host::PerDeviceOnce setup;  // once per instance and device
  if (!setup.done(d.ordinal)) {
    // the setmaxnreg split is only safe with exactly the planned launch registers
    if (bsg::RegSplit<BNQ>::kEnabled) {
      cudaFuncAttributes fa{};
      if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess || fa.numRegs != bsg::kLaunchRegs)
        return BSGEMM_ERR_CUDA;
    }
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SC::kSmemBytes) != cudaSuccess)
      return BSGEMM_ERR_CUDA;
    setup.mark(d.ordinal);
  }
  kern<<<plan.grid, bsg::kNumThreads, SC::kSmemBytes, stream>>>(tm_p, tm_q, tm_out, prm);
  return cudaGetLastError() == cudaSuccess ? BSGEMM_OK : BSGEMM_ERR_CUDA;
}

template <int GRAN>
bsgemm_status dispatch_fixed(const bsgemm_plan& pl, const void* a, const void* b, const float* sa,
                             const float* sb, void* out, int M, int N, int K, cudaStream_t s,
                             const DeviceScratch& d) {
  if (pl.swap_ab) {
    switch (pl.bnq) {
      case 16:  return launch_fixed<16, GRAN, true>(pl, a, b, sa, sb, out, M, N, K, s, d);
      case 32:  return launch_fixed<32, GRAN, true>(pl, a, b, sa, sb, out, M, N, K, s, d);
      case 64:  return launch_fixed<64, GRAN, true>(pl, a, b, sa, sb, out, M, N, K, s, d);
      case 128: return launch_fixed<128, GRAN, true>(pl, a, b, sa, sb, out, M, N, K, s, d);
      default:  return BSGEMM_ERR_INVALID_ARG;
    }
  }
  switch (pl.bnq) {
    case 128: return launch_fixed<128, GRAN, false>(pl, a, b, sa, sb, out, M, N, K, s, d);
    case 256: return launch_fixed<256, GRAN, false>(pl, a, b, sa, sb, out, M, N, K, s, d);
    default:  return BSGEMM_ERR_INVALID_ARG;
  }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

}  // namespace

extern "C" bsgemm_status bsgemm_fp8_nt_noalloc(const void* a, const void* b, const float* scale_a,
                                               const float* scale_b, void* out, int64_t M, int64_t N,
                                               int64_t K, int gran, bsgemm_stream_t stream) {
  if (!a || !b || !scale_a || !scale_b || !out) return BSGEMM_ERR_INVALID_ARG;
  if (M <= 0 || N <= 0 || K <= 0 || M > (1 << 30) || N > (1 << 30) || K > (1 << 30))
    return BSGEMM_ERR_INVALID_ARG;
  if (gran != 64 && gran != 128 && gran != 256) return BSGEMM_ERR_UNSUPPORTED_GRAN;
  if (!aligned16(a) || !aligned16(b) || !aligned16(out) || !aligned4(scale_a) || !aligned4(scale_b))
    return BSGEMM_ERR_MISALIGNED;
  if (K % 16 || N % 8) return BSGEMM_ERR_MISALIGNED;
  DeviceScratch* d = nullptr;
  bsgemm_status st = setup_current_device(d);
  if (st != BSGEMM_OK) return st;
  // The regular plan when its scratch fits.  Otherwise the same variant and
  // tile width without stream-K, with the heuristic's split count lowered
  // until its partial tiles fit the array; one split needs no scratch, so
  // every problem the regular entry point runs, this one runs too.
  // This entry point launches single-CTA tiles only: where the regular plan
  // takes CTA pairs (large g = 256 problems), it takes 128-row data-parallel
  // tiles instead.
  bsgemm_plan pl;
  st = bsgemm_make_plan(BSGEMM_LAYOUT_NT, M, N, K, gran, d->num_sms, nullptr, &pl);
  if (st != BSGEMM_OK) return st;
  if (pl.cta_pair) {
    const bsgemm_tuning dp = {BSGEMM_VARIANT_DATA_PARALLEL, 0, 0, 0};
    st = bsgemm_make_plan(BSGEMM_LAYOUT_NT, M, N, K, gran, d->num_sms, &dp, &pl);
    if (st != BSGEMM_OK) return st;
  }
  if (!fits(pl)) {
    const int variant = pl.swap_ab ? BSGEMM_VARIANT_SWAP_AB : BSGEMM_VARIANT_DATA_PARALLEL;
    const bsgemm_tuning no_sk = {variant, pl.bnq, 0, -1};
    st = bsgemm_make_plan(BSGEMM_LAYOUT_NT, M, N, K, gran, d->num_sms, &no_sk, &pl);
    if (st != BSGEMM_OK) return st;
    for (int s = pl.splits - 1; !fits(pl) && s >= 1; --s) {
      const bsgemm_tuning capped = {variant, pl.bnq, s, -1};
      st = bsgemm_make_plan(BSGEMM_LAYOUT_NT, M, N, K, gran, d->num_sms, &capped, &pl);
      if (st != BSGEMM_OK) return st;
    }
    if (!fits(pl)) return BSGEMM_ERR_SCRATCH_LIMIT;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int m = static_cast<int>(M), n = static_cast<int>(N), k = static_cast<int>(K);
  switch (gran) {
    case 64:  return dispatch_fixed<64>(pl, a, b, scale_a, scale_b, out, m, n, k, s, *d);
    case 128: return dispatch_fixed<128>(pl, a, b, scale_a, scale_b, out, m, n, k, s, *d);
    default:  return dispatch_fixed<256>(pl, a, b, scale_a, scale_b, out, m, n, k, s, *d);
  }
}
