// Kernel instances and launch code for one (granularity, layout) pair.
// The build compiles this file once per pair with -DBSG_GRAN=<64|128|256>
// and -DBSG_LAYOUT=<nt|tn|nn|tt>, so the twelve pairs build in parallel.
#include <cstring>

#include "bsgemm_host.h"
#include "bsgemm_kernel.cuh"
#include "bsgemm_pair.cuh"

#ifndef BSG_GRAN
#error "compile with -DBSG_GRAN=64|128|256"
#endif
#ifndef BSG_LAYOUT
#error "compile with -DBSG_LAYOUT=nt|tn|nn|tt"
#endif

#define BSG_CAT2(a, b, c, d) a##b##_##c
#define BSG_RUN_NAME(G, L) BSG_CAT2(run_g, G, L, )
#define BSG_STR2(x) #x
#define BSG_STR(x) BSG_STR2(x)

namespace bsg_host {
namespace {

// A stored [K,M] for tn/tt; B stored [K,N] for tn/nn (first letter A, second B).
constexpr const char* kLayout = BSG_STR(BSG_LAYOUT);
constexpr bool kAMn = kLayout[0] == 't';
constexpr bool kBMn = kLayout[1] == 'n';

// Format fields of the instruction descriptor for operands P (MMA A side)
// and Q (MMA B side).
inline uint32_t fmt_bits(int p_fmt, int q_fmt) {
  return (static_cast<uint32_t>(p_fmt) << 7) | (static_cast<uint32_t>(q_fmt) << 10);
}

template <int BNQ, int GRAN, bool SWAP, bool P_MN, bool Q_MN, bool SPLIT, bool GROUPED = false>
bsgemm_status launch(const bsgemm_plan& plan, const void* a, const void* b, const float* sa,
                     const float* sb, void* out, int M, int N, int K, const CallOpts& opts,
                     cudaStream_t stream, const DeviceInfo& dev) {
  using SC = bsg::StageCfg<BNQ, Q_MN, SWAP, GROUPED>;
  auto kern = bsg::bsgemm_kernel<BNQ, GRAN, SWAP, P_MN, Q_MN, SPLIT, GROUPED>;

  // P/Q operands: normally P = A (M rows), Q = B (N rows); swapped P = B, Q = A
  const void* p_ptr = SWAP ? b : a;
  const void* q_ptr = SWAP ? a : b;
  const int P = SWAP ? N : M;
  // grouped: B holds num_groups stacked [N, K] matrices
  const int Q = SWAP ? M : (GROUPED ? N * opts.num_groups : N);
  CUtensorMap tm_p, tm_q;
  bool ok = true;
  if (P_MN) ok &= make_map_2d(&tm_p, p_ptr, CU_TENSOR_MAP_DATA_TYPE_UINT8, P, K, P, 128, bsg::BK);
  else      ok &= make_map_2d(&tm_p, p_ptr, CU_TENSOR_MAP_DATA_TYPE_UINT8, K, P, K, bsg::BK, bsg::BM);
  if (Q_MN) ok &= make_map_2d(&tm_q, q_ptr, CU_TENSOR_MAP_DATA_TYPE_UINT8, Q, K, Q, 128, bsg::BK);
  else      ok &= make_map_2d(&tm_q, q_ptr, CU_TENSOR_MAP_DATA_TYPE_UINT8, K, Q, K, bsg::BK, BNQ);
  CUtensorMap tm_out;
  std::memset(&tm_out, 0, sizeof tm_out);
  if (SC::kTmaStore) ok &= make_out_map(&tm_out, out, M, N, (opts.epi & bsg::kEpiOutF32) != 0);
  if (SC::kSwapTmaStore && !(opts.epi & bsg::kEpiOutF32)) ok &= make_swap_out_map(&tm_out, out, M, N, BNQ);
  if (!ok) return BSGEMM_ERR_CUDA;

  bsg::Params prm{};
  prm.M = M; prm.N = N; prm.K = K;
  prm.Kb = (K + GRAN - 1) / GRAN;
  // grouped: sA has ceil(max_rows / g) + num_groups rows, sB ceil(N / g) per group
  prm.Pb = (P + GRAN - 1) / GRAN + (GROUPED ? opts.num_groups : 0);
  prm.Qb = ((GROUPED ? N : Q) + GRAN - 1) / GRAN;
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
  prm.fmt_bits = SWAP ? fmt_bits(opts.b_fmt, opts.a_fmt) : fmt_bits(opts.a_fmt, opts.b_fmt);
  prm.epi = opts.epi;
  prm.bias = opts.bias;
  prm.group_m = opts.group_m;
  prm.num_groups = GROUPED ? opts.num_groups : 0;
  prm.sP = SWAP ? sb : sa;
  prm.sQ = SWAP ? sa : sb;
  prm.out = static_cast<__nv_bfloat16*>(out);
  prm.status = dev.status;
  prm.timeout_ns = wait_timeout_ns();
  if (SPLIT && (plan.splits > 1 || plan.sk_ctas > 0)) {
    // split-K: one partial tile per piece; stream-K: two per CTA (its first and last tile)
    const size_t partials = plan.sk_ctas > 0 ? 2 * (size_t)plan.sk_ctas : (size_t)prm.num_work;
    const size_t counters = plan.sk_ctas > 0 ? (size_t)(num_tiles - plan.sk_first_tile) : (size_t)num_tiles;
    Workspace w;
    bsgemm_status st = get_workspace(stream, partials * BNQ * bsg::BM * sizeof(float), counters, w);
    if (st != BSGEMM_OK) return st;
    prm.ws = w.ws;
    prm.counters = w.counters;
  }

  static PerDeviceOnce setup;  // once per instance and device
  if (!setup.done(dev.ordinal)) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SC::kSmemBytes) != cudaSuccess)
      return BSGEMM_ERR_CUDA;
    if (bsg::RegSplit<BNQ>::kEnabled) {
      // the setmaxnreg split is only safe with exactly the planned launch registers
      cudaFuncAttributes fa{};
      if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess || fa.numRegs != bsg::kLaunchRegs)
        return BSGEMM_ERR_CUDA;
    }
    setup.mark(dev.ordinal);
  }
  // programmatic dependent launch: the kernel's set-up may overlap the tail
  // of the previous grid on the stream; it waits for that grid before any
  // global memory access (grid_dependency_wait)
  cudaLaunchConfig_t cfg{};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3(plan.grid, 1, 1);
  cfg.blockDim = dim3(bsg::kNumThreads, 1, 1);
  cfg.dynamicSmemBytes = SC::kSmemBytes;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, tm_p, tm_q, tm_out, prm) != cudaSuccess) return BSGEMM_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? BSGEMM_OK : BSGEMM_ERR_CUDA;
}

// 256 x 256 tiles on CTA pairs (cluster of 2); whole tiles only.
template <int GRAN, bool P_MN, bool Q_MN>
bsgemm_status launch_pair(const bsgemm_plan& plan, const void* a, const void* b, const float* sa,
                          const float* sb, void* out, int M, int N, int K, const CallOpts& opts,
                          cudaStream_t stream, const DeviceInfo& dev) {
  using PC = bsg::PairCfg;
  auto kern = bsg::bsgemm_pair_kernel<GRAN, P_MN, Q_MN>;
  CUtensorMap tm_p, tm_q;
  bool ok = true;
  if (P_MN) ok &= make_map_2d(&tm_p, a, CU_TENSOR_MAP_DATA_TYPE_UINT8, M, K, M, 128, bsg::BK);
  else      ok &= make_map_2d(&tm_p, a, CU_TENSOR_MAP_DATA_TYPE_UINT8, K, M, K, bsg::BK, bsg::BM);
  if (Q_MN) ok &= make_map_2d(&tm_q, b, CU_TENSOR_MAP_DATA_TYPE_UINT8, N, K, N, 128, bsg::BK);
  else      ok &= make_map_2d(&tm_q, b, CU_TENSOR_MAP_DATA_TYPE_UINT8, K, N, K, bsg::BK, bsg::kPairQRows);
  CUtensorMap tm_out;
  ok &= make_out_map(&tm_out, out, M, N, (opts.epi & bsg::kEpiOutF32) != 0);
  if (!ok) return BSGEMM_ERR_CUDA;

  bsg::Params prm{};
  prm.M = M; prm.N = N; prm.K = K;
  prm.Kb = (K + GRAN - 1) / GRAN;
  prm.Pb = (M + GRAN - 1) / GRAN;
  prm.Qb = (N + GRAN - 1) / GRAN;
  prm.tiles_p = plan.tiles_p;
  prm.tiles_q = plan.tiles_q;
  prm.splits = 1;
  prm.kb_per_split = prm.Kb;
  prm.num_work = plan.tiles_p * plan.tiles_q;
  prm.group_p = plan.group_p;
  prm.fmt_bits = fmt_bits(opts.a_fmt, opts.b_fmt);
  prm.epi = opts.epi;
  prm.bias = opts.bias;
  prm.sP = sa;
  prm.sQ = sb;
  prm.out = static_cast<__nv_bfloat16*>(out);
  prm.status = dev.status;
  prm.timeout_ns = wait_timeout_ns();

  cudaLaunchConfig_t cfg{};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // see launch()
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.blockDim = dim3(bsg::kNumThreads, 1, 1);
  cfg.dynamicSmemBytes = PC::kSmemBytes;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 2;

  // co-resident CTA pairs, found once per instance and device
  static PerDeviceOnce setup;
  static std::atomic<int> resident_pairs[64];
  const int slot = dev.ordinal >= 0 && dev.ordinal < 64 ? dev.ordinal : -1;
  int max_pairs = slot >= 0 && setup.done(slot) ? resident_pairs[slot].load(std::memory_order_relaxed) : 0;
  if (max_pairs == 0) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, PC::kSmemBytes) != cudaSuccess)
      return BSGEMM_ERR_CUDA;
    // the setmaxnreg split is only safe with exactly the planned launch registers
    cudaFuncAttributes fa{};
    if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess || fa.numRegs != bsg::kLaunchRegs)
      return BSGEMM_ERR_CUDA;
    cfg.gridDim = dim3(plan.grid, 1, 1);
    cfg.numAttrs = 1;  // the cluster shape alone decides residency
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) return BSGEMM_ERR_CUDA;
    cfg.numAttrs = 2;
    max_pairs = n;
    if (slot >= 0) {
      resident_pairs[slot].store(n, std::memory_order_relaxed);
      setup.mark(slot);
    }
  }
  // a persistent grid no larger than the pairs that can be resident at once
  int pairs = plan.grid / 2;
  if (pairs > max_pairs) pairs = max_pairs;
  if (pairs < 1) return BSGEMM_ERR_INVALID_ARG;
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  if (cudaLaunchKernelEx(&cfg, kern, tm_p, tm_q, tm_out, prm) != cudaSuccess) return BSGEMM_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? BSGEMM_OK : BSGEMM_ERR_CUDA;
}

}  // namespace

bsgemm_status BSG_RUN_NAME(BSG_GRAN, BSG_LAYOUT)(const bsgemm_plan& pl, const void* a, const void* b,
                                                 const float* sa, const float* sb, void* out, int M,
                                                 int N, int K, const CallOpts& o, cudaStream_t s,
                                                 const DeviceInfo& d) {
  constexpr int G = BSG_GRAN;
  if (pl.grouped) {
    // grouped GEMM: NT only, whole tiles
    if constexpr (!kAMn && !kBMn) {
      if (pl.bnq == 128) return launch<128, G, false, false, false, false, true>(pl, a, b, sa, sb, out, M, N, K, o, s, d);
      return launch<256, G, false, false, false, false, true>(pl, a, b, sa, sb, out, M, N, K, o, s, d);
    } else {
      return BSGEMM_ERR_INVALID_ARG;
    }
  }
  if (pl.cta_pair) return launch_pair<G, kAMn, kBMn>(pl, a, b, sa, sb, out, M, N, K, o, s, d);
  if (pl.swap_ab) {
    // P = B, Q = A
    switch (pl.bnq) {
      case 16:  return launch<16, G, true, kBMn, kAMn, true>(pl, a, b, sa, sb, out, M, N, K, o, s, d);
      case 32:  return launch<32, G, true, kBMn, kAMn, true>(pl, a, b, sa, sb, out, M, N, K, o, s, d);
      case 64:  return launch<64, G, true, kBMn, kAMn, true>(pl, a, b, sa, sb, out, M, N, K, o, s, d);
      case 128: return launch<128, G, true, kBMn, kAMn, true>(pl, a, b, sa, sb, out, M, N, K, o, s, d);
      default:  return BSGEMM_ERR_INVALID_ARG;
    }
  }
  const bool split = pl.splits > 1 || pl.sk_ctas > 0;
  switch (pl.bnq) {
    case 128:
      return split ? launch<128, G, false, kAMn, kBMn, true>(pl, a, b, sa, sb, out, M, N, K, o, s, d)
                   : launch<128, G, false, kAMn, kBMn, false>(pl, a, b, sa, sb, out, M, N, K, o, s, d);
    case 256:
      return split ? launch<256, G, false, kAMn, kBMn, true>(pl, a, b, sa, sb, out, M, N, K, o, s, d)
                   : launch<256, G, false, kAMn, kBMn, false>(pl, a, b, sa, sb, out, M, N, K, o, s, d);
    default:
      return BSGEMM_ERR_INVALID_ARG;
  }
}

}  // namespace bsg_host
