// Block-scaled FP8 GEMM on CTA pairs (cluster of 2, tcgen05 cta_group::2).
//
// Same arithmetic as bsgemm_kernel (hncyxsy.com/news/191052, §2.2 block
// scaling, §3.2 promotion of each K-block's partial to FP32 with its scales),
// with a 256 x 256 output tile per CTA pair instead of 128 x 256 per CTA:
//   CTA r of the pair loads rows [256 tp + 128 r, +128) of A and rows
//   [256 tq + 128 r, +128) of B (N columns 128 r .. 128 r + 127 of the tile);
//   one thread of the even CTA issues tcgen05.mma.cta_group::2 (M = 256,
//   N = 256, K = 32), which reads A and B from both CTAs' shared memory and
//   writes rows 128 r .. 128 r + 127 of the partial into CTA r's TMEM.
// Each SM therefore streams 32 KB of operands per 128-deep stage for the same
// tensor work that costs 48 KB with a 128 x 256 tile per CTA, and six stages
// fit in shared memory beside the 32 KB of epilogue staging, instead of four.
// The epilogue is the single-CTA kernel's: each promotion warp stages its 32
// rows x 128 columns in 128-byte-swizzled chunks and one lane issues bulk
// tensor stores, so a tile's output leaves while the next tile's first
// K-blocks are promoted.
//
// Synchronisation (all mbarrier waits bounded, as in bsgemm_kernel):
//   full[s]        even CTA only: the even CTA's producer expects both CTAs'
//                  bytes; both producers' TMA loads complete on it;
//   empty[s]       both CTAs: the issuers' commits arrive on both;
//   tmem_full[b]   both CTAs: the issuing thread's commit arrives on both;
//   tmem_empty[b]  even CTA only: 16 arrivals, 8 promotion warps per CTA
//                  (the odd CTA's arrive across the cluster);
//   mma_done       even CTA only.
// A cluster barrier follows barrier initialisation and TMEM allocation, and
// another precedes TMEM release and exit, so neither CTA leaves while its
// peer may still touch its shared memory or TMEM.
#pragma once
#include "bsgemm_kernel.cuh"

namespace bsg {

constexpr int kPairM = 256;      // MMA M of the pair (128 rows per CTA)
constexpr int kPairN = 256;      // MMA N of the pair (tile width)
constexpr int kPairQRows = 128;  // Q rows (N columns) each CTA holds

struct PairCfg {
  static constexpr int kPBytes = BM * BK;          // 16 KB
  static constexpr int kQBytes = kPairQRows * BK;  // 16 KB
  static constexpr int kStageBytes = kPBytes + kQBytes;
  static constexpr int kEpiBytes = kNumEpiWarps * kEpiChunkBytes;  // 32 KB of store staging
  static constexpr int kBudget = 227 * 1024 - 1024 /*align slack*/ - 512 /*barriers*/;
  static constexpr int kStagesRaw = (kBudget - kEpiBytes) / kStageBytes;
  static constexpr int kStages = kStagesRaw > 8 ? 8 : kStagesRaw;
  static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + kEpiBytes + 512;
};

template <bool P_MN, bool Q_MN>
__device__ __forceinline__ constexpr uint32_t instr_desc_pair() {
  return (1u << 4)                                        // D format: F32
         | (0u << 7) | (0u << 10)                         // A, B format: or-ed in at run time
         | ((P_MN ? 1u : 0u) << 15) | ((Q_MN ? 1u : 0u) << 16)
         | (static_cast<uint32_t>(kPairN >> 3) << 17)
         | (static_cast<uint32_t>(kPairM >> 4) << 24);
}

// Whole 256 x 256 tiles only (no split-K / stream-K); Params.tiles_p and
// tiles_q count pair tiles, Params.num_work is their number.
template <int GRAN, bool P_MN, bool Q_MN>
__global__ void __launch_bounds__(kNumThreads, 1)
    bsgemm_pair_kernel(const __grid_constant__ CUtensorMap tm_p, const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_out, const Params p) {
  using PC = PairCfg;
  constexpr int STAGES = PC::kStages;
  constexpr int BNQ = kPairN;
  constexpr int kHalf = BNQ / 2;                      // columns per promotion warp
  constexpr int kNumGroups = (kHalf > GRAN) ? kHalf / GRAN : 1;
  constexpr int kGroupCols = kHalf / kNumGroups;
  constexpr int kBufs = 2;
  constexpr uint32_t kTmemCols = 512;
  constexpr uint32_t kTxBytes = 2 * PC::kStageBytes;  // both CTAs' loads of a stage
  static_assert(GRAN == 64 || GRAN == 128 || GRAN == 256, "granularity");
  static_assert(STAGES >= 4, "stages");
  // Two MMA-issuing warps of the even CTA take the K-blocks in turn, under
  // the single-CTA kernel's rules: buffers (2, even) belong to one issuer;
  // at g = 128 with an even ring every stage belongs to one issuer, else both
  // wait for every stage and release it (the other by a commit of no MMAs).
  constexpr int kIssuers = 2;
  constexpr bool kSharedStages = (GRAN != BK) || (STAGES % kIssuers != 0);
  constexpr int kStageUsers = kSharedStages ? 2 : 1;
  static_assert(kBufs % kIssuers == 0, "TMEM buffers split evenly between the issuers");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* p_tiles = smem;
  uint8_t* q_tiles = smem + STAGES * PC::kPBytes;
  uint8_t* epi_bufs = q_tiles + STAGES * PC::kQBytes;  // 1024-aligned: stage sizes are multiples of 1 KB
  Barriers* bars = reinterpret_cast<Barriers*>(epi_bufs + PC::kEpiBytes);

  const int warp = threadIdx.x / 32;
  const uint32_t lane = lane_id();
  const uint32_t rank = cluster_ctarank();          // 0: even CTA (issues the MMAs)
  const int cluster = static_cast<int>(blockIdx.x) >> 1;
  const int num_clusters = static_cast<int>(gridDim.x) >> 1;

  // -------------------------------------------------------------- setup
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_addr(&bars->full[s]), 1);
      mbar_init(smem_addr(&bars->empty[s]), kStageUsers);
    }
    for (int b = 0; b < kBufs; ++b) {
      mbar_init(smem_addr(&bars->tmem_full[b]), 1);
      mbar_init(smem_addr(&bars->tmem_empty[b]), 2 * kNumEpiWarps);
    }
    mbar_init(smem_addr(&bars->mma_done), kIssuers);
    bars->abort_flag = 0;
    bars->split_last = 0;
    fence_barrier_init();
  }
  if (warp == kProducerWarp && lane == 0) {
    tma_prefetch_desc(&tm_p);
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_out);
  }
  if (warp == kMmaWarp) {
    tmem_alloc_pair(smem_addr(&bars->tmem_base), kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = bars->tmem_base;
  // global memory is touched only after the grids this one depends on are
  // complete (programmatic dependent launch; see bsgemm_kernel); before
  // that, the producers pull their first tile's first stages towards L2
  // (a prefetch returns nothing, and L2 is coherent)
  if (warp == kProducerWarp && lane == 0 && cluster < p.num_work) {
    int tp, tq;
    tile_coords(p, cluster, tp, tq);
    const int prow = tp * kPairM + static_cast<int>(rank) * BM;
    const int qrow = tq * kPairN + static_cast<int>(rank) * kPairQRows;
    const int nst = (p.K + BK - 1) / BK;
    const int stop = nst < STAGES ? nst : STAGES;
    for (int st = 0; st < stop; ++st) {
      const int k = st * BK;
      if constexpr (P_MN) tma_prefetch_l2_2d(&tm_p, prow, k);
      else                tma_prefetch_l2_2d(&tm_p, k, prow);
      if constexpr (Q_MN) tma_prefetch_l2_2d(&tm_q, qrow, k);
      else                tma_prefetch_l2_2d(&tm_q, k, qrow);
    }
  }
  grid_dependency_wait();
  if (threadIdx.x == 0) grid_launch_dependents();

  if (warp < kFirstEpiWarp) {
    set_max_regs_dec<kProducerRegs>();
  if (warp == kProducerWarp) {
    // ============================================================ TMA producer (both CTAs)
    if (lane == 0) {
      uint32_t it = 0;  // stage-slot uses so far
      bool ok = true;
      for (int t = cluster; t < p.num_work && ok; t += num_clusters) {
        int tp, tq;
        tile_coords(p, t, tp, tq);
        const int prow = tp * kPairM + static_cast<int>(rank) * BM;
        const int qrow = tq * kPairN + static_cast<int>(rank) * kPairQRows;
        const int nst = (p.K + BK - 1) / BK;
        for (int st = 0; st < nst; ++st, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!bounded_wait<32>(smem_addr(&bars->empty[s]), ph ^ 1, p, bars, 1)) { ok = false; break; }
          const uint32_t fb_local = smem_addr(&bars->full[s]);
          if (rank == 0) mbar_arrive_expect_tx(fb_local, kTxBytes);
          const uint32_t fb = mapa_shared(fb_local, 0);  // the even CTA's full[s]
          const uint32_t pd = smem_addr(p_tiles + s * PC::kPBytes);
          const uint32_t qd = smem_addr(q_tiles + s * PC::kQBytes);
          const int k = st * BK;
          if constexpr (P_MN) tma_load_2d_pair(pd, &tm_p, fb, prow, k);
          else                tma_load_2d_pair(pd, &tm_p, fb, k, prow);
          if constexpr (Q_MN) tma_load_2d_pair(qd, &tm_q, fb, qrow, k);
          else                tma_load_2d_pair(qd, &tm_q, fb, k, qrow);
        }
      }
      if (!ok) {
        // drain the copies in flight before leaving: the even CTA waits for
        // the last stages' phases (they complete only when both CTAs' bytes
        // have landed); the odd CTA cannot observe its copies, so it waits a
        // fixed 100 us, far above any copy's latency
        if (rank == 0) {
          const uint32_t first = it > STAGES ? it - STAGES : 0;
          for (uint32_t j = first; j < it; ++j)
            bounded_wait(smem_addr(&bars->full[j % STAGES]), (j / STAGES) & 1, p, bars, 9, true);
        } else {
          const uint64_t t0 = globaltimer_ns();
          while (globaltimer_ns() - t0 < 100000ull) __nanosleep(1000);
        }
      }
    }
  } else if (warp == kMmaWarp || warp == kMmaWarp + 1) {
    // ============================================================ MMA issuers (even CTA)
    // Issuer i (warp kMmaWarp + i) takes the K-blocks x with x % 2 == i,
    // counted over the pair's tiles; both walk every stage.  Each warp runs
    // converged and predicates its tcgen05 instructions on elect.sync.
    if (rank == 0) {
      const uint32_t issuer = static_cast<uint32_t>(warp - kMmaWarp);
      const uint32_t idesc = instr_desc_pair<P_MN, Q_MN>() | p.fmt_bits;
      constexpr uint64_t kPStep = P_MN ? (kMmaK * 128) >> 4 : kMmaK >> 4;
      constexpr uint64_t kQStep = Q_MN ? (kMmaK * 128) >> 4 : kMmaK >> 4;
      constexpr uint64_t kPStage = PC::kPBytes >> 4, kQStage = PC::kQBytes >> 4;
      constexpr uint16_t kBoth = 0x3;
      const uint64_t ad0 = smem_desc_sw128(smem_addr(p_tiles), P_MN ? 128 * BK : 16);
      const uint64_t bd0 = smem_desc_sw128(smem_addr(q_tiles), Q_MN ? 128 * BK : 16);
      uint32_t s = 0, ph = 0;
      uint32_t x = 0;             // K-blocks so far
      bool ok = true;
      for (int t = cluster; t < p.num_work && ok; t += num_clusters) {
        for (int kb = 0; kb < p.Kb; ++kb, ++x) {
          // operands first (normally already there), then the TMEM buffer;
          // tmem_full is committed before the stage release
          const uint32_t b = x % kBufs, bph = (x / kBufs) & 1;
          const uint32_t d_tmem = tmem_base + b * BNQ;
          if constexpr (GRAN >= BK) {
            const bool mine = (x & 1) == issuer;
#pragma unroll
            for (int j = 0; j < GRAN / BK; ++j) {
              const int k0 = kb * GRAN + j * BK;
              if (k0 >= p.K) break;
              if (!mine && kSharedStages) {
                // the other issuer's stage: observe its fill and release it
                if (!warp_wait_all(smem_addr(&bars->full[s]), ph, p, bars, 2)) { ok = false; break; }
                mma_commit_pair_elect(smem_addr(&bars->empty[s]), kBoth);
              }
              if (mine) {
                if (!warp_wait_all(smem_addr(&bars->full[s]), ph, p, bars, 2)) { ok = false; break; }
                if (j == 0 && !warp_wait_all(smem_addr(&bars->tmem_empty[b]), bph ^ 1, p, bars, 3)) {
                  ok = false;
                  break;
                }
                const uint64_t ad = ad0 + s * kPStage, bd = bd0 + s * kQStage;
                if (k0 + BK <= p.K) {
#pragma unroll
                  for (int u = 0; u < BK / kMmaK; ++u)
                    mma_f8f6f4_pair_elect(d_tmem, ad + u * kPStep, bd + u * kQStep, idesc,
                                          (j > 0 || u > 0) ? 1u : 0u);
                } else {
                  const int nsteps = (p.K - k0 + kMmaK - 1) / kMmaK;
                  for (int u = 0; u < nsteps; ++u)
                    mma_f8f6f4_pair_elect(d_tmem, ad + u * kPStep, bd + u * kQStep, idesc,
                                          (j > 0 || u > 0) ? 1u : 0u);
                }
                if (j == GRAN / BK - 1 || k0 + BK >= p.K) mma_commit_pair_elect(smem_addr(&bars->tmem_full[b]), kBoth);
                mma_commit_pair_elect(smem_addr(&bars->empty[s]), kBoth);
              }
              if (++s == STAGES) { s = 0; ph ^= 1; }
            }
            if (!ok) break;
          } else {
            // GRAN == 64: a K-block is half a stage; a stage holds blocks x
            // and x + 1, one per issuer, and each releases it after its half;
            // at the K tail the other issuer waits for and releases a stage
            // that has no second half
            const int k0 = kb * GRAN;
            const int t0 = (kb & 1) * 2;
            const bool last_in_stage = (t0 == 2 || k0 + GRAN >= p.K);
            if ((x & 1) == issuer) {
              if (!warp_wait_all(smem_addr(&bars->full[s]), ph, p, bars, 2)) { ok = false; break; }
              if (!warp_wait_all(smem_addr(&bars->tmem_empty[b]), bph ^ 1, p, bars, 3)) { ok = false; break; }
              const uint64_t ad = ad0 + s * kPStage, bd = bd0 + s * kQStage;
              const int nsteps = (p.K - k0 >= GRAN) ? 2 : (p.K - k0 + kMmaK - 1) / kMmaK;
              for (int u = 0; u < nsteps; ++u)
                mma_f8f6f4_pair_elect(d_tmem, ad + (t0 + u) * kPStep, bd + (t0 + u) * kQStep, idesc,
                                      u > 0 ? 1u : 0u);
              mma_commit_pair_elect(smem_addr(&bars->tmem_full[b]), kBoth);
              mma_commit_pair_elect(smem_addr(&bars->empty[s]), kBoth);
            } else if (t0 == 0 && last_in_stage) {
              if (!warp_wait_all(smem_addr(&bars->full[s]), ph, p, bars, 2)) { ok = false; break; }
              mma_commit_pair_elect(smem_addr(&bars->empty[s]), kBoth);
            }
            if (last_in_stage) {
              if (++s == STAGES) { s = 0; ph ^= 1; }
            }
          }
        }
      }
      // every pair MMA both issuers issued completes before TMEM is freed
      mma_commit_pair_elect(smem_addr(&bars->mma_done), 0x1);
      warp_wait_all(smem_addr(&bars->mma_done), 0, p, bars, 8, true);
    }
  }
  } else {
    // ============================================================ promotion + epilogue (both CTAs)
    set_max_regs_inc<kPromoteRegs>();
    const int ew = warp - kFirstEpiWarp;   // 0..7
    const int quad = warp & 3;             // TMEM lane quadrant this warp may access
    const int half = ew >> 2;              // which half of the tile's columns
    const int row_in_tile = quad * 32 + static_cast<int>(lane);
    const uint32_t t_lane = static_cast<uint32_t>(quad * 32) << 16;
    uint32_t pc = 0;
    bool ok = true;
    float2 acc[kHalf / 2];

    for (int t = cluster; t < p.num_work && ok; t += num_clusters) {
      int tp, tq;
      tile_coords(p, t, tp, tq);
      const int prow0 = tp * kPairM + static_cast<int>(rank) * BM;   // first P row of this CTA
#pragma unroll
      for (int i = 0; i < kHalf / 2; ++i) acc[i] = make_float2(0.f, 0.f);

      int pb = (prow0 + quad * 32) / GRAN;
      pb = pb < p.Pb - 1 ? pb : p.Pb - 1;
      int qb[kNumGroups];
#pragma unroll
      for (int j = 0; j < kNumGroups; ++j) {
        const int bq = (tq * kPairN + half * kHalf + j * kGroupCols) / GRAN;
        qb[j] = bq < p.Qb - 1 ? bq : p.Qb - 1;
      }
      const float* sp_row = p.sP + static_cast<size_t>(pb) * p.Kb;
      float sc_cur[kNumGroups], sc_nxt[kNumGroups];
      auto load_chunk = [&](int base, float (&dst)[kNumGroups]) {
        const int kb = base + static_cast<int>(lane);
        const bool in = kb < p.Kb;
        const float a = in ? __ldg(sp_row + kb) : 0.f;
#pragma unroll
        for (int j = 0; j < kNumGroups; ++j)
          dst[j] = in ? a * __ldg(p.sQ + static_cast<size_t>(qb[j]) * p.Kb + kb) : 0.f;
      };
      load_chunk(0, sc_cur);
      load_chunk(32, sc_nxt);

      for (int kb = 0; kb < p.Kb; ++kb, ++pc) {
        if (kb > 0 && (kb & 31) == 0) {
#pragma unroll
          for (int j = 0; j < kNumGroups; ++j) sc_cur[j] = sc_nxt[j];
          load_chunk(kb + 32, sc_nxt);
        }
        float2 s2[kNumGroups];
#pragma unroll
        for (int j = 0; j < kNumGroups; ++j) {
          const float sv = __shfl_sync(0xffffffffu, sc_cur[j], kb & 31);
          s2[j] = make_float2(sv, sv);
        }
        const uint32_t buf = pc % kBufs;
        // every lane waits on the barrier itself: they all wake together when
        // the commit lands (a lane-0 wait plus a shuffle measured ~5 % slower)
        if (!warp_wait_all(smem_addr(&bars->tmem_full[buf]), (pc / kBufs) & 1, p, bars, 4)) { ok = false; break; }
        const uint32_t taddr = tmem_base + t_lane + buf * BNQ + half * kHalf;
        {
          // 64-column chunks; the buffer is released (to the even CTA's
          // tmem_empty) once the last chunk is in registers
          constexpr int CW = 64;
          constexpr int NC = kHalf / CW;
          uint32_t r[CW];
#pragma unroll
          for (int c = 0; c < NC; ++c) {
            tmem_ld(taddr + c * CW, r);
            tmem_wait_ld(r);
            if (c == NC - 1) {
              __syncwarp();
              if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_addr(&bars->tmem_empty[buf]), 0));
            }
#pragma unroll
            for (int i = 0; i < CW / 2; ++i) {
              const float2 sv = s2[(c * CW + 2 * i) / kGroupCols];
              acc[c * (CW / 2) + i] =
                  ffma2(make_float2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1])), sv,
                        acc[c * (CW / 2) + i]);
            }
          }
        }
      }
      if (!ok) break;

      // ---------------------------------------------------------- epilogue + store
      // this thread owns row prow0 + row_in_tile, columns [n0, n0 + kHalf);
      // the warp stores its 32 rows through its staging buffer
      const int n0 = tq * kPairN + half * kHalf;
      apply_epi<kHalf / 2>(p, n0, acc);
      store_tile_tma<kHalf / 2>(p, &tm_out, smem_addr(epi_bufs + ew * kEpiChunkBytes), prow0 + quad * 32, n0,
                                acc, lane);
    }
    // every bulk store this warp issued has finished before the CTA exits
    if (lane == 0) bulk_wait_group0();
  }
  __syncwarp();

  // -------------------------------------------------------------- teardown
  tc_fence_before();
  cluster_sync_all();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

}  // namespace bsg
