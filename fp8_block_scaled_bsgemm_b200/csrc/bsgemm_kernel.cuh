// Block-scaled FP8 GEMM kernel for sm_100a (B200).
//
// Computes, per output element (hncyxsy.com/news/191052, §2.2 block scaling,
// §3.2 "K is cut into segments, accumulated separately, then added"):
//   out[m,n] = bf16( sum_kb sA[m/g][kb] * sB[n/g][kb] * P_kb[m,n] ),
//   P_kb[m,n] = sum_{k in K-block kb} A[m,k] * B[n,k]   (E4M3 x E4M3 -> FP32)
//
// The kernel speaks of two operands, P and Q:
//   P feeds the MMA's M side (128 TMEM lanes per tile),
//   Q feeds the MMA's N side (BNQ TMEM columns per tile).
// Normally P = A and Q = B.  For small M ("swap-AB") P = B and Q = A, so the
// weight rows fill the 128-row MMA and the few token rows sit in the narrow N.
//
// One persistent CTA per SM, 12 warps (3 warpgroups):
//   warp 0   TMA producer: P and Q tiles of 128 K-bytes into a STAGES-deep
//            ring of 128B-swizzled shared-memory buffers (mbarrier full/empty);
//   warp 1   TMEM owner and MMA issuer: for each K-block, tcgen05.mma
//            (kind::f8f6f4, K = 32 per instruction) into one of two TMEM
//            partial buffers, then tcgen05.commit to tell the promoters;
//   warps 2-3 idle (they complete the first warpgroup);
//   warps 4-11 promotion + epilogue: tcgen05.ld each K-block's partial,
//            acc += (sP*sQ) * partial in FP32 registers (packed f32x2 FMAs),
//            release the TMEM buffer, and at the end of a tile round to BF16
//            and store it (TMA store, or direct stores in swap-AB mode).
// Split-K: a tile's K-blocks are divided among `splits` work items; each
// writes an FP32 partial tile to a workspace, and the last to arrive (per-tile
// counter) adds all partials in split order -- the same order every run -- and
// stores the BF16 tile.
//
// Every mbarrier wait is bounded by a %globaltimer deadline.  When one runs
// out the kernel records BSGEMM_ERR_DEVICE_TIMEOUT in the status word, raises
// a CTA-wide abort flag that every other wait checks, drains its own copies in
// flight, frees TMEM and returns.  Nothing traps.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace bsg {

constexpr int kNumThreads = 384;
constexpr int kProducerWarp = 0;
constexpr int kMmaWarp = 1;
constexpr int kFirstEpiWarp = 4;
constexpr int kNumEpiWarps = 8;
constexpr int kNumEpiThreads = kNumEpiWarps * 32;
constexpr int BM = 128;       // MMA M = TMEM lanes per tile
constexpr int BK = 128;       // K elements (= bytes, FP8) per pipeline stage
constexpr int kMmaK = 32;     // K per tcgen05.mma kind::f8f6f4
constexpr int kTimeoutCode = 6;  // BSGEMM_ERR_DEVICE_TIMEOUT

// Register split for the widest tiles (128 accumulator columns per promotion
// thread): the launch gives every thread kLaunchRegs; the producer/MMA
// warpgroup gives registers back and the two promotion warpgroups take them.
// setmaxnreg.inc can only be satisfied if the launch really had kLaunchRegs
// per thread, so the host checks the compiled count before every launch.
constexpr int kLaunchRegs = 168;
constexpr int kProducerRegs = 72;
constexpr int kPromoteRegs = 216;
static_assert(kProducerRegs * 128 + kPromoteRegs * 256 <= kLaunchRegs * kNumThreads,
              "register split exceeds the launch allocation");

template <int BNQ>
struct RegSplit {
  static constexpr bool kEnabled = (BNQ == 256);
};

struct Params {
  int M, N, K;           // logical GEMM sizes
  int P, Q;              // rows of the P operand and of the Q operand
  int Kb;                // ceil(K / gran)
  int Pb, Qb;            // ceil(P / gran), ceil(Q / gran)
  int tiles_p, tiles_q;  // tiles along P (128 rows) and along Q (BNQ rows)
  int num_tiles;
  int splits;            // K splits per tile (1 = none)
  int kb_per_split;      // K-blocks per split (even when gran == 64)
  int num_work;          // num_tiles * splits
  int group_p;           // raster group height in P tiles (L2 locality)
  const float* sP;       // [Pb][Kb]
  const float* sQ;       // [Qb][Kb]
  __nv_bfloat16* out;    // [M][N] row-major (direct stores in swap mode)
  float* ws;             // split partials: [num_tiles][splits][BNQ][BM]
  int* counters;         // [num_tiles], zero between launches
  int* status;           // device status word
  unsigned long long timeout_ns;
};

template <int BNQ, bool Q_MN>
struct Tiles {
  static constexpr int kPBytes = BM * BK;                                // 16 KB
  static constexpr int kQRows = (Q_MN && BNQ < 128) ? 128 : BNQ;         // MN-major: 128-wide atom
  static constexpr int kQBytes = kQRows * BK;
};

template <int BNQ, bool Q_MN, bool SWAP>
struct StageCfg {
  static constexpr int kStageBytes = Tiles<BNQ, Q_MN>::kPBytes + Tiles<BNQ, Q_MN>::kQBytes;
  static constexpr int kEpiBytes = SWAP ? 0 : kNumEpiWarps * 32 * 128;  // 4 KB per warp
  static constexpr int kBudget = 227 * 1024 - 1024 /*align slack*/ - 512 /*barriers*/;
  static constexpr int kStagesRaw = (kBudget - kEpiBytes) / kStageBytes;
  static constexpr int kStages = kStagesRaw > 8 ? 8 : kStagesRaw;
  static_assert(kStages >= 2, "shared memory too small for two stages");
  static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + kEpiBytes + 512;
};

struct __align__(8) Barriers {
  uint64_t full[8];
  uint64_t empty[8];
  uint64_t tmem_full[2];
  uint64_t tmem_empty[2];
  uint64_t mma_done;
  uint64_t epi_sync;     // bounded rendezvous of the promotion warps (split-K)
  uint32_t tmem_base;
  int abort_flag;
  int split_last;
};

// ---------------------------------------------------------------- helpers
__device__ __forceinline__ void record_timeout(const Params& p, Barriers* bars, int where) {
  *reinterpret_cast<volatile int*>(&bars->abort_flag) = 1;
  atomicCAS(p.status, 0, kTimeoutCode | (where << 8));
}

// Bounded mbarrier wait. Returns false on timeout or when another warp of the
// CTA has raised the abort flag (unless ignore_abort).
__device__ __forceinline__ bool bounded_wait(uint32_t bar, uint32_t parity, const Params& p,
                                          Barriers* bars, int where, bool ignore_abort = false) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (!ignore_abort && *reinterpret_cast<volatile int*>(&bars->abort_flag)) return false;
    if (globaltimer_ns() - t0 > p.timeout_ns) {
      if (!ignore_abort) record_timeout(p, bars, where);
      return false;
    }
  }
}

// Warp-uniform bounded wait: lane 0 waits, every lane gets the same answer,
// and the warp is converged afterwards (needed before .sync.aligned ops).
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, const Params& p,
                                          Barriers* bars, int where) {
  int ok = 0;
  if (lane_id() == 0) ok = bounded_wait(bar, parity, p, bars, where) ? 1 : 0;
  ok = __shfl_sync(0xffffffffu, ok, 0);
  __syncwarp();
  return ok != 0;
}

// Bounded rendezvous of the promotion warps (replaces an unbounded bar.sync,
// which would hang if one warp had left on an abort). `uses` counts this
// thread's previous rendezvous.
__device__ __forceinline__ bool epi_rendezvous(uint32_t& uses, const Params& p, Barriers* bars) {
  __syncwarp();
  const uint32_t bar = smem_addr(&bars->epi_sync);
  if (lane_id() == 0) mbar_arrive(bar);
  const bool ok = warp_wait(bar, uses & 1, p, bars, 5);
  ++uses;
  return ok;
}

// Shared-memory matrix descriptor for tcgen05 (sm_100 format, version 1),
// 128-byte swizzle.  K-major: rows of 128 B, 8-row groups 1024 B apart (SBO);
// MN-major: k-rows of 128 B, 8-k-row groups 1024 B apart (SBO), 128-element
// MN chunks `lbo` bytes apart (LBO).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr, uint32_t lbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((addr >> 4) & 0x3FFF);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFF) << 16;
  d |= static_cast<uint64_t>((1024 >> 4) & 0x3FFF) << 32;
  d |= 1ull << 46;  // descriptor version for sm_100
  d |= 2ull << 61;  // SWIZZLE_128B
  return d;
}

// Instruction descriptor: kind::f8f6f4, A = B = E4M3, D = F32, M = 128, N = BNQ.
template <int BNQ, bool P_MN, bool Q_MN>
__device__ __forceinline__ constexpr uint32_t instr_desc() {
  return (1u << 4)                               // D format: F32
         | (0u << 7) | (0u << 10)                // A, B format: E4M3
         | ((P_MN ? 1u : 0u) << 15)              // A major (0 = K)
         | ((Q_MN ? 1u : 0u) << 16)              // B major
         | (static_cast<uint32_t>(BNQ >> 3) << 17)
         | (static_cast<uint32_t>(BM >> 4) << 24);
}

struct Work {
  int tile, split, tp, tq, kb0, kb1;
};

__device__ __forceinline__ Work decode_work(const Params& p, int w) {
  Work x;
  x.tile = w / p.splits;
  x.split = w - x.tile * p.splits;
  // grouped raster: walk group_p P-tiles down, then across Q
  const int per_group = p.group_p * p.tiles_q;
  const int grp = x.tile / per_group;
  const int first_p = grp * p.group_p;
  int rows = p.tiles_p - first_p;
  rows = rows < p.group_p ? rows : p.group_p;
  const int local = x.tile - grp * per_group;
  x.tp = first_p + local % rows;
  x.tq = local / rows;
  x.kb0 = x.split * p.kb_per_split;
  x.kb1 = x.kb0 + p.kb_per_split;
  if (x.kb1 > p.Kb) x.kb1 = p.Kb;
  return x;
}

// Pipeline stages [st0, st1) of 128 K-elements that K-blocks [kb0, kb1) cover.
template <int GRAN>
__device__ __forceinline__ void stage_range(const Params& p, const Work& w, int& st0, int& st1) {
  const int nst = (p.K + BK - 1) / BK;
  if constexpr (GRAN >= BK) {
    constexpr int spp = GRAN / BK;
    st0 = w.kb0 * spp;
    st1 = w.kb1 * spp;
  } else {
    st0 = w.kb0 / 2;
    st1 = (w.kb1 + 1) / 2;
  }
  if (st1 > nst) st1 = nst;
}

// ---------------------------------------------------------------- kernel
template <int BNQ, int GRAN, bool SWAP, bool P_MN, bool Q_MN, bool SPLIT>
__global__ void __launch_bounds__(kNumThreads, 1)
    bsgemm_kernel(const __grid_constant__ CUtensorMap tm_p, const __grid_constant__ CUtensorMap tm_q,
                  const __grid_constant__ CUtensorMap tm_out, const Params p) {
  using TL = Tiles<BNQ, Q_MN>;
  using SC = StageCfg<BNQ, Q_MN, SWAP>;
  constexpr int STAGES = SC::kStages;
  constexpr int kHalf = BNQ / 2;                      // columns per promotion warp
  constexpr int kNumGroups = (kHalf > GRAN) ? kHalf / GRAN : 1;  // scale groups per warp
  constexpr int kGroupCols = kHalf / kNumGroups;
  constexpr uint32_t kTmemCols = (2 * BNQ <= 32) ? 32 : (2 * BNQ <= 64) ? 64
                                : (2 * BNQ <= 128) ? 128 : (2 * BNQ <= 256) ? 256 : 512;
  constexpr uint32_t kTxBytes = TL::kPBytes + TL::kQBytes;
  static_assert(BNQ % 16 == 0 && BNQ >= 16 && BNQ <= 256, "MMA N must be a multiple of 16 in [16, 256]");
  static_assert(GRAN == 64 || GRAN == 128 || GRAN == 256, "granularity");
  static_assert(kHalf % 8 == 0, "columns per warp");
  static_assert(SWAP || kHalf % 64 == 0, "TMA-store epilogue writes 64-column boxes");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* p_tiles = smem;
  uint8_t* q_tiles = smem + STAGES * TL::kPBytes;
  uint8_t* epi_buf = q_tiles + STAGES * TL::kQBytes;
  Barriers* bars = reinterpret_cast<Barriers*>(epi_buf + SC::kEpiBytes);

  const int warp = threadIdx.x / 32;
  const uint32_t lane = lane_id();

  // -------------------------------------------------------------- setup
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_addr(&bars->full[s]), 1);
      mbar_init(smem_addr(&bars->empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_addr(&bars->tmem_full[b]), 1);
      mbar_init(smem_addr(&bars->tmem_empty[b]), kNumEpiWarps);
    }
    mbar_init(smem_addr(&bars->mma_done), 1);
    mbar_init(smem_addr(&bars->epi_sync), kNumEpiWarps);
    bars->abort_flag = 0;
    bars->split_last = 0;
    fence_barrier_init();
  }
  if (warp == kProducerWarp && lane == 0) {
    tma_prefetch_desc(&tm_p);
    tma_prefetch_desc(&tm_q);
    if (!SWAP) tma_prefetch_desc(&tm_out);
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_addr(&bars->tmem_base), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = bars->tmem_base;

  if (warp < kFirstEpiWarp) {
    // warpgroup 0: producer, MMA issuer and two idle warps
    if constexpr (RegSplit<BNQ>::kEnabled) set_max_regs_dec<kProducerRegs>();
  if (warp == kProducerWarp) {
    // ============================================================ TMA producer
    if (lane == 0) {
      uint32_t it = 0;  // stage-slot uses so far
      bool ok = true;
      for (int wi = blockIdx.x; wi < p.num_work && ok; wi += gridDim.x) {
        const Work w = decode_work(p, wi);
        int st0, st1;
        stage_range<GRAN>(p, w, st0, st1);
        for (int st = st0; st < st1; ++st, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!bounded_wait(smem_addr(&bars->empty[s]), ph ^ 1, p, bars, 1)) { ok = false; break; }
          const uint32_t fb = smem_addr(&bars->full[s]);
          mbar_arrive_expect_tx(fb, kTxBytes);
          const uint32_t pd = smem_addr(p_tiles + s * TL::kPBytes);
          const uint32_t qd = smem_addr(q_tiles + s * TL::kQBytes);
          const int k = st * BK;
          if constexpr (P_MN) tma_load_2d(pd, &tm_p, fb, w.tp * BM, k);
          else                tma_load_2d(pd, &tm_p, fb, k, w.tp * BM);
          if constexpr (Q_MN) {
#pragma unroll
            for (int c = 0; c < TL::kQRows / 128; ++c)
              tma_load_2d(qd + c * 128 * BK, &tm_q, fb, w.tq * BNQ + c * 128, k);
          } else {
            tma_load_2d(qd, &tm_q, fb, k, w.tq * BNQ);
          }
        }
      }
      if (!ok) {
        // drain: wait (bounded, ignoring the abort flag) for the copies this
        // thread started and nobody consumed, so none lands after exit
        const uint32_t first = it > STAGES ? it - STAGES : 0;
        for (uint32_t j = first; j < it; ++j)
          bounded_wait(smem_addr(&bars->full[j % STAGES]), (j / STAGES) & 1, p, bars, 9, true);
      }
    }
  } else if (warp == kMmaWarp) {
    // ============================================================ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = instr_desc<BNQ, P_MN, Q_MN>();
      uint32_t it = 0;   // stage-slot uses so far
      uint32_t pc = 0;   // K-blocks (TMEM partials) produced so far
      bool ok = true;
      for (int wi = blockIdx.x; wi < p.num_work && ok; wi += gridDim.x) {
        const Work w = decode_work(p, wi);
        int st0, st1;
        stage_range<GRAN>(p, w, st0, st1);
        int cur_kb = -1;
        uint32_t buf = 0, accum = 0;
        for (int st = st0; st < st1 && ok; ++st, ++it) {
          const int s = it % STAGES;
          if (!bounded_wait(smem_addr(&bars->full[s]), (it / STAGES) & 1, p, bars, 2)) { ok = false; break; }
          tc_fence_after();
          const uint32_t pa = smem_addr(p_tiles + s * TL::kPBytes);
          const uint32_t qa = smem_addr(q_tiles + s * TL::kQBytes);
#pragma unroll
          for (int kk = 0; kk < BK / kMmaK; ++kk) {
            const int k = st * BK + kk * kMmaK;
            const int kb = k / GRAN;
            if (k >= p.K || kb >= w.kb1) break;
            if (kb < w.kb0) continue;
            if (kb != cur_kb) {
              if (cur_kb >= 0) { mma_commit(smem_addr(&bars->tmem_full[buf])); ++pc; }
              cur_kb = kb;
              buf = pc & 1;
              if (!bounded_wait(smem_addr(&bars->tmem_empty[buf]), ((pc >> 1) & 1) ^ 1, p, bars, 3)) {
                ok = false;
                break;
              }
              tc_fence_after();
              accum = 0;
            }
            const uint64_t ad = P_MN ? smem_desc_sw128(pa + kk * kMmaK * 128, 128 * BK)
                                     : smem_desc_sw128(pa + kk * kMmaK, 16);
            const uint64_t bd = Q_MN ? smem_desc_sw128(qa + kk * kMmaK * 128, 128 * BK)
                                     : smem_desc_sw128(qa + kk * kMmaK, 16);
            mma_f8f6f4(tmem_base + buf * BNQ, ad, bd, idesc, accum);
            accum = 1;
          }
          mma_commit(smem_addr(&bars->empty[s]));  // stage free once these MMAs finish
        }
        if (ok && cur_kb >= 0) { mma_commit(smem_addr(&bars->tmem_full[buf])); ++pc; }
      }
      // all MMAs issued by this thread complete before TMEM is freed
      mma_commit(smem_addr(&bars->mma_done));
      bounded_wait(smem_addr(&bars->mma_done), 0, p, bars, 8, true);
    }
  }
  } else {
    // ============================================================ promotion + epilogue
    if constexpr (RegSplit<BNQ>::kEnabled) set_max_regs_inc<kPromoteRegs>();
    const int ew = warp - kFirstEpiWarp;   // 0..7
    const int quad = warp & 3;             // TMEM lane quadrant this warp may access
    const int half = ew >> 2;              // which half of the BNQ columns
    const int row_in_tile = quad * 32 + static_cast<int>(lane);
    const uint32_t t_lane = static_cast<uint32_t>(quad * 32) << 16;
    uint32_t pc = 0;          // K-blocks consumed so far (TMEM buffer / phase)
    uint32_t sync_uses = 0;   // epilogue rendezvous so far
    bool ok = true;
    float2 acc[kHalf / 2];    // this thread's row, columns [half*kHalf, (half+1)*kHalf)

    for (int wi = blockIdx.x; wi < p.num_work && ok; wi += gridDim.x) {
      const Work w = decode_work(p, wi);
#pragma unroll
      for (int i = 0; i < kHalf / 2; ++i) acc[i] = make_float2(0.f, 0.f);

      // scale rows for this warp: one P block, kNumGroups Q blocks (clamped:
      // rows past the end of P/Q hold zeros and are never stored)
      int pb = (w.tp * BM + quad * 32) / GRAN;
      pb = pb < p.Pb - 1 ? pb : p.Pb - 1;
      int qb[kNumGroups];
#pragma unroll
      for (int j = 0; j < kNumGroups; ++j) {
        const int b = (w.tq * BNQ + half * kHalf + j * kGroupCols) / GRAN;
        qb[j] = b < p.Qb - 1 ? b : p.Qb - 1;
      }
      const float* sp_row = p.sP + static_cast<size_t>(pb) * p.Kb;
      // lane i holds sP*sQ of K-block (chunk base + i); the next chunk is in flight
      float sc_cur[kNumGroups], sc_nxt[kNumGroups];
      auto load_chunk = [&](int base, float (&dst)[kNumGroups]) {
        const int kb = base + static_cast<int>(lane);
        const bool in = kb < w.kb1;
        const float a = in ? __ldg(sp_row + kb) : 0.f;
#pragma unroll
        for (int j = 0; j < kNumGroups; ++j)
          dst[j] = in ? a * __ldg(p.sQ + static_cast<size_t>(qb[j]) * p.Kb + kb) : 0.f;
      };
      load_chunk(w.kb0, sc_cur);
      load_chunk(w.kb0 + 32, sc_nxt);

      for (int kb = w.kb0; kb < w.kb1; ++kb, ++pc) {
        const int rel = kb - w.kb0;
        if (rel > 0 && (rel & 31) == 0) {
#pragma unroll
          for (int j = 0; j < kNumGroups; ++j) sc_cur[j] = sc_nxt[j];
          load_chunk(kb + 32, sc_nxt);
        }
        float2 s2[kNumGroups];
#pragma unroll
        for (int j = 0; j < kNumGroups; ++j) {
          const float sv = __shfl_sync(0xffffffffu, sc_cur[j], rel & 31);
          s2[j] = make_float2(sv, sv);
        }

        const uint32_t buf = pc & 1;
        if (!warp_wait(smem_addr(&bars->tmem_full[buf]), (pc >> 1) & 1, p, bars, 4)) { ok = false; break; }
        tc_fence_after();
        const uint32_t taddr = tmem_base + t_lane + buf * BNQ + half * kHalf;
        {
          // TMEM -> registers in chunks of CW columns, two chunks in flight;
          // 128 accumulator columns per thread leave room for 2 x 8 only
          constexpr int CW = (kHalf >= 128 || kHalf % 16 != 0) ? 8 : 16;
          constexpr int NC = kHalf / CW;
          uint32_t ra[CW], rb[CW];
          auto fma_chunk = [&](const uint32_t (&r)[CW], int c) {
            const float2 sv = s2[(c * CW) / kGroupCols];
#pragma unroll
            for (int i = 0; i < CW / 2; ++i)
              acc[c * (CW / 2) + i] =
                  ffma2(make_float2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1])), sv,
                        acc[c * (CW / 2) + i]);
          };
          tmem_ld(taddr, ra);
          tmem_wait_ld(ra);
#pragma unroll
          for (int c = 0; c < NC; c += 2) {
            if (c + 1 < NC) tmem_ld(taddr + (c + 1) * CW, rb);
            fma_chunk(ra, c);
            if (c + 1 < NC) {
              tmem_wait_ld(rb);
              if (c + 2 < NC) tmem_ld(taddr + (c + 2) * CW, ra);
              fma_chunk(rb, c + 1);
              if (c + 2 < NC) tmem_wait_ld(ra);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_addr(&bars->tmem_empty[buf]));
      }
      if (!ok) break;

      // ---------------------------------------------------------- split-K fix-up
      if constexpr (SPLIT) {
        if (p.splits > 1) {
          // partial tile, column-major [BNQ][BM]: a warp writes 128 contiguous bytes per column
          float* my_ws = p.ws + (static_cast<size_t>(w.tile) * p.splits + w.split) * (BNQ * BM);
#pragma unroll
          for (int i = 0; i < kHalf / 2; ++i) {
            __stcg(my_ws + (half * kHalf + 2 * i) * BM + row_in_tile, acc[i].x);
            __stcg(my_ws + (half * kHalf + 2 * i + 1) * BM + row_in_tile, acc[i].y);
          }
          __threadfence();
          // the partial now lives in the workspace; acc is dead until the sum below
          if (!epi_rendezvous(sync_uses, p, bars)) { ok = false; break; }
          if (ew == 0 && lane == 0) {
            const int old = atomicAdd(p.counters + w.tile, 1);
            bars->split_last = (old == p.splits - 1) ? 1 : 0;
          }
          if (!epi_rendezvous(sync_uses, p, bars)) { ok = false; break; }
          const bool last = *reinterpret_cast<volatile int*>(&bars->split_last) != 0;
          // nobody may overwrite split_last before every warp has read it
          if (!epi_rendezvous(sync_uses, p, bars)) { ok = false; break; }
          if (!last) continue;
          __threadfence();
          // fixed order: split 0, 1, ..., whoever arrived last
          const float* tile_ws = p.ws + static_cast<size_t>(w.tile) * p.splits * (BNQ * BM) +
                                 (half * kHalf) * BM + row_in_tile;
#pragma unroll
          for (int i = 0; i < kHalf / 2; ++i) {
            acc[i].x = __ldcg(tile_ws + (2 * i) * BM);
            acc[i].y = __ldcg(tile_ws + (2 * i + 1) * BM);
          }
          for (int sidx = 1; sidx < p.splits; ++sidx) {
            const float* src = tile_ws + static_cast<size_t>(sidx) * (BNQ * BM);
#pragma unroll
            for (int i = 0; i < kHalf / 2; ++i) {
              acc[i].x += __ldcg(src + (2 * i) * BM);
              acc[i].y += __ldcg(src + (2 * i + 1) * BM);
            }
          }
          if (ew == 0 && lane == 0) p.counters[w.tile] = 0;  // ready for the next launch
        }
      }

      // ---------------------------------------------------------- BF16 store
      if constexpr (SWAP) {
        // tile rows are N, tile columns are M: out[m][n]
        const int n = w.tp * BM + row_in_tile;
        if (n < p.N) {
#pragma unroll
          for (int i = 0; i < kHalf; ++i) {
            const int m = w.tq * BNQ + half * kHalf + i;
            const float v = (i & 1) ? acc[i / 2].y : acc[i / 2].x;
            if (m < p.M) p.out[static_cast<size_t>(m) * p.N + n] = __float2bfloat16_rn(v);
          }
        }
      } else {
        uint8_t* stage_buf = epi_buf + ew * (32 * 128);
        const uint32_t sbase = smem_addr(stage_buf);
#pragma unroll
        for (int box = 0; box < kHalf / 64; ++box) {
          if (lane == 0) bulk_wait_group_read0();  // previous store done reading the buffer
          __syncwarp();
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const int i0 = box * 32 + c * 4;  // float2 index of column box*64 + c*8
            const uint32_t x = pack_bf16x2(acc[i0].x, acc[i0].y);
            const uint32_t y = pack_bf16x2(acc[i0 + 1].x, acc[i0 + 1].y);
            const uint32_t z = pack_bf16x2(acc[i0 + 2].x, acc[i0 + 2].y);
            const uint32_t q = pack_bf16x2(acc[i0 + 3].x, acc[i0 + 3].y);
            // 128B swizzle: 16-byte chunk c of row `lane` lives at chunk c ^ (lane % 8)
            const uint32_t off = lane * 128 + ((c ^ (lane & 7)) * 16);
            asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(sbase + off), "r"(x), "r"(y),
                         "r"(z), "r"(q)
                         : "memory");
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tm_out, sbase, w.tq * BNQ + half * kHalf + box * 64, w.tp * BM + quad * 32);
            bulk_commit_group();
          }
        }
      }
    }
    if (!SWAP && lane == 0) bulk_wait_group0();
  }
  __syncwarp();

  // -------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace bsg
