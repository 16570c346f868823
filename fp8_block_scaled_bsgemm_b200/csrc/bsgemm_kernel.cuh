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
//   warps 1-2 MMA issuers (warp 1 also owns TMEM), taking the K-blocks in
//            turn: tcgen05.mma (kind::f8f6f4, K = 32 per instruction) into
//            one of 2..8 TMEM partial buffers, then tcgen05.commit to tell
//            the promoters;
//   warp 3   stream-K publisher: releases the CTA's one partial that another
//            CTA reduces (idle otherwise);
//   warps 4-11 promotion + epilogue: tcgen05.ld each K-block's partial,
//            acc += (sP*sQ) * partial in FP32 registers (packed f32x2 FMAs),
//            release the TMEM buffer, and at the end of a tile round to BF16
//            and store it: through shared memory and a TMA bulk tensor store
//            for data-parallel tiles, straight from registers otherwise.
// Work is split three ways:
//   whole tiles (data-parallel), walked by the persistent CTAs in raster order;
//   split-K: every tile's K-blocks cut into `splits` equal pieces;
//   stream-K: after the full waves of whole tiles, the remaining tiles'
//     K-blocks, laid end to end, are cut into equal contiguous ranges, one
//     per CTA, so no SM idles in a ragged last wave.
// A piece that is not a whole tile writes its FP32 partial tile to a
// workspace slot and arrives on a per-tile counter; the tile's reducer (for
// split-K the last piece to arrive, for stream-K the piece that starts the
// tile, which keeps its own partial in registers) adds all the tile's
// partials in K order -- the same order every run -- and stores the BF16 tile.
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
constexpr int kProducerRegs = 56;
constexpr int kPromoteRegs = 224;
static_assert(kProducerRegs * 128 + kPromoteRegs * 256 <= kLaunchRegs * kNumThreads,
              "register split exceeds the launch allocation");

template <int BNQ>
struct RegSplit {
  static constexpr bool kEnabled = (BNQ == 256);
};

struct Params {
  int M, N, K;           // logical GEMM sizes
  int Kb;                // ceil(K / gran)
  int Pb, Qb;            // ceil(P / gran), ceil(Q / gran)
  int tiles_p, tiles_q;  // tiles along P (128 rows) and along Q (BNQ rows)
  int splits;            // K splits per tile (1 = none)
  int kb_per_split;      // K-blocks per split (even when gran == 64)
  int num_work;          // whole-tile or split-K work items: tiles before sk_first_tile, times splits
  int sk_first_tile;     // stream-K: first tile handled by stream-K (tiles before it are whole)
  int sk_units_per_tile; // stream-K: units (K-blocks; pairs of K-blocks when gran == 64) per tile
  int sk_ctas;           // stream-K: CTAs sharing the stream-K units (0 = no stream-K)
  int sk_q, sk_r;        // stream-K: the stream-K units number sk_q * sk_ctas + sk_r; the first
                         // sk_r CTAs take sk_q + 1 of them, the others sk_q
  int group_p;           // raster group height in P tiles (L2 locality)
  uint32_t fmt_bits;     // instruction-descriptor format fields of P and Q (E4M3 0, E5M2 1)
  int epi;               // epilogue: activation (bits 0-1: 0 none, 1 ReLU, 2 GELU), bit 2 FP32 output
  int num_groups;        // grouped GEMM: number of groups (0 otherwise)
  const float* bias;     // FP32 [N] added before the activation, or null
  const int* group_m;    // grouped GEMM: rows of each group (device, num_groups entries)
  const float* sP;       // [Pb][Kb]
  const float* sQ;       // [Qb][Kb]
  __nv_bfloat16* out;    // [M][N] row-major, BF16 (FP32 when epi bit 2 is set)
  float* ws;             // partial tiles [slot][BNQ/4][BM][4]: split-K slot tile*splits+split,
                         // stream-K slot 2*cta + (0: the CTA's first tile, 1: its last)
  int* counters;         // one per split or stream-K tile, zero between launches
  int* status;           // device status word
  unsigned long long timeout_ns;
};

template <int BNQ, bool Q_MN>
struct Tiles {
  static constexpr int kPBytes = BM * BK;                                // 16 KB
  static constexpr int kQRows = (Q_MN && BNQ < 128) ? 128 : BNQ;         // MN-major: 128-wide atom
  static constexpr int kQBytes = kQRows * BK;
};

// Epilogue staging for the TMA store: each promotion warp owns one buffer of
// 32 rows x 128 bytes (64 BF16 or 32 FP32 columns), in the 128-byte swizzled
// layout of the output tensor map.
constexpr int kEpiChunkBytes = 32 * 128;

template <int BNQ, bool Q_MN, bool SWAP, bool GROUPED = false>
struct StageCfg {
  static constexpr int kStageBytes = Tiles<BNQ, Q_MN>::kPBytes + Tiles<BNQ, Q_MN>::kQBytes;
  // Data-parallel tiles store through TMA from a per-warp staging buffer.
  // Swap-AB tiles stage the whole BF16 tile, transposed to the output's
  // [M][N] order ([BNQ][128] BF16), and store it with one TMA copy (their FP32
  // output stores from registers).  Grouped tiles (a tile may end inside the
  // next group's rows) store straight from registers.
  static constexpr bool kTmaStore = !SWAP && !GROUPED;
  static constexpr bool kSwapTmaStore = SWAP;
  static constexpr int kEpiBytes = kTmaStore ? kNumEpiWarps * kEpiChunkBytes : (SWAP ? BNQ * BM * 2 : 0);
  static constexpr int kBudget = 227 * 1024 - 1024 /*align slack*/ - 512 /*barriers*/;
  static constexpr int kStagesRaw = (kBudget - kEpiBytes) / kStageBytes;
  static constexpr int kStages = kStagesRaw > 8 ? 8 : kStagesRaw;
  static_assert(kStages >= 2, "shared memory too small for two stages");
  static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + kEpiBytes + 512;
};

struct __align__(8) Barriers {
  uint64_t full[8];
  uint64_t empty[8];
  uint64_t tmem_full[8];
  uint64_t tmem_empty[8];
  uint64_t mma_done;
  uint64_t publish;      // stream-K: the promotion warps' partial is written
  uint32_t tmem_base;
  int abort_flag;
  int split_last;
  // per promotion warp: the current work item's Pieces (pieces, slot,
  // counter, slot0, slot_base, slot_step), parked here for the K-loop
  int pieces[kNumEpiWarps][6];
};
static_assert(sizeof(Barriers) <= 512, "barrier block is 512 bytes");

// ---------------------------------------------------------------- helpers
__device__ __forceinline__ void record_timeout(const Params& p, Barriers* bars, int where) {
  *reinterpret_cast<volatile int*>(&bars->abort_flag) = 1;
  atomicCAS(p.status, 0, kTimeoutCode | (where << 8));
}

// Bounded mbarrier wait. Returns false on timeout or when another warp of the
// CTA has raised the abort flag (unless ignore_abort).  Waiters that are not
// on the critical path pass a backoff so that their polling does not crowd
// the barrier unit that the critical hand-offs go through.
template <int kBackoffNs = 0>
__device__ __forceinline__ bool bounded_wait(uint32_t bar, uint32_t parity, const Params& p,
                                          Barriers* bars, int where, bool ignore_abort = false) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i) {
      if (mbar_try_wait(bar, parity)) return true;
      if constexpr (kBackoffNs > 0) __nanosleep(kBackoffNs);
    }
    if (!ignore_abort && *reinterpret_cast<volatile int*>(&bars->abort_flag)) return false;
    if (globaltimer_ns() - t0 > p.timeout_ns) {
      if (!ignore_abort) record_timeout(p, bars, where);
      return false;
    }
  }
}

// Bounded wait of one thread until the counter at `ctr` reaches `target`,
// with acquire semantics at GPU scope (the publishers' stores before their
// release adds are visible afterwards).  Returns false on timeout (recorded)
// or when another warp of the CTA raised the abort flag.
__device__ __forceinline__ bool wait_counter_acquire(const Params& p, Barriers* bars, const int* ctr,
                                                     int target, int where) {
  if (ld_acquire_gpu(ctr) >= target) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i) {
      __nanosleep(64);
      if (ld_acquire_gpu(ctr) >= target) return true;
    }
    if (*reinterpret_cast<volatile int*>(&bars->abort_flag)) return false;
    if (globaltimer_ns() - t0 > p.timeout_ns) {
      record_timeout(p, bars, where);
      return false;
    }
  }
}

// Bounded wait run by every lane of a converged warp; the answer is made
// warp-uniform (a lane whose deadline ran out makes the whole warp give up),
// so the warp stays converged.
__device__ __forceinline__ bool warp_wait_all(uint32_t bar, uint32_t parity, const Params& p,
                                              Barriers* bars, int where, bool ignore_abort = false) {
  const bool ok = bounded_wait(bar, parity, p, bars, where, ignore_abort);
  return __all_sync(0xffffffffu, ok);
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

// Instruction descriptor: kind::f8f6f4, D = F32, M = 128, N = BNQ; the A and B
// format fields (bits 7-9, 10-12: E4M3 0, E5M2 1) come from Params.fmt_bits.
template <int BNQ, bool P_MN, bool Q_MN>
__device__ __forceinline__ constexpr uint32_t instr_desc() {
  return (1u << 4)                               // D format: F32
         | (0u << 7) | (0u << 10)                // A, B format: or-ed in at run time
         | ((P_MN ? 1u : 0u) << 15)              // A major (0 = K)
         | ((Q_MN ? 1u : 0u) << 16)              // B major
         | (static_cast<uint32_t>(BNQ >> 3) << 17)
         | (static_cast<uint32_t>(BM >> 4) << 24);
}

struct Work {
  int tile, tp, tq, kb0, kb1;  // output tile and its K-blocks [kb0, kb1)
  // grouped GEMM (zero / unused otherwise): the group's first row in A, out
  // and its first scale row in sA, its first row in B and in sB, its rows
  int g_row, g_srow, g_qrow, g_sqrow, g_rows;
};

// Tile index -> (P tile, Q tile) in grouped raster order: group_p P-tiles
// down, then across Q, so concurrently running CTAs share operand tiles in L2.
__device__ __forceinline__ void tile_coords(const Params& p, int tile, int& tp, int& tq) {
  const int per_group = p.group_p * p.tiles_q;
  const int grp = tile / per_group;
  const int first_p = grp * p.group_p;
  int rows = p.tiles_p - first_p;
  rows = rows < p.group_p ? rows : p.group_p;
  const int local = tile - grp * per_group;
  tp = first_p + local % rows;
  tq = local / rows;
}

// Stream-K: CTA c owns units [sk_start(c), sk_start(c + 1)); the first sk_r
// CTAs take sk_q + 1 units, the others sk_q (32-bit arithmetic throughout).
// A unit is one K-block, or two (one 128-deep stage) when gran == 64.
__device__ __forceinline__ int sk_start(const Params& p, int c) {
  return c * p.sk_q + min(c, p.sk_r);
}
// The CTA whose range holds unit u.
__device__ __forceinline__ int sk_owner(const Params& p, int u) {
  const int split = p.sk_r * (p.sk_q + 1);  // units held by the CTAs with one extra unit
  return u < split ? u / (p.sk_q + 1) : p.sk_r + (u - split) / p.sk_q;
}

// Every role of a CTA walks the same sequence of work items: first its whole
// tiles or split-K pieces (blockIdx.x, +gridDim.x, ...), then the segments of
// its stream-K range, one per tile the range touches.
struct WorkIter {
  int wi;  // next whole-tile / split-K item
  int u;   // next stream-K unit
  // grouped GEMM cursor: current group, its first tile, rows, tiles, first
  // row and first scale row
  int g, g_first, g_m, g_tiles, g_row, g_srow;
};

// Grouped GEMM: advance the cursor to the group that holds tile it.wi (tiles
// are numbered group by group; each group has ceil(rows / 128) x tiles_q).
// Returns false once every group is used up.
template <int GRAN>
__device__ __forceinline__ bool group_seek(const Params& p, WorkIter& it) {
  while (it.wi >= it.g_first + it.g_tiles) {
    it.g_first += it.g_tiles;
    it.g_row += it.g_m;
    it.g_srow += (it.g_m + GRAN - 1) / GRAN;
    if (++it.g >= p.num_groups) return false;
    it.g_m = max(0, __ldg(p.group_m + it.g));
    it.g_tiles = (it.g_m + BM - 1) / BM * p.tiles_q;
  }
  return true;
}

template <bool SPLIT, bool GROUPED = false>
__device__ __forceinline__ void work_begin(const Params& p, WorkIter& it) {
  it.wi = blockIdx.x;
  it.u = 0;
  if (SPLIT && static_cast<int>(blockIdx.x) < p.sk_ctas) it.u = sk_start(p, blockIdx.x);
  if constexpr (GROUPED) {
    it.g = 0;
    it.g_first = 0;
    it.g_row = 0;
    it.g_srow = 0;
    it.g_m = max(0, __ldg(p.group_m));
    it.g_tiles = (it.g_m + BM - 1) / BM * p.tiles_q;
  }
}

// Instances without the partial-tile fix-up (SPLIT false) never get a
// stream-K range, so their walk is the whole-tile loop alone.
template <int GRAN, bool SPLIT, bool GROUPED = false>
__device__ __forceinline__ bool work_next(const Params& p, WorkIter& it, Work& w) {
  if constexpr (GROUPED) {
    // whole tiles, group by group; within a group the P (row) tile varies
    // fastest, so CTAs running together share the group's B tiles
    if (!group_seek<GRAN>(p, it)) return false;
    const int lt = it.wi - it.g_first;
    const int tiles_p = (it.g_m + BM - 1) / BM;
    w.tile = it.wi;
    w.tp = lt % tiles_p;
    w.tq = lt / tiles_p;
    w.kb0 = 0;
    w.kb1 = p.Kb;
    w.g_row = it.g_row;
    w.g_srow = it.g_srow;
    w.g_qrow = it.g * p.N;
    w.g_sqrow = it.g * p.Qb;
    w.g_rows = it.g_m;
    it.wi += gridDim.x;
    return true;
  }
  if (it.wi < p.num_work) {
    w.tile = it.wi / p.splits;
    const int split = it.wi - w.tile * p.splits;
    tile_coords(p, w.tile, w.tp, w.tq);
    w.kb0 = split * p.kb_per_split;
    w.kb1 = min(p.Kb, w.kb0 + p.kb_per_split);
    it.wi += gridDim.x;
    return true;
  }
  if constexpr (SPLIT) {
    const int bid = static_cast<int>(blockIdx.x);
    const int u_end = bid < p.sk_ctas ? sk_start(p, bid + 1) : 0;
    if (it.u < u_end) {
      constexpr int kUnitKb = GRAN == 64 ? 2 : 1;
      const int U = p.sk_units_per_tile;
      const int t_local = it.u / U;
      const int tile_u0 = t_local * U;
      const int seg_end = min(u_end, tile_u0 + U);
      w.tile = p.sk_first_tile + t_local;
      tile_coords(p, w.tile, w.tp, w.tq);
      w.kb0 = (it.u - tile_u0) * kUnitKb;
      w.kb1 = min(p.Kb, (seg_end - tile_u0) * kUnitKb);
      it.u = seg_end;
      return true;
    }
  }
  return false;
}

// Where a work item's partial goes and where its tile's other pieces are,
// from the item alone.
struct Pieces {
  int pieces;   // pieces the tile is cut into (1: the item is the whole tile)
  int slot;     // workspace slot of this item's partial
  int counter;  // arrival counter of the tile
  // slots of the tile's pieces in K order: piece 0 in slot0, piece j > 0 in
  // slot_base + j * slot_step
  int slot0, slot_base, slot_step;
};

template <int GRAN>
__device__ __forceinline__ Pieces pieces_of(const Params& p, const Work& w) {
  Pieces r;
  if (p.sk_ctas == 0 || w.tile < p.sk_first_tile) {
    // whole tile or split-K piece
    r.pieces = p.splits;
    r.counter = w.tile;
    r.slot0 = r.slot_base = w.tile * p.splits;
    r.slot_step = 1;
    r.slot = r.slot_base + w.kb0 / p.kb_per_split;
    return r;
  }
  // stream-K segment.  A CTA's partial pieces are the first and the last
  // segment of its range: slot 2c for its first, 2c + 1 for its last.  Piece
  // j > 0 of a tile starts its CTA's range (slot 2c); piece 0 is its CTA's
  // first segment only if that CTA's range starts at the tile's first unit.
  constexpr int kUnitKb = GRAN == 64 ? 2 : 1;
  const int U = p.sk_units_per_tile;
  const int t_local = w.tile - p.sk_first_tile;
  const int tile_u0 = t_local * U;
  const int bid = static_cast<int>(blockIdx.x);
  r.counter = t_local;
  r.pieces = 1;
  r.slot = r.slot0 = r.slot_base = 0;
  r.slot_step = 2;
  if (w.kb0 != 0 || w.kb1 != p.Kb) {
    const int first_cta = sk_owner(p, tile_u0);
    r.pieces = sk_owner(p, tile_u0 + U - 1) - first_cta + 1;
    r.slot = 2 * bid + (tile_u0 + w.kb0 / kUnitKb == sk_start(p, bid) ? 0 : 1);
    r.slot_base = 2 * first_cta;
    r.slot0 = r.slot_base + (sk_start(p, first_cta) < tile_u0 ? 1 : 0);
  }
  return r;
}

__device__ __forceinline__ int piece_slot(const Pieces& pc, int j) {
  return j == 0 ? pc.slot0 : pc.slot_base + j * pc.slot_step;
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

// ---------------------------------------------------------------- epilogue
// out = act(acc + bias[n]), the pages' fused-epilogue extension point
// (hncyxsy.com/news/191052 §2.3, §6). GELU is the erf form,
// 0.5 v (1 + erf(v / sqrt 2)).
constexpr int kEpiRelu = 1, kEpiGelu = 2, kEpiOutF32 = 4;

__device__ __forceinline__ float epi_act(float v, int act) {
  if (act == kEpiRelu) return fmaxf(v, 0.f);
  if (act == kEpiGelu) return 0.5f * v * (1.0f + erff(v * 0.70710678118654752f));
  return v;
}

template <int ACT>
__device__ __forceinline__ float epi_act_t(float v) {
  if constexpr (ACT == kEpiRelu) return fmaxf(v, 0.f);
  if constexpr (ACT == kEpiGelu) return 0.5f * v * (1.0f + erff(v * 0.70710678118654752f));
  return v;
}

template <int V>
struct ActTag {
  static constexpr int value = V;
};

// Calls f(ActTag<ACT>{}) for the run-time activation code, so loops over
// elements are instantiated per activation and never carry the other
// activations' code (evaluated per element, the erf path cost ~90 cycles a
// value even when the activation was none).
template <typename F>
__device__ __forceinline__ void with_act(int act, F&& f) {
  if (act == kEpiGelu) f(ActTag<kEpiGelu>{});
  else if (act == kEpiRelu) f(ActTag<kEpiRelu>{});
  else f(ActTag<0>{});
}

// out = act(acc + bias[n]) in place on one thread's run of columns
// [n0, n0 + 2 * NP) (acc pairs in column order).
template <int NP>
__device__ __forceinline__ void apply_epi(const Params& p, int n0, float2 (&acc)[NP]) {
  const int act = p.epi & 3;
  if (p.bias != nullptr || act != 0) {
#pragma unroll
    for (int i = 0; i < NP; ++i) {
      const int n = n0 + 2 * i;
      float b0 = 0.f, b1 = 0.f;
      if (p.bias != nullptr && n < p.N) {
        b0 = __ldg(p.bias + n);
        b1 = __ldg(p.bias + n + 1);
      }
      acc[i].x = epi_act(acc[i].x + b0, act);
      acc[i].y = epi_act(acc[i].y + b1, act);
    }
  }
}

__device__ __forceinline__ void st_shared_b16(uint32_t addr, unsigned short v) {
  asm volatile("st.shared.b16 [%0], %1;" ::"r"(addr), "h"(v) : "memory");
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(x), "r"(y), "r"(z), "r"(w)
               : "memory");
}

// TMA-store epilogue of one promotion warp: lane l holds row m0 + l, columns
// [n0, n0 + 2 * NP) (acc pairs in column order, epilogue already applied).
// The warp's rows go out in chunks of 128 bytes per row (64 BF16 or 32 FP32
// columns): every lane writes its row of the chunk into the warp's staging
// buffer -- 16-byte piece u of row l at l * 128 + ((u ^ (l % 8)) * 16), the
// tensor map's 128-byte swizzle, so a warp's store touches every bank evenly
// -- then one lane issues the bulk tensor store.  The tensor map clips rows
// past M and columns past N.  Before a buffer is rewritten, the store that
// read it must have finished reading (cp.async.bulk.wait_group.read).
template <int NP>
__device__ __forceinline__ void store_tile_tma(const Params& p, const CUtensorMap* tm_out,
                                               uint32_t buf, int m0, int n0, float2 (&acc)[NP],
                                               uint32_t lane) {
  const uint32_t row = buf + lane * 128;
  const uint32_t sw = lane & 7;
  if (m0 >= p.M) return;  // the warp's rows are all past the end
  if (!(p.epi & kEpiOutF32)) {
    static_assert((2 * NP) % 64 == 0, "BF16 chunks of 64 columns");
#pragma unroll
    for (int c = 0; c < 2 * NP / 64; ++c) {
      if (n0 + c * 64 < p.N) {
        if (lane == 0) bulk_wait_group_read0();
        __syncwarp();
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int i = c * 32 + 4 * u;
          st_shared_v4(row + ((u ^ sw) << 4), pack_bf16x2(acc[i].x, acc[i].y),
                       pack_bf16x2(acc[i + 1].x, acc[i + 1].y), pack_bf16x2(acc[i + 2].x, acc[i + 2].y),
                       pack_bf16x2(acc[i + 3].x, acc[i + 3].y));
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(tm_out, buf, n0 + c * 64, m0);
          bulk_commit_group();
        }
      }
    }
  } else {
    static_assert((2 * NP) % 32 == 0, "FP32 chunks of 32 columns");
#pragma unroll
    for (int c = 0; c < 2 * NP / 32; ++c) {
      if (n0 + c * 32 < p.N) {
        if (lane == 0) bulk_wait_group_read0();
        __syncwarp();
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int i = c * 16 + 2 * u;
          st_shared_v4(row + ((u ^ sw) << 4), __float_as_uint(acc[i].x), __float_as_uint(acc[i].y),
                       __float_as_uint(acc[i + 1].x), __float_as_uint(acc[i + 1].y));
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(tm_out, buf, n0 + c * 32, m0);
          bulk_commit_group();
        }
      }
    }
  }
}

// One thread's run of columns [n0, n0 + 2 * NP) of row m: acc pairs in
// column order. Applies the epilogue in place and stores BF16 (8 per 16-byte
// store) or FP32 (4 per 16-byte store); N % 8 == 0, so a group of 8 columns
// is wholly inside or outside the matrix.
template <int NP>
__device__ __forceinline__ void store_row_run(const Params& p, int m, int n0, float2 (&acc)[NP]) {
  apply_epi(p, n0, acc);
  if (p.epi & kEpiOutF32) {
    float* row = reinterpret_cast<float*>(p.out) + static_cast<size_t>(m) * p.N + n0;
#pragma unroll
    for (int c = 0; c < NP / 2; ++c)
      if (n0 + c * 4 < p.N)
        *reinterpret_cast<float4*>(row + c * 4) =
            make_float4(acc[2 * c].x, acc[2 * c].y, acc[2 * c + 1].x, acc[2 * c + 1].y);
  } else {
    __nv_bfloat16* row = p.out + static_cast<size_t>(m) * p.N + n0;
#pragma unroll
    for (int c = 0; c < NP / 4; ++c) {
      if (n0 + c * 8 < p.N) {
        uint4 v;
        v.x = pack_bf16x2(acc[c * 4].x, acc[c * 4].y);
        v.y = pack_bf16x2(acc[c * 4 + 1].x, acc[c * 4 + 1].y);
        v.z = pack_bf16x2(acc[c * 4 + 2].x, acc[c * 4 + 2].y);
        v.w = pack_bf16x2(acc[c * 4 + 3].x, acc[c * 4 + 3].y);
        *reinterpret_cast<uint4*>(row + c * 8) = v;
      }
    }
  }
}

// ---------------------------------------------------------------- kernel
template <int BNQ, int GRAN, bool SWAP, bool P_MN, bool Q_MN, bool SPLIT, bool GROUPED = false>
__global__ void __launch_bounds__(kNumThreads, 1)
    bsgemm_kernel(const __grid_constant__ CUtensorMap tm_p, const __grid_constant__ CUtensorMap tm_q,
                  const __grid_constant__ CUtensorMap tm_out, const Params p) {
  using TL = Tiles<BNQ, Q_MN>;
  using SC = StageCfg<BNQ, Q_MN, SWAP, GROUPED>;
  constexpr int STAGES = SC::kStages;
  constexpr int kHalf = BNQ / 2;                      // columns per promotion warp
  constexpr int kNumGroups = (kHalf > GRAN) ? kHalf / GRAN : 1;  // scale groups per warp
  constexpr int kGroupCols = kHalf / kNumGroups;
  // TMEM partial buffers: as many as fit (up to 8) so the MMA can run ahead of
  // the promotion warps; 512 columns hold 2 x 256, 4 x 128 or 8 x 64.
  constexpr int kBufs = (BNQ >= 256) ? 2 : (BNQ >= 128) ? 4 : 8;
  constexpr uint32_t kTmemCols = (kBufs * BNQ <= 32) ? 32 : (kBufs * BNQ <= 64) ? 64
                                : (kBufs * BNQ <= 128) ? 128 : (kBufs * BNQ <= 256) ? 256 : 512;
  static_assert(kBufs * BNQ <= 512, "TMEM holds 512 columns");
  // Two MMA-issuing warps take the K-blocks in turn (issuer x % 2 takes the
  // CTA's K-block x, counted over all its work items).  One warp issues a
  // tcgen05.mma about every 80 cycles whatever its N (measured on B200), and
  // each barrier wait and commit adds to that, so one warp alone leaves the
  // tensor core idle between narrow instructions.  Parity waits are only
  // sound when a waiter observes every phase of its barrier in turn, so:
  // - every TMEM buffer belongs to one issuer (kBufs even, x % kBufs);
  // - at g = 128 a K-block is one stage, so with an even number of stages
  //   every stage belongs to one issuer, which alone releases it;
  // - otherwise stages change hands (g = 64: a stage holds blocks x and
  //   x + 1; g = 256: a block is two stages, or one at the K tail; an odd
  //   ring, as in the grouped 128-wide tiles' seven stages), and both
  //   issuers wait for every stage and release it: the owner after its MMAs,
  //   the other by a commit of no MMAs.  Having waited for the stage's fill,
  //   whose phase the previous release completed, neither release can land
  //   in an earlier phase.
  constexpr int kIssuers = 2;
  constexpr bool kSharedStages = (GRAN != BK) || (STAGES % kIssuers != 0);
  constexpr int kStageUsers = kSharedStages ? 2 : 1;
  static_assert(kBufs % kIssuers == 0, "TMEM buffers split evenly between the issuers");
  constexpr uint32_t kTxBytes = TL::kPBytes + TL::kQBytes;
  static_assert(BNQ % 16 == 0 && BNQ >= 16 && BNQ <= 256, "MMA N must be a multiple of 16 in [16, 256]");
  static_assert(GRAN == 64 || GRAN == 128 || GRAN == 256, "granularity");
  static_assert(kHalf % 8 == 0, "columns per warp");
  static_assert(SWAP || kHalf % 8 == 0, "the epilogue stores 8 BF16 columns at a time");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* p_tiles = smem;
  uint8_t* q_tiles = smem + STAGES * TL::kPBytes;
  uint8_t* epi_bufs = q_tiles + STAGES * TL::kQBytes;  // 1024-aligned: stage sizes are multiples of 1 KB
  Barriers* bars = reinterpret_cast<Barriers*>(epi_bufs + SC::kEpiBytes);

  const int warp = threadIdx.x / 32;
  const uint32_t lane = lane_id();

  // -------------------------------------------------------------- setup
  // Warp 2 (otherwise idle) initialises the barriers and warp 1 allocates
  // TMEM, while the producer prefetches the tensor maps and works out its
  // first work item (integer divisions: ~1000 cycles of one thread), so its
  // first TMA load issues right after the set-up barrier.
  if (warp == 2 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_addr(&bars->full[s]), 1);
      mbar_init(smem_addr(&bars->empty[s]), kStageUsers);
    }
    for (int b = 0; b < kBufs; ++b) {
      mbar_init(smem_addr(&bars->tmem_full[b]), 1);
      mbar_init(smem_addr(&bars->tmem_empty[b]), kNumEpiWarps);
    }
    mbar_init(smem_addr(&bars->mma_done), kIssuers);
    mbar_init(smem_addr(&bars->publish), kNumEpiWarps);
    bars->abort_flag = 0;
    bars->split_last = 0;
    fence_barrier_init();
  }
  WorkIter pwit;        // the producer's work cursor and first item
  Work pw;
  bool pmore = false;
  if (warp == kProducerWarp && lane == 0) {
    tma_prefetch_desc(&tm_p);
    tma_prefetch_desc(&tm_q);
    // the output map exists for data-parallel tiles and for BF16 swap-AB tiles
    if constexpr (SC::kTmaStore) tma_prefetch_desc(&tm_out);
    if constexpr (SC::kSwapTmaStore) {
      if (!(p.epi & kEpiOutF32)) tma_prefetch_desc(&tm_out);
    }
    if constexpr (!GROUPED) {
      // from the launch parameters alone: no global memory
      work_begin<SPLIT, GROUPED>(p, pwit);
      pmore = work_next<GRAN, SPLIT, GROUPED>(p, pwit, pw);
    }
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_addr(&bars->tmem_base), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = bars->tmem_base;
  // Programmatic dependent launch: everything above (barriers, TMEM, the
  // tensor-map prefetch) and the producer's first work item touch no global
  // memory, so they may overlap the previous grid's last CTAs.  The producer
  // and the promotion warps -- the only roles that read or write global
  // memory (operands, scales, workspace, output) -- wait for that grid
  // (grid_dependency_wait) first, and so does the stream-K publisher; the MMA
  // issuers touch only shared memory and TMEM.  The next grid may start its
  // own set-up as soon as SMs free up.
  if (threadIdx.x == 0) grid_launch_dependents();

  if (warp < kFirstEpiWarp) {
    // warpgroup 0: producer, two MMA issuers and the stream-K publisher
    if constexpr (RegSplit<BNQ>::kEnabled) set_max_regs_dec<kProducerRegs>();
  if (warp == kProducerWarp) {
    // ============================================================ TMA producer
    if (lane == 0) {
      uint32_t it = 0;  // stage-slot uses so far
      bool ok = true;
      WorkIter gwit;      // grouped: the cursor starts after the wait
      Work gw;
      WorkIter& wit = GROUPED ? gwit : pwit;
      Work& w = GROUPED ? gw : pw;
      bool more = pmore;
      if constexpr (GROUPED) {
        // the grouped work list reads the group sizes from global memory
        grid_dependency_wait();
        work_begin<SPLIT, GROUPED>(p, wit);
        more = work_next<GRAN, SPLIT, GROUPED>(p, wit, w);
      } else {
        // While the previous grid finishes, pull the first ring's worth of
        // this CTA's operand tiles towards L2.  A prefetch returns nothing to
        // the program and L2 is coherent, so the loads after the wait still
        // read what the previous grid wrote; they find the bytes nearer.
        if (more) {
          int st0, st1;
          stage_range<GRAN>(p, w, st0, st1);
          const int stop = st1 < st0 + STAGES ? st1 : st0 + STAGES;
          const int prow = w.tp * BM, qrow = w.tq * BNQ;
          for (int st = st0; st < stop; ++st) {
            const int k = st * BK;
            if constexpr (P_MN) tma_prefetch_l2_2d(&tm_p, prow, k);
            else                tma_prefetch_l2_2d(&tm_p, k, prow);
            if constexpr (Q_MN) {
#pragma unroll
              for (int c = 0; c < TL::kQRows / 128; ++c) tma_prefetch_l2_2d(&tm_q, qrow + c * 128, k);
            } else {
              tma_prefetch_l2_2d(&tm_q, k, qrow);
            }
          }
        }
        grid_dependency_wait();
      }
      for (; ok && more; more = work_next<GRAN, SPLIT, GROUPED>(p, wit, w)) {
        int st0, st1;
        stage_range<GRAN>(p, w, st0, st1);
        for (int st = st0; st < st1; ++st, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!bounded_wait<32>(smem_addr(&bars->empty[s]), ph ^ 1, p, bars, 1)) { ok = false; break; }
          const uint32_t fb = smem_addr(&bars->full[s]);
          mbar_arrive_expect_tx(fb, kTxBytes);
          const uint32_t pd = smem_addr(p_tiles + s * TL::kPBytes);
          const uint32_t qd = smem_addr(q_tiles + s * TL::kQBytes);
          const int k = st * BK;
          const int prow = (GROUPED ? w.g_row : 0) + w.tp * BM;
          const int qrow = (GROUPED ? w.g_qrow : 0) + w.tq * BNQ;
          if constexpr (P_MN) tma_load_2d(pd, &tm_p, fb, prow, k);
          else                tma_load_2d(pd, &tm_p, fb, k, prow);
          if constexpr (Q_MN) {
#pragma unroll
            for (int c = 0; c < TL::kQRows / 128; ++c)
              tma_load_2d(qd + c * 128 * BK, &tm_q, fb, qrow + c * 128, k);
          } else {
            tma_load_2d(qd, &tm_q, fb, k, qrow);
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
  } else if (warp == kMmaWarp || warp == kMmaWarp + 1) {
    // ============================================================ MMA issuers
    // Issuer i (warp kMmaWarp + i) takes the K-blocks of parity i, in K
    // order: it claims the block's TMEM buffer, issues the block's MMAs
    // (K = 32 each) stage by stage -- waiting for a stage at its first k-step,
    // releasing it after its last -- and commits the buffer to the promotion
    // warps after the block's last MMA (the promotion of block x gates the
    // MMAs of block x + kBufs).  Both issuers walk every work item and stage,
    // so the stage ring and the K-block counter (buffer x % kBufs) agree
    // between them, the producer and the promotion warps.  A commit tracks
    // the MMAs of its own thread only, so the issuers' commits are
    // independent.  Each warp runs converged: every lane polls the barriers,
    // descriptors are warp-uniform, and each tcgen05 instruction is
    // predicated on elect.sync, so one lane (always the same) issues it.
    {
      const uint32_t issuer = static_cast<uint32_t>(warp - kMmaWarp);
      const uint32_t idesc = instr_desc<BNQ, P_MN, Q_MN>() | p.fmt_bits;
      // descriptor steps: per k-step of 32 (K-major +32 B, MN-major +32 rows
      // of 128 B) and per pipeline stage, in the descriptor's 16-byte units
      constexpr uint64_t kPStep = P_MN ? (kMmaK * 128) >> 4 : kMmaK >> 4;
      constexpr uint64_t kQStep = Q_MN ? (kMmaK * 128) >> 4 : kMmaK >> 4;
      constexpr uint64_t kPStage = TL::kPBytes >> 4, kQStage = TL::kQBytes >> 4;
      const uint64_t ad0 = smem_desc_sw128(smem_addr(p_tiles), P_MN ? 128 * BK : 16);
      const uint64_t bd0 = smem_desc_sw128(smem_addr(q_tiles), Q_MN ? 128 * BK : 16);
      uint32_t s = 0, ph = 0;     // pipeline stage and its phase
      uint32_t x = 0;             // K-blocks so far
      bool ok = true;
      WorkIter wit;
      // the grouped work list reads the group sizes from global memory
      if constexpr (GROUPED) grid_dependency_wait();
      work_begin<SPLIT, GROUPED>(p, wit);
      for (Work w; ok && work_next<GRAN, SPLIT, GROUPED>(p, wit, w);) {
        for (int kb = w.kb0; kb < w.kb1; ++kb, ++x) {
          // Order of the waits: the stage's operands first (normally already
          // loaded, so that wait is cheap), then the TMEM buffer, which gates
          // the MMAs; the promotion warps arrive on tmem_empty only after
          // tcgen05.wait::ld, so their reads of the buffer are complete
          // before it is overwritten.  Commits: tmem_full first (the
          // promotion warps wait on it), then the stage release.
          const uint32_t b = x % kBufs, bph = (x / kBufs) & 1;
          const uint32_t d_tmem = tmem_base + b * BNQ;
          if constexpr (GRAN >= BK) {
            // whole stages: GRAN / 128 of them, 4 k-steps each (fewer at the K tail)
            const bool mine = (x & 1) == issuer;
#pragma unroll
            for (int j = 0; j < GRAN / BK; ++j) {
              const int k0 = kb * GRAN + j * BK;
              if (k0 >= p.K) break;
              if (!mine && kSharedStages) {
                // the other issuer's stage: observe its fill and release it
                // (a commit of no MMAs: it follows this issuer's own MMAs)
                if (!warp_wait_all(smem_addr(&bars->full[s]), ph, p, bars, 2)) { ok = false; break; }
                mma_commit_elect(smem_addr(&bars->empty[s]));
              }
              if (mine) {
                // TMA writes and MMA reads are async-proxy accesses ordered by this barrier
                if (!warp_wait_all(smem_addr(&bars->full[s]), ph, p, bars, 2)) { ok = false; break; }
                if (j == 0 && !warp_wait_all(smem_addr(&bars->tmem_empty[b]), bph ^ 1, p, bars, 3)) {
                  ok = false;
                  break;
                }
                const uint64_t ad = ad0 + s * kPStage, bd = bd0 + s * kQStage;
                if (k0 + BK <= p.K) {
#pragma unroll
                  for (int t = 0; t < BK / kMmaK; ++t)
                    mma_f8f6f4_elect(d_tmem, ad + t * kPStep, bd + t * kQStep, idesc, (j > 0 || t > 0) ? 1u : 0u);
                } else {
                  const int nsteps = (p.K - k0 + kMmaK - 1) / kMmaK;
                  for (int t = 0; t < nsteps; ++t)
                    mma_f8f6f4_elect(d_tmem, ad + t * kPStep, bd + t * kQStep, idesc, (j > 0 || t > 0) ? 1u : 0u);
                }
                if (j == GRAN / BK - 1 || k0 + BK >= p.K) mma_commit_elect(smem_addr(&bars->tmem_full[b]));
                mma_commit_elect(smem_addr(&bars->empty[s]));  // stage free once these MMAs finish
              }
              if (++s == STAGES) { s = 0; ph ^= 1; }
            }
            if (!ok) break;
          } else {
            // GRAN == 64: a K-block is half a stage (work items start on even
            // K-blocks, so a stage holds consecutive blocks x and x + 1, one
            // per issuer) and each issuer releases the stage after its half.
            // Where the K tail leaves a stage without its second half, the
            // other issuer waits for it and releases it all the same.
            const int k0 = kb * GRAN;
            const int t0 = (kb & 1) * 2;
            const bool last_in_stage = (t0 == 2 || k0 + GRAN >= p.K);
            if ((x & 1) == issuer) {
              // (a stage's two halves belong to different issuers, so each
              // issuer waits for every stage once)
              if (!warp_wait_all(smem_addr(&bars->full[s]), ph, p, bars, 2)) { ok = false; break; }
              if (!warp_wait_all(smem_addr(&bars->tmem_empty[b]), bph ^ 1, p, bars, 3)) { ok = false; break; }
              const uint64_t ad = ad0 + s * kPStage, bd = bd0 + s * kQStage;
              const int nsteps = (p.K - k0 >= GRAN) ? 2 : (p.K - k0 + kMmaK - 1) / kMmaK;
              for (int t = 0; t < nsteps; ++t)
                mma_f8f6f4_elect(d_tmem, ad + (t0 + t) * kPStep, bd + (t0 + t) * kQStep, idesc, t > 0 ? 1u : 0u);
              mma_commit_elect(smem_addr(&bars->tmem_full[b]));
              mma_commit_elect(smem_addr(&bars->empty[s]));
            } else if (t0 == 0 && last_in_stage) {
              // the stage has no second half: wait for it all the same
              if (!warp_wait_all(smem_addr(&bars->full[s]), ph, p, bars, 2)) { ok = false; break; }
              mma_commit_elect(smem_addr(&bars->empty[s]));
            }
            if (last_in_stage) {
              if (++s == STAGES) { s = 0; ph ^= 1; }
            }
          }
        }
      }
      // all MMAs issued by both issuers complete before TMEM is freed
      mma_commit_elect(smem_addr(&bars->mma_done));
      warp_wait_all(smem_addr(&bars->mma_done), 0, p, bars, 8, true);
    }
  } else if (warp == 3) {
    // ============================================================ stream-K publisher
    // A CTA's stream-K range holds at most one piece that is not its tile's
    // reducer: the range's first segment, when it starts inside a tile.  The
    // promotion warps write that piece's partial, arrive on `publish`
    // (release, CTA scope) and go straight on to their next item; this warp
    // waits for them (acquire) and makes the partial visible to the
    // reducer with one release add on the tile's counter (GPU scope), so the
    // promotion warps never wait for that release to complete.
    if constexpr (SPLIT) {
      if (p.sk_ctas > 0) {
        grid_dependency_wait();
        WorkIter wit;
        work_begin<SPLIT, GROUPED>(p, wit);
        for (Work w; work_next<GRAN, SPLIT, GROUPED>(p, wit, w);) {
          if (w.tile < p.sk_first_tile || w.kb0 == 0) continue;   // whole tile, or the reducer
          const Pieces pq = pieces_of<GRAN>(p, w);
          if (pq.pieces <= 1) continue;
          if (!warp_wait_all(smem_addr(&bars->publish), 0, p, bars, 6)) break;
          if (lane == 0) red_add_release_gpu(p.counters + pq.counter, 1);
          __syncwarp();
          break;
        }
      }
    }
  }
  } else {
    // ============================================================ promotion + epilogue
    if constexpr (RegSplit<BNQ>::kEnabled) set_max_regs_inc<kPromoteRegs>();
    grid_dependency_wait();
    const int ew = warp - kFirstEpiWarp;   // 0..7
    const int quad = warp & 3;             // TMEM lane quadrant this warp may access
    const int half = ew >> 2;              // which half of the BNQ columns
    const int row_in_tile = quad * 32 + static_cast<int>(lane);
    const uint32_t t_lane = static_cast<uint32_t>(quad * 32) << 16;
    uint32_t pc = 0;          // K-blocks consumed so far (TMEM buffer / phase)
    bool ok = true;
    float2 acc[kHalf / 2];    // this thread's row, columns [half*kHalf, (half+1)*kHalf)

    WorkIter wit;
    work_begin<SPLIT, GROUPED>(p, wit);
    for (Work w; ok && work_next<GRAN, SPLIT, GROUPED>(p, wit, w);) {
      if constexpr (SPLIT) {
        // where this item's partial goes: worked out while the accumulator
        // is dead and parked in shared memory (registers are short during
        // the K-loop); each warp has its own copy
        const Pieces pq = pieces_of<GRAN>(p, w);
        __syncwarp();
        if (lane == 0) {
          volatile int* d = bars->pieces[ew];
          d[0] = pq.pieces; d[1] = pq.slot; d[2] = pq.counter;
          d[3] = pq.slot0; d[4] = pq.slot_base; d[5] = pq.slot_step;
        }
        __syncwarp();
      }
#pragma unroll
      for (int i = 0; i < kHalf / 2; ++i) acc[i] = make_float2(0.f, 0.f);

      // scale rows for this warp: one P block, kNumGroups Q blocks (clamped:
      // rows past the end of P/Q hold zeros and are never stored)
      int pb = (w.tp * BM + quad * 32) / GRAN;
      int qb[kNumGroups];
      if constexpr (GROUPED) {
        // the group's own scale rows (clamped inside the group and inside sA)
        const int last = max(0, (w.g_rows - 1) / GRAN);
        pb = w.g_srow + (pb < last ? pb : last);
        pb = pb < p.Pb - 1 ? pb : p.Pb - 1;
      } else {
        pb = pb < p.Pb - 1 ? pb : p.Pb - 1;
      }
#pragma unroll
      for (int j = 0; j < kNumGroups; ++j) {
        const int b = (w.tq * BNQ + half * kHalf + j * kGroupCols) / GRAN;
        qb[j] = (b < p.Qb - 1 ? b : p.Qb - 1) + (GROUPED ? w.g_sqrow : 0);
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

        const uint32_t buf = pc % kBufs;
        // tcgen05.commit arrives only once the MMAs' TMEM writes are complete
        // every lane waits on the barrier itself: they all wake together when
        // the commit lands (a lane-0 wait plus a shuffle measured ~5 % slower)
        if (!warp_wait_all(smem_addr(&bars->tmem_full[buf]), (pc / kBufs) & 1, p, bars, 4)) { ok = false; break; }
        const uint32_t taddr = tmem_base + t_lane + buf * BNQ + half * kHalf;
        {
          // TMEM -> registers in chunks of up to 64 columns.  The buffer is
          // released as soon as the last chunk is in registers, before that
          // chunk is scaled, so the MMA can start refilling it sooner.
          constexpr int CW = kHalf < 64 ? kHalf : 64;
          constexpr int NC = kHalf / CW;
          uint32_t r[CW];
#pragma unroll
          for (int c = 0; c < NC; ++c) {
            tmem_ld(taddr + c * CW, r);
            tmem_wait_ld(r);
            if (c == NC - 1) {
              __syncwarp();
              if (lane == 0) mbar_arrive(smem_addr(&bars->tmem_empty[buf]));
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

      // ---------------------------------------------------------- partial-tile fix-up
      if constexpr (SPLIT) {
        Pieces pcs;
        {
          const volatile int* d = bars->pieces[ew];
          pcs.pieces = d[0]; pcs.slot = d[1]; pcs.counter = d[2];
          pcs.slot0 = d[3]; pcs.slot_base = d[4]; pcs.slot_step = d[5];
        }
        if (pcs.pieces > 1) {
          // Stream-K: the piece that starts the tile (kb0 == 0) is the last
          // segment of its CTA's range, so it ends after the tile's other
          // pieces, which each start a CTA's range.  It keeps its partial in
          // registers, waits for the others and adds them in K order.
          // Split-K pieces all end at about the same time; there the last to
          // arrive adds all of them.  Either way the sum is piece 0 + piece 1
          // + ... in FP32, in that order, every run.
          const bool reducer = p.sk_ctas > 0 && w.tile >= p.sk_first_tile && w.kb0 == 0;
          const size_t chunk_off = static_cast<size_t>(half * kHalf / 4) * BM + row_in_tile;
          if (!reducer) {
            // partial tile as 16-byte chunks [BNQ / 4][BM][4]: each thread writes
            // its row's kHalf / 4 chunks, and a warp (32 consecutive rows) writes
            // 512 contiguous bytes per chunk
            float4* my_ws = reinterpret_cast<float4*>(p.ws + static_cast<size_t>(pcs.slot) * (BNQ * BM)) +
                            (half * kHalf / 4) * BM + row_in_tile;
#pragma unroll
            for (int c = 0; c < kHalf / 4; ++c)
              __stcg(my_ws + c * BM, make_float4(acc[2 * c].x, acc[2 * c].y, acc[2 * c + 1].x, acc[2 * c + 1].y));
            if (p.sk_ctas > 0 && w.tile >= p.sk_first_tile) {
              // stream-K: the publisher warp releases the partial; this
              // warp's stores come before its lane 0's arrive (the warp
              // barrier orders them, the arrive is a CTA-scope release)
              __syncwarp();
              if (lane == 0) mbar_arrive(smem_addr(&bars->publish));
              continue;
            }
            // Split-K: the partial now lives in the workspace; acc is dead
            // until the sum below.  Publishing it takes one release: every
            // promotion thread's stores come before the CTA barrier, the
            // barrier before the leader's acq_rel add on the tile counter
            // (GPU scope), which also acquires the earlier pieces and tells
            // whether this piece arrived last.
            named_barrier_sync(1, kNumEpiThreads);
            if (ew == 0 && lane == 0)
              bars->split_last = atom_add_acq_rel_gpu(p.counters + pcs.counter, 1) == pcs.pieces - 1;
            named_barrier_sync(1, kNumEpiThreads);
            const bool last = *reinterpret_cast<volatile int*>(&bars->split_last) != 0;
            // nobody may overwrite split_last before every thread has read it
            named_barrier_sync(1, kNumEpiThreads);
            if (!last) continue;
            // split-K, last to arrive: piece 0 from the workspace first
            const float4* src =
                reinterpret_cast<const float4*>(p.ws + static_cast<size_t>(piece_slot(pcs, 0)) * (BNQ * BM)) + chunk_off;
#pragma unroll
            for (int c = 0; c < kHalf / 4; ++c) {
              const float4 v = __ldcg(src + c * BM);
              acc[2 * c] = make_float2(v.x, v.y);
              acc[2 * c + 1] = make_float2(v.z, v.w);
            }
          } else {
            // stream-K reducer: the leader waits (bounded) until the other
            // pieces - 1 pieces have published (acquire), and the barrier
            // hands them to the other threads
            if (ew == 0 && lane == 0)
              bars->split_last = wait_counter_acquire(p, bars, p.counters + pcs.counter, pcs.pieces - 1, 5) ? 1 : 0;
            named_barrier_sync(1, kNumEpiThreads);
            const bool got = *reinterpret_cast<volatile int*>(&bars->split_last) != 0;
            named_barrier_sync(1, kNumEpiThreads);
            if (!got) { ok = false; break; }
          }
          // piece 0 is in acc; the others follow in K order.  A piece's
          // kHalf / 4 chunk loads are independent, so they are all in flight
          // together
          for (int j = 1; j < pcs.pieces; ++j) {
            const float4* src =
                reinterpret_cast<const float4*>(p.ws + static_cast<size_t>(piece_slot(pcs, j)) * (BNQ * BM)) + chunk_off;
            float4 v[kHalf / 4];
#pragma unroll
            for (int c = 0; c < kHalf / 4; ++c) v[c] = __ldcg(src + c * BM);
#pragma unroll
            for (int c = 0; c < kHalf / 4; ++c) {
              acc[2 * c].x += v[c].x;
              acc[2 * c].y += v[c].y;
              acc[2 * c + 1].x += v[c].z;
              acc[2 * c + 1].y += v[c].w;
            }
          }
          if (ew == 0 && lane == 0) p.counters[pcs.counter] = 0;  // ready for the next launch
        }
      }

      // ---------------------------------------------------------- epilogue + store
      if constexpr (SWAP) {
        // tile rows are N, tile columns are M: out[m][n]
        const int n = w.tp * BM + row_in_tile;
        if (!(p.epi & kEpiOutF32)) {
          // BF16: the whole tile goes through the staging buffer, [BNQ][128]
          // in the output's order: for each m, the warp's 32 lanes write 32
          // consecutive n (64 bytes); then one TMA copy stores the tile (rows
          // past M and columns past N are clipped by the tensor map)
          const uint32_t stage = smem_addr(epi_bufs);
          const int act = p.epi & 3;
          const float bn = (p.bias != nullptr && n < p.N) ? __ldg(p.bias + n) : 0.f;
          // the previous tile's store must have finished reading the buffer
          if (ew == 0 && lane == 0) bulk_wait_group_read0();
          named_barrier_sync(2, kNumEpiThreads);
          const uint32_t col0 = stage + (half * kHalf * BM + row_in_tile) * 2;  // m = half * kHalf
          if (p.bias == nullptr && act == 0) {
            // the plain BF16 output: no activation code in the loop (evaluated
            // per element, the erf branch cost ~90 cycles a value)
#pragma unroll
            for (int i = 0; i < kHalf / 2; ++i) {
              const __nv_bfloat162 h = __float22bfloat162_rn(acc[i]);
              st_shared_b16(col0 + (2 * i) * BM * 2, __bfloat16_as_ushort(h.x));
              st_shared_b16(col0 + (2 * i + 1) * BM * 2, __bfloat16_as_ushort(h.y));
            }
          } else {
            with_act(act, [&](auto tag) {
              constexpr int ACT = decltype(tag)::value;
#pragma unroll
              for (int i = 0; i < kHalf; ++i) {
                const float v = epi_act_t<ACT>(((i & 1) ? acc[i / 2].y : acc[i / 2].x) + bn);
                st_shared_b16(col0 + i * BM * 2, __bfloat16_as_ushort(__float2bfloat16_rn(v)));
              }
            });
          }
          fence_proxy_async_smem();
          named_barrier_sync(2, kNumEpiThreads);
          if (ew == 0 && lane == 0) {
            tma_store_2d(&tm_out, stage, w.tp * BM, w.tq * BNQ);
            bulk_commit_group();
          }
        } else if (n < p.N) {
          const int act = p.epi & 3;
          const float bn = p.bias != nullptr ? __ldg(p.bias + n) : 0.f;
          with_act(act, [&](auto tag) {
            constexpr int ACT = decltype(tag)::value;
#pragma unroll
            for (int i = 0; i < kHalf; ++i) {
              const int m = w.tq * BNQ + half * kHalf + i;
              const float v = epi_act_t<ACT>(((i & 1) ? acc[i / 2].y : acc[i / 2].x) + bn);
              if (m < p.M) reinterpret_cast<float*>(p.out)[static_cast<size_t>(m) * p.N + n] = v;
            }
          });
        }
      } else if constexpr (SC::kTmaStore) {
        // this thread owns row m0 + lane, columns [n0, n0 + kHalf); the warp
        // stores its 32 rows through its staging buffer
        const int n0 = w.tq * BNQ + half * kHalf;
        apply_epi<kHalf / 2>(p, n0, acc);
        store_tile_tma<kHalf / 2>(p, &tm_out, smem_addr(epi_bufs + ew * kEpiChunkBytes),
                                  w.tp * BM + quad * 32, n0, acc, lane);
      } else {
        // this thread owns row m, columns [n0, n0 + kHalf)
        const int m_local = w.tp * BM + row_in_tile;
        const int m = (GROUPED ? w.g_row : 0) + m_local;
        const int n0 = w.tq * BNQ + half * kHalf;
        if (m < p.M && (!GROUPED || m_local < w.g_rows)) store_row_run<kHalf / 2>(p, m, n0, acc);
      }
    }
    // every bulk store this warp issued has finished (reads of its staging
    // buffer and writes to global memory) before the CTA exits
    if constexpr (SC::kTmaStore || SC::kSwapTmaStore) {
      if (lane == 0) bulk_wait_group0();
    }
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
