// Host-side pieces shared by the C ABI (bsgemm_api.cu) and the kernel
// instance units (bsgemm_inst.cu, compiled once per granularity and layout).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstddef>
#include <cstdint>

#include "bsgemm.h"

namespace bsg_host {

struct DeviceInfo {
  bool ok = false;
  int ordinal = 0;        // CUDA device number
  int num_sms = 0;
  int* status = nullptr;  // device address of the status word
};

// One-time per-device launch setup of one kernel instance (function
// attributes are set per device): a bit per device for devices 0..63;
// higher-numbered devices simply redo the setup on every launch.
class PerDeviceOnce {
 public:
  bool done(int dev) const {
    return dev >= 0 && dev < 64 && ((bits_.load(std::memory_order_acquire) >> dev) & 1u);
  }
  void mark(int dev) {
    if (dev >= 0 && dev < 64) bits_.fetch_or(uint64_t(1) << dev, std::memory_order_acq_rel);
  }

 private:
  std::atomic<uint64_t> bits_{0};
};

struct Workspace {
  float* ws = nullptr;
  size_t ws_bytes = 0;
  int* counters = nullptr;
  size_t n_counters = 0;
};

// 2D tensor map with 128-byte swizzle; `inner` is the contiguous extent.
bool make_map_2d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint64_t inner,
                 uint64_t outer, uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer);

// Tensor map of the [M, N] row-major output for the TMA-store epilogue: BF16
// boxes of 32 rows x 64 columns, or FP32 boxes of 32 x 32 (128 bytes a row,
// 128-byte swizzle).
bool make_out_map(CUtensorMap* m, void* out, int M, int N, bool f32);

// Tensor map of the BF16 [M, N] output for swap-AB tiles: boxes of BNQ rows
// (m) x 128 columns (n), no swizzle (the staging tile is [BNQ][128] BF16).
bool make_swap_out_map(CUtensorMap* m, void* out, int M, int N, int bnq);

// Split-K workspace of at least `ws_bytes` bytes and `n_counters` zeroed
// counters for (current device, stream).
bsgemm_status get_workspace(cudaStream_t stream, size_t ws_bytes, size_t n_counters, Workspace& out);

// Limit of every bounded device-side wait, in nanoseconds.
unsigned long long wait_timeout_ns();

// Device address of the current device's status word (looked up on every
// call; allocates nothing).
bsgemm_status device_status_address(int** out);

// Per-call options beyond the plan: operand formats and the epilogue.
struct CallOpts {
  int a_fmt = BSGEMM_FP8_E4M3;   // bsgemm_fp8_format of the logical A operand
  int b_fmt = BSGEMM_FP8_E4M3;   // ... and of B
  const float* bias = nullptr;   // FP32 [N] or null
  int epi = 0;                   // activation (bits 0-1) | FP32 output (bit 2)
  const int* group_m = nullptr;  // grouped GEMM: device rows per group
  int num_groups = 0;
};

#define BSG_RUN_DECL(G, L)                                                                       \
  bsgemm_status run_g##G##_##L(const bsgemm_plan& plan, const void* a, const void* b,          \
                               const float* sa, const float* sb, void* out, int M, int N, int K, \
                               const CallOpts& opts, cudaStream_t stream, const DeviceInfo& dev);
BSG_RUN_DECL(64, nt) BSG_RUN_DECL(64, tn) BSG_RUN_DECL(64, nn) BSG_RUN_DECL(64, tt)
BSG_RUN_DECL(128, nt) BSG_RUN_DECL(128, tn) BSG_RUN_DECL(128, nn) BSG_RUN_DECL(128, tt)
BSG_RUN_DECL(256, nt) BSG_RUN_DECL(256, tn) BSG_RUN_DECL(256, nn) BSG_RUN_DECL(256, tt)
#undef BSG_RUN_DECL

}  // namespace bsg_host
