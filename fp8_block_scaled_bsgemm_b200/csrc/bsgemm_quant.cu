// Per-block FP8 quantiser: the step the pages put in front of the GEMM
// (hncyxsy.com/news/191052 §4.4: the quantisation granularity must match the
// GEMM's; §5.2: quantisation divides by the scale, dequantisation multiplies).
//
// For each g x g block of a row-major [rows, cols] FP32 or BF16 matrix:
//   amax = max |x| over the block's elements;
//   s    = amax / FMAX in FP32, correctly rounded (FMAX = 448 for E4M3,
//          57344 for E5M2), or 1 when amax is 0;
//   q    = FP8 code of x / s (FP32 division, correctly rounded), rounded to
//          nearest with ties to even and saturated to +-FMAX.
// (For BF16 input the correctly rounded x / s is formed without a division;
// see quotient() below.)
// The codes go to q [rows, cols] (row-major, one byte each) and the scales
// to scales [ceil(rows/g), ceil(cols/g)] (row-major FP32): exactly the
// operand and scale tensors the GEMM takes.
//
// One CTA per block for g <= 128; for g = 256 a cluster of four CTAs per
// block, each taking 64 of its rows, which exchange their partial maxima
// through distributed shared memory. Each thread keeps its part of the block in
// registers between the amax pass and the encode pass. Each thread handles
// runs of 8 consecutive columns: 32-byte (FP32) or 16-byte (BF16) loads,
// 8-byte stores of 8 codes. This is HBM-bound work: no tensor cores.
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <type_traits>

#include "bsgemm.h"
#include "ptx.cuh"

namespace bsgq {

// CTAs per block: a g = 256 block is split by rows over a cluster of four, so
// that every CTA holds 64 x 256 values, as many as a g = 128 block.
template <int G>
constexpr int kParts = G == 256 ? 4 : 1;

// Threads per CTA: 512 from FP32 at g >= 128 (each thread holds 4 runs), else
// 256 (8 runs held from BF16 at g >= 128; 2 at g = 64).
template <int G, bool BF16_IN>
constexpr int kThreads = (G >= 128 && !BF16_IN) ? 512 : 256;
constexpr int kVec = 8;  // columns per run

// One run of 8 source values as loaded: one 16-byte word of BF16 values, or
// two of FP32 values. A run is held in this form and widened on use, so a
// BF16 run costs 4 registers rather than 8.
template <bool BF16_IN>
struct Run {
  uint4 w[BF16_IN ? 1 : 2];
};

// Store a float to a CTA's shared memory in the cluster (a shared::cluster address).
__device__ __forceinline__ void st_shared_cluster_f32(uint32_t addr, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}

template <bool BF16_IN>
__device__ __forceinline__ Run<BF16_IN> load_run(const void* x, int64_t off) {
  Run<BF16_IN> r;
  if constexpr (BF16_IN) {
    r.w[0] = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(x) + off));
  } else {
    const uint4* p = reinterpret_cast<const uint4*>(static_cast<const float*>(x) + off);
    r.w[0] = __ldg(p);
    r.w[1] = __ldg(p + 1);
  }
  return r;
}

template <bool BF16_IN>
__device__ __forceinline__ void widen(const Run<BF16_IN>& r, float (&v)[kVec]) {
  if constexpr (BF16_IN) {
    const uint32_t w[4] = {r.w[0].x, r.w[0].y, r.w[0].z, r.w[0].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  } else {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      v[4 * h + 0] = __uint_as_float(r.w[h].x);
      v[4 * h + 1] = __uint_as_float(r.w[h].y);
      v[4 * h + 2] = __uint_as_float(r.w[h].z);
      v[4 * h + 3] = __uint_as_float(r.w[h].w);
    }
  }
}

template <bool BF16_IN>
__device__ __forceinline__ void load8(const void* x, int64_t off, float (&v)[kVec]) {
  widen<BF16_IN>(load_run<BF16_IN>(x, off), v);
}

// FP8 codes of a (low byte) and b (the byte above): round to nearest even,
// saturating to the largest finite value; one conversion for the pair
template <int FMT>
__device__ __forceinline__ uint32_t encode2(float a, float b) {
  return static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE,
                                                        FMT == BSGEMM_FP8_E5M2 ? __NV_E5M2 : __NV_E4M3));
}

// x / s, correctly rounded in FP32.
//
// FAST = false: the division itself.
// FAST = true: Markstein's correction step for division. From the correctly
// rounded reciprocal rs = RN(1/s), take q0 = RN(x * rs), form the residual
// negated, q0 * s - x, exactly with one fma, and subtract residual * rs from q0
// with a second fma. Taking the residual negated keeps the sign of a zero x:
// -0 gives -0.
//
// The fast form is used only for BF16 input and only for s >= kFastMinScale.
// There the residual is exact wherever the FP8 code depends on it.
// tests/quant_division_model.c runs the same steps for every BF16 block amax
// (s = RN(amax / FMAX)) and every BF16 x with |x| <= amax, for E4M3 and E5M2,
// about 1.9e9 pairs. Where |x / s| >= 2^-18, q equals RN(x / s) bit for bit.
// Below that, both are under 2^-17 with the same sign, so both give the code
// +-0. FP32 input is not covered by that enumeration and keeps the division.
constexpr float kFastMinScale = 0x1p-60f;

template <bool FAST>
__device__ __forceinline__ float quotient(float x, float s, float rs) {
  if constexpr (FAST) {
    const float q0 = __fmul_rn(x, rs);
    return __fmaf_rn(-__fmaf_rn(q0, s, -x), rs, q0);
  } else {
    return __fdiv_rn(x, s);
  }
}

// CTAs per SM each instance's registers are held to: at g >= 128 (BF16: 256
// threads at 64 registers, 4 CTAs; FP32: 512 threads at 64 registers, 2 CTAs);
// g = 64 runs 8 (BF16) or 6 (FP32).
template <int G, bool BF16_IN>
constexpr int kMinCtasPerSm = G >= 128 ? (BF16_IN ? 4 : 2) : (BF16_IN ? 8 : 6);

template <int G, bool BF16_IN, int FMT>
__global__ void __launch_bounds__((kThreads<G, BF16_IN>), (kMinCtasPerSm<G, BF16_IN>))
    quant_kernel(const void* __restrict__ x, int64_t rows, int64_t cols, int64_t col_blocks,
                 uint8_t* __restrict__ q, float* __restrict__ scales) {
  constexpr int kT = kThreads<G, BF16_IN>;
  constexpr int kP = kParts<G>;
  constexpr int kRuns = (G / kP) * G / kVec;   // runs of 8 columns in this CTA's rows of a full block
  constexpr int kRunsPerRow = G / kVec;
  constexpr float kFmax = FMT == BSGEMM_FP8_E5M2 ? 57344.0f : 448.0f;
  __shared__ float warp_max[kT / 32];
  __shared__ float block_scale;
  __shared__ float part_max[kParts<G>];   // the shares of a split block's amax, one per CTA

  // block blk; this CTA takes its rows [part * G / kP, (part + 1) * G / kP)
  // (a cluster is kP consecutive CTAs of the grid, so part is the rank)
  const int64_t blk = blockIdx.x / kP;
  const int part = static_cast<int>(blockIdx.x % kP);
  const int64_t r0 = (blk / col_blocks) * G + part * (G / kP);
  const int64_t c0 = (blk % col_blocks) * G;
  // the thread's runs stay in registers between the two passes
  constexpr int kHeld = kRuns / kT <= 8 ? kRuns / kT : 0;
  Run<BF16_IN> held[kHeld > 0 ? kHeld : 1];

  // ---- pass 1: amax over the block (elements outside the matrix are skipped)
  float amax = 0.f;
  if constexpr (kHeld > 0) {
#pragma unroll
    for (int j = 0; j < kHeld; ++j) {
      const int run = threadIdx.x + j * kT;
      const int64_t r = r0 + run / kRunsPerRow;
      const int64_t c = c0 + (run % kRunsPerRow) * kVec;
      if (r < rows && c < cols) {  // cols % 8 == 0: a run is wholly in or out
        held[j] = load_run<BF16_IN>(x, r * cols + c);
      } else {
#pragma unroll
        for (int h = 0; h < (BF16_IN ? 1 : 2); ++h) held[j].w[h] = make_uint4(0, 0, 0, 0);
      }
    }
    if constexpr (BF16_IN) {
      // |x| max on packed pairs (NaN-ignoring, like fmaxf): the runs stay
      // packed until the encode pass widens them
      __nv_bfloat162 m2 = __float2bfloat162_rn(0.f);
#pragma unroll
      for (int j = 0; j < kHeld; ++j) {
        const uint32_t w[4] = {held[j].w[0].x, held[j].w[0].y, held[j].w[0].z, held[j].w[0].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          __nv_bfloat162_raw raw;
          raw.x = static_cast<unsigned short>(w[i] & 0xFFFFu);
          raw.y = static_cast<unsigned short>(w[i] >> 16);
          m2 = __hmax2(m2, __habs2(__nv_bfloat162(raw)));
        }
      }
      amax = fmaxf(__low2float(m2), __high2float(m2));
    } else {
#pragma unroll
      for (int j = 0; j < kHeld; ++j) {
        float v[kVec];
        widen<BF16_IN>(held[j], v);
#pragma unroll
        for (int i = 0; i < kVec; ++i) amax = fmaxf(amax, fabsf(v[i]));
      }
    }
  } else {
    for (int run = threadIdx.x; run < kRuns; run += kT) {
      const int64_t r = r0 + run / kRunsPerRow;
      const int64_t c = c0 + (run % kRunsPerRow) * kVec;
      if (r < rows && c < cols) {
        float v[kVec];
        load8<BF16_IN>(x, r * cols + c, v);
#pragma unroll
        for (int i = 0; i < kVec; ++i) amax = fmaxf(amax, fabsf(v[i]));
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = amax;
  __syncthreads();
  float cta_max = 0.f;
  if (threadIdx.x == 0) {
    cta_max = warp_max[0];
#pragma unroll
    for (int w = 1; w < kT / 32; ++w) cta_max = fmaxf(cta_max, warp_max[w]);
  }
  if constexpr (kP > 1) {
    // the block's amax: thread 0 of each CTA writes its share into slot
    // `part` of every CTA of the cluster, its own included. One cluster
    // barrier (every thread; release then acquire) makes all kP shares
    // visible in each CTA's own shared memory, and no CTA touches another's
    // shared memory after it, so any CTA may then run on to its exit.
    if (threadIdx.x == 0) {
      const uint32_t slot = static_cast<uint32_t>(__cvta_generic_to_shared(&part_max[part]));
#pragma unroll
      for (int r = 0; r < kP; ++r) st_shared_cluster_f32(bsg::mapa_shared(slot, r), cta_max);
    }
    bsg::cluster_sync_all();
    if (threadIdx.x == 0) {
#pragma unroll
      for (int r = 0; r < kP; ++r) cta_max = fmaxf(cta_max, part_max[r]);
    }
  }
  if (threadIdx.x == 0) {
    const float s = cta_max > 0.f ? __fdiv_rn(cta_max, kFmax) : 1.0f;
    block_scale = s;
    if (part == 0) scales[blk] = s;
  }
  __syncthreads();
  const float s = block_scale;

  // ---- pass 2: encode.  The quotient's form is chosen once per block.
  auto encode_block = [&](auto fast_tag) {
    constexpr bool kFast = decltype(fast_tag)::value;
    const float rs = kFast ? __frcp_rn(s) : 0.f;
    auto encode_run = [&](const float (&v)[kVec], int64_t r, int64_t c) {
      float d[kVec];
#pragma unroll
      for (int i = 0; i < kVec; ++i) d[i] = quotient<kFast>(v[i], s, rs);
      const uint32_t lo = encode2<FMT>(d[0], d[1]) | (encode2<FMT>(d[2], d[3]) << 16);
      const uint32_t hi = encode2<FMT>(d[4], d[5]) | (encode2<FMT>(d[6], d[7]) << 16);
      *reinterpret_cast<uint2*>(q + r * cols + c) = make_uint2(lo, hi);
    };
    if constexpr (kHeld > 0) {
#pragma unroll
      for (int j = 0; j < kHeld; ++j) {
        const int run = threadIdx.x + j * kT;
        const int64_t r = r0 + run / kRunsPerRow;
        const int64_t c = c0 + (run % kRunsPerRow) * kVec;
        if (r < rows && c < cols) {
          float v[kVec];
          widen<BF16_IN>(held[j], v);
          encode_run(v, r, c);
        }
      }
    } else {
      for (int run = threadIdx.x; run < kRuns; run += kT) {
        const int64_t r = r0 + run / kRunsPerRow;
        const int64_t c = c0 + (run % kRunsPerRow) * kVec;
        if (r < rows && c < cols) {
          float v[kVec];
          load8<BF16_IN>(x, r * cols + c, v);
          encode_run(v, r, c);
        }
      }
    }
  };
  if constexpr (BF16_IN) {
    if (s >= kFastMinScale) encode_block(std::true_type{});
    else                    encode_block(std::false_type{});
  } else {
    encode_block(std::false_type{});
  }
}

template <int G, bool BF16_IN, int FMT>
bsgemm_status launch(const void* x, int64_t rows, int64_t cols, uint8_t* q, float* scales,
                     cudaStream_t stream) {
  const int64_t rb = (rows + G - 1) / G, cb = (cols + G - 1) / G;
  const int64_t ctas = rb * cb * kParts<G>;
  if (ctas > 0x7FFFFFFFll) return BSGEMM_ERR_INVALID_ARG;
  if constexpr (kParts<G> == 1) {
    quant_kernel<G, BF16_IN, FMT><<<static_cast<unsigned>(ctas), kThreads<G, BF16_IN>, 0, stream>>>(
        x, rows, cols, cb, q, scales);
  } else {
    // a cluster of kParts CTAs per block
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(ctas), 1, 1);
    cfg.blockDim = dim3(kThreads<G, BF16_IN>, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kParts<G>;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, quant_kernel<G, BF16_IN, FMT>, x, rows, cols, cb, q, scales) != cudaSuccess)
      return BSGEMM_ERR_CUDA;
  }
  return cudaGetLastError() == cudaSuccess ? BSGEMM_OK : BSGEMM_ERR_CUDA;
}

template <int G>
bsgemm_status dispatch_g(int src, int fmt, const void* x, int64_t rows, int64_t cols, uint8_t* q,
                         float* s, cudaStream_t st) {
  if (src == BSGEMM_SRC_BF16)
    return fmt == BSGEMM_FP8_E5M2 ? launch<G, true, BSGEMM_FP8_E5M2>(x, rows, cols, q, s, st)
                                  : launch<G, true, BSGEMM_FP8_E4M3>(x, rows, cols, q, s, st);
  return fmt == BSGEMM_FP8_E5M2 ? launch<G, false, BSGEMM_FP8_E5M2>(x, rows, cols, q, s, st)
                                : launch<G, false, BSGEMM_FP8_E4M3>(x, rows, cols, q, s, st);
}

}  // namespace bsgq

extern "C" bsgemm_status bsgemm_quantize_fp8(int src_dtype, int fp8_format, const void* x,
                                             int64_t rows, int64_t cols, int gran, void* q,
                                             float* scales, bsgemm_stream_t stream) {
  if (!x || !q || !scales || rows <= 0 || cols <= 0) return BSGEMM_ERR_INVALID_ARG;
  if (src_dtype != BSGEMM_SRC_F32 && src_dtype != BSGEMM_SRC_BF16) return BSGEMM_ERR_INVALID_ARG;
  if (fp8_format != BSGEMM_FP8_E4M3 && fp8_format != BSGEMM_FP8_E5M2) return BSGEMM_ERR_INVALID_ARG;
  if (gran != 64 && gran != 128 && gran != 256) return BSGEMM_ERR_UNSUPPORTED_GRAN;
  if (cols % 16 != 0 || (reinterpret_cast<uintptr_t>(x) & 15) != 0 ||
      (reinterpret_cast<uintptr_t>(q) & 15) != 0 || (reinterpret_cast<uintptr_t>(scales) & 3) != 0)
    return BSGEMM_ERR_MISALIGNED;
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return BSGEMM_ERR_CUDA;
  if (major != 10) return BSGEMM_ERR_UNSUPPORTED_DEVICE;
  auto* qq = static_cast<uint8_t*>(q);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  switch (gran) {
    case 64:  return bsgq::dispatch_g<64>(src_dtype, fp8_format, x, rows, cols, qq, scales, s);
    case 128: return bsgq::dispatch_g<128>(src_dtype, fp8_format, x, rows, cols, qq, scales, s);
    default:  return bsgq::dispatch_g<256>(src_dtype, fp8_format, x, rows, cols, qq, scales, s);
  }
}
