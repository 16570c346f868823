/*
 * bsgemm.h -- C ABI of the B200 (sm_100a) block-scaled FP8 GEMM library.
 *
 * Operation (hncyxsy.com/news/191052, "DeepGEMM实战: FP8矩阵乘法加速与Hopper
 * 架构优化指南", §2.2 block-wise scaling, §3.2 segment-wise FP32 accumulation,
 * §4.2 the gemm_fp8_fp8_bf16_nt call and its NT/TN/NN/TT flags):
 *
 *   out[m,n] = bf16( sum_kb  sA[m/g][kb] * sB[n/g][kb]
 *                            * sum_{k in K-block kb} A[m,k] * B[n,k] )
 *
 * A and B hold FP8 E4M3 codes (OCP "e4m3fn": no infinities, 0x7F/0xFF NaN).
 * Each operand carries one FP32 scale per g x g block (§2.2, §3.1 table:
 * g = 128 by default, 64 and 256 as variants); the scale multiplies the code
 * (§5.2: quantisation divides, dequantisation multiplies).  Each K-block's
 * partial sum is taken on the tensor cores and promoted into an FP32
 * accumulator with sA*sB applied (§3.2); the result is rounded to BF16
 * (round to nearest even).
 *
 * Argument conventions shared by every entry point:
 *   a, b      device pointers to E4M3 bytes, dense (no padding between rows):
 *               _nt: A stored [M,K] row-major, B stored [N,K] row-major
 *               _tn: A stored [K,M],           B stored [K,N]
 *               _nn: A stored [M,K],           B stored [K,N]
 *               _tt: A stored [K,M],           B stored [N,K]
 *             (first letter A, second letter B; for A "N" means [M,K] and "T"
 *             means [K,M]; for B "T" means [N,K] and "N" means [K,N]).  The
 *             transposed forms are read through the TMA descriptors; no
 *             transposed copy is made (§3.3).
 *   scale_a   device pointer, FP32 [ceil(M/g)][ceil(K/g)] row-major
 *   scale_b   device pointer, FP32 [ceil(N/g)][ceil(K/g)] row-major
 *             Scales are indexed by logical block, whatever the layout.  A
 *             partial last block (M, N or K not a multiple of g) has its own
 *             scale and simply covers fewer rows/columns.
 *   out       device pointer, BF16 [M,N] row-major, preallocated by the caller
 *   M, N, K   logical sizes, each > 0
 *   gran      g, one of 64, 128, 256 (the same for A, B and the K blocks)
 *   stream    CUDA stream; the call is asynchronous with respect to the host
 *
 * Ownership: all pointers belong to the caller, who keeps them alive until
 * the stream has passed the call.  The library keeps no pointer beyond the
 * call.  It owns an internal split-K workspace per (device, stream), grown on
 * demand and never shrunk; two calls that run concurrently on different
 * streams never share it.  Growth is stream-ordered on the call's stream
 * (cudaFreeAsync of the old buffer, cudaMallocAsync of the new one), so a
 * growing call neither synchronises the device nor waits for other streams.
 * Workspaces are keyed by the stream's process-unique id (cudaStreamGetId),
 * so a stream created after another was destroyed never inherits its
 * workspace, even with the same handle value; the destroyed stream's
 * workspace stays allocated until bsgemm_release_workspaces() or process
 * exit.  A call captured into a CUDA graph can only use the workspace that
 * earlier uncaptured calls on the same stream made big enough; otherwise it
 * fails with BSGEMM_ERR_CUDA before anything is captured, and the capture
 * stays valid: run the same call once on that stream before capturing it.
 *
 * Alignment (TMA rules), checked on the host before any launch:
 *   a, b, out 16-byte aligned; scale_a, scale_b 4-byte aligned;
 *   every row stride a multiple of 16 bytes: K % 16 == 0 for K-major
 *   operands, M % 16 == 0 when A is stored [K,M], N % 16 == 0 when B is
 *   stored [K,N]; N % 8 == 0 for out.
 *
 * Errors: argument and alignment problems and a device that is not sm_100
 * are reported before anything is launched, and nothing is written to out.
 * A failed launch returns BSGEMM_ERR_CUDA.  Waits inside the kernels are
 * bounded: a wait that runs out records BSGEMM_ERR_DEVICE_TIMEOUT in a device
 * status word (read with bsgemm_get_last_device_status) and the kernel
 * returns without trapping, so the context stays usable.
 *
 * Results are deterministic: the same inputs give bit-identical outputs
 * (split-K partials are added in a fixed order).
 *
 * Launches use programmatic dependent launch: a GEMM kernel may start its
 * set-up (barriers, TMEM, descriptor prefetch) while the previous kernel on
 * the stream is finishing, and waits for that kernel to complete, with its
 * memory visible, before it reads or writes any global memory.  Stream
 * order is therefore unchanged for the caller.  A later kernel that the
 * caller launches with programmatic serialisation of its own must likewise
 * wait (griddepcontrol.wait) before it reads this call's output.
 */
#ifndef BSGEMM_H
#define BSGEMM_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Opaque CUDA stream handle (cudaStream_t); 0 is the legacy default stream. */
typedef void *bsgemm_stream_t;

typedef enum {
    BSGEMM_OK = 0,
    BSGEMM_ERR_INVALID_ARG = 1,      /* null pointer, size <= 0, bad layout */
    BSGEMM_ERR_UNSUPPORTED_GRAN = 2, /* gran not in {64, 128, 256} */
    BSGEMM_ERR_MISALIGNED = 3,       /* a TMA alignment rule above is broken */
    BSGEMM_ERR_UNSUPPORTED_DEVICE = 4, /* current device is not sm_100 */
    BSGEMM_ERR_CUDA = 5,             /* a CUDA runtime/driver call failed */
    BSGEMM_ERR_DEVICE_TIMEOUT = 6,   /* a bounded device-side wait ran out */
    BSGEMM_ERR_SCRATCH_LIMIT = 7     /* bsgemm_fp8_nt_noalloc: the problem needs more
                                        scratch than its fixed array holds */
} bsgemm_status;

/* NT: A [M,K], B [N,K] -- the native form (§3.3: fastest). */
bsgemm_status bsgemm_fp8_nt(const void *a, const void *b, const float *scale_a,
                            const float *scale_b, void *out, int64_t M, int64_t N, int64_t K,
                            int gran, bsgemm_stream_t stream);

/* TN: A stored [K,M], B stored [K,N]. */
bsgemm_status bsgemm_fp8_tn(const void *a, const void *b, const float *scale_a,
                            const float *scale_b, void *out, int64_t M, int64_t N, int64_t K,
                            int gran, bsgemm_stream_t stream);

/* NN: A stored [M,K], B stored [K,N]. */
bsgemm_status bsgemm_fp8_nn(const void *a, const void *b, const float *scale_a,
                            const float *scale_b, void *out, int64_t M, int64_t N, int64_t K,
                            int gran, bsgemm_stream_t stream);

/* TT: A stored [K,M], B stored [N,K]. */
bsgemm_status bsgemm_fp8_tt(const void *a, const void *b, const float *scale_a,
                            const float *scale_b, void *out, int64_t M, int64_t N, int64_t K,
                            int gran, bsgemm_stream_t stream);

/* ---- explicit-layout form, plan inspection and tuning ------------------ */

typedef enum {
    BSGEMM_LAYOUT_NT = 0, /* A [M,K], B [N,K] */
    BSGEMM_LAYOUT_TN = 1, /* A [K,M], B [K,N] */
    BSGEMM_LAYOUT_NN = 2, /* A [M,K], B [K,N] */
    BSGEMM_LAYOUT_TT = 3  /* A [K,M], B [N,K] */
} bsgemm_layout;

typedef enum {
    BSGEMM_VARIANT_AUTO = 0,          /* library heuristic */
    BSGEMM_VARIANT_DATA_PARALLEL = 1, /* 128 rows of A per tile on the MMA M side */
    BSGEMM_VARIANT_SWAP_AB = 2,       /* 128 rows of B per tile on the MMA M side (small M) */
    BSGEMM_VARIANT_CTA_PAIR = 3       /* 256 x 256 tiles, each computed by a pair of CTAs
                                         (tcgen05 cta_group::2); whole tiles only */
} bsgemm_variant;

/* Optional overrides of the plan; 0 in any field means "choose". */
typedef struct {
    int variant;  /* bsgemm_variant */
    int bnq;      /* tile width on the MMA N side: 128/256 (data-parallel), 16..128 (swap-AB);
                     256 for CTA pairs */
    int splits;   /* K splits per output tile (split-K); > 0 turns stream-K off */
    int stream_k; /* 0 choose, 1 use stream-K whenever tiles would leave SMs idle, -1 never */
} bsgemm_tuning;

/* What one call will launch (filled by bsgemm_make_plan). */
typedef struct {
    int layout, gran;
    int swap_ab;        /* 1 if B feeds the MMA M side */
    int bnq;            /* tile width on the MMA N side */
    int tiles_p, tiles_q; /* tiles along the MMA M side (128 rows) and N side (bnq rows) */
    int splits;         /* K splits per tile */
    int kb_per_split;   /* K blocks per split */
    int grid;           /* persistent CTAs launched (<= number of SMs) */
    int group_p;        /* raster group height in tiles */
    int kernels;        /* kernel launches per call */
    int sk_first_tile;  /* stream-K: tiles before this one are computed whole, in full waves */
    int sk_units_per_tile; /* stream-K: units per tile (a unit is one K block; two when gran = 64) */
    int sk_ctas;        /* stream-K: CTAs sharing the remaining tiles' units (0: no stream-K) */
    int sk_units;       /* stream-K: units of all stream-K tiles together */
    int cta_pair;       /* 1: 256 x 256 tiles on CTA pairs (tiles_p, tiles_q count those;
                           grid counts CTAs, two per pair) */
    int grouped;        /* 1: grouped GEMM (tiles_p is per group, found on the device) */
} bsgemm_plan;

/* FP8 formats of the operands (hncyxsy.com/news/191052 §2.2 names both).
 * E4M3: the OCP "fn" variant, 1 sign, 4 exponent (bias 7), 3 mantissa bits,
 * largest finite 448, no infinities, NaN 0x7F/0xFF.
 * E5M2: 1 sign, 5 exponent (bias 15), 2 mantissa bits, largest finite 57344,
 * +-Inf 0x7C/0xFC, NaN 0x7D-0x7F/0xFD-0xFF.
 * Operands must hold finite codes only; the result for NaN or Inf inputs is
 * unspecified (the call still completes and writes out). */
typedef enum {
    BSGEMM_FP8_E4M3 = 0,
    BSGEMM_FP8_E5M2 = 1
} bsgemm_fp8_format;

/* The operation above with the layout as an argument and optional tuning
 * (NULL = heuristic). Same argument rules and errors as bsgemm_fp8_nt. */
bsgemm_status bsgemm_fp8_gemm_ex(int layout, const void *a, const void *b, const float *scale_a,
                                 const float *scale_b, void *out, int64_t M, int64_t N, int64_t K,
                                 int gran, const bsgemm_tuning *tuning, bsgemm_stream_t stream);

/* The operation with each operand's FP8 format given: a_format, b_format are
 * bsgemm_fp8_format values (any combination; the tensor core decodes both,
 * the products and block sums are the same FP32 path as E4M3 x E4M3).
 * Everything else as bsgemm_fp8_gemm_ex; BSGEMM_ERR_INVALID_ARG for an
 * unknown format. bsgemm_fp8_gemm_ex is this call with E4M3 x E4M3. */
bsgemm_status bsgemm_fp8_gemm_fmt(int layout, int a_format, int b_format, const void *a,
                                  const void *b, const float *scale_a, const float *scale_b,
                                  void *out, int64_t M, int64_t N, int64_t K, int gran,
                                  const bsgemm_tuning *tuning, bsgemm_stream_t stream);

/* ---- per-block FP8 quantiser ---------------------------------------------
 * The caller-side step the GEMM's scales come from (§4.4: the quantisation
 * granularity must match the GEMM's; §5.2: quantising divides by the scale,
 * dequantising multiplies). For each g x g block of the row-major
 * [rows, cols] source x (FP32, or BF16 bits):
 *   amax = max |x| over the block's elements (fewer in a partial block);
 *   s    = amax / FMAX in FP32 (FMAX = 448 E4M3, 57344 E5M2), 1 if amax == 0;
 *   q    = FP8 code of x / s (FP32 division, correctly rounded), nearest with
 *          ties to even, saturated to +-FMAX.
 * Outputs: q [rows, cols] row-major codes (the GEMM's A or B operand with
 * K = cols) and scales [ceil(rows/g), ceil(cols/g)] row-major FP32 (its
 * scale_a / scale_b). All pointers are device pointers owned by the caller;
 * asynchronous on `stream`.
 * Errors (before any launch, nothing written): NULL pointers or rows/cols
 * <= 0 or unknown src_dtype / fp8_format -> BSGEMM_ERR_INVALID_ARG; gran not
 * 64/128/256 -> BSGEMM_ERR_UNSUPPORTED_GRAN; cols % 16 != 0, x or q not
 * 16-byte aligned, scales not 4-byte aligned -> BSGEMM_ERR_MISALIGNED; not an
 * sm_100 device -> BSGEMM_ERR_UNSUPPORTED_DEVICE. Inputs must be finite. */
typedef enum {
    BSGEMM_SRC_F32 = 0,
    BSGEMM_SRC_BF16 = 1
} bsgemm_src_dtype;

bsgemm_status bsgemm_quantize_fp8(int src_dtype, int fp8_format, const void *x, int64_t rows,
                                  int64_t cols, int gran, void *q, float *scales,
                                  bsgemm_stream_t stream);

/* ---- fused epilogue -------------------------------------------------------
 * The pages' extension point for work fused before write-back (§2.3, §6):
 *   out[m,n] = act(acc[m,n] + bias[n])
 * where acc is the block-scaled product in FP32, bias an optional FP32 [N]
 * vector, and act one of: none, ReLU (max(v, 0)), GELU in its erf form
 * (0.5 v (1 + erf(v / sqrt 2))). The result is stored as BF16 (round to
 * nearest even) or FP32 [M,N] row-major. With split-K or stream-K the
 * epilogue runs once, after the pieces are summed. */
typedef enum {
    BSGEMM_ACT_NONE = 0,
    BSGEMM_ACT_RELU = 1,
    BSGEMM_ACT_GELU = 2
} bsgemm_activation;

typedef enum {
    BSGEMM_OUT_BF16 = 0,
    BSGEMM_OUT_F32 = 1
} bsgemm_out_dtype;

typedef struct {
    const float *bias; /* device FP32 [N], 4-byte aligned, or NULL */
    int activation;    /* bsgemm_activation */
    int out_dtype;     /* bsgemm_out_dtype: the element type of out */
} bsgemm_epilogue;

/* bsgemm_fp8_gemm_fmt with a fused epilogue (NULL = none: BF16 output).
 * out must be [M,N] of epi->out_dtype; same alignment rules (16-byte base,
 * N % 8 == 0). Unknown activation or out_dtype -> BSGEMM_ERR_INVALID_ARG,
 * misaligned bias -> BSGEMM_ERR_MISALIGNED. */
bsgemm_status bsgemm_fp8_gemm_fused(int layout, int a_format, int b_format, const void *a,
                                    const void *b, const float *scale_a, const float *scale_b,
                                    const bsgemm_epilogue *epi, void *out, int64_t M, int64_t N,
                                    int64_t K, int gran, const bsgemm_tuning *tuning,
                                    bsgemm_stream_t stream);

/* ---- grouped GEMM ---------------------------------------------------------
 * Many independent NT products in one persistent launch, the pages' "batch
 * of matrices with different shapes" (§2.1) for a shared N and K, e.g. one
 * weight matrix per expert and a variable number of rows per expert:
 *   for group i with M_i = group_m[i] rows (M_i >= 0):
 *     out_i[M_i, N] = block-scaled product of A_i [M_i, K] and B_i [N, K]
 * Storage (all device memory owned by the caller):
 *   a       [max_rows, K] codes; group i's rows start at row R_i = sum_{j<i} M_j
 *   scale_a FP32 [S_rows, Kb] with group i's blocks starting at row
 *           S_i = sum_{j<i} ceil(M_j / gran); S_rows >= ceil(max_rows / gran)
 *           + num_groups covers every split of max_rows into groups
 *   b       [num_groups, N, K] codes; scale_b FP32 [num_groups, ceil(N/gran), Kb]
 *   out     [max_rows, N] BF16; rows R_i .. R_i + M_i - 1 are written, the
 *           rest untouched
 *   group_m int32 [num_groups] on the device, read by the kernel (so sizes
 *           produced on the GPU need no copy to the host)
 * sum M_i must not exceed max_rows: rows past max_rows are neither read
 * (they load as zeros) nor written, and scale reads stay inside the S_rows
 * bound above. The scale blocks never straddle groups.
 * Errors as bsgemm_fp8_gemm_fmt, plus BSGEMM_ERR_INVALID_ARG for
 * num_groups < 1 or max_rows < 1, BSGEMM_ERR_MISALIGNED for a group_m
 * pointer that is not 4-byte aligned. */
bsgemm_status bsgemm_fp8_grouped_nt(int a_format, int b_format, const void *a, const void *b,
                                    const float *scale_a, const float *scale_b, void *out,
                                    const int32_t *group_m, int num_groups, int64_t max_rows,
                                    int64_t N, int64_t K, int gran, bsgemm_stream_t stream);

/* Host-only: the plan a call with these sizes would use on a device with
 * `num_sms` SMs. Touches no device. */
bsgemm_status bsgemm_make_plan(int layout, int64_t M, int64_t N, int64_t K, int gran, int num_sms,
                               const bsgemm_tuning *tuning, bsgemm_plan *plan);

/* Human-readable name of a status code (static string, never NULL). */
const char *bsgemm_status_string(bsgemm_status status);

/* Synchronises `stream`, then returns and clears the device status word of
 * the current device: BSGEMM_OK, or BSGEMM_ERR_DEVICE_TIMEOUT if a bounded
 * wait ran out in any kernel since the last call. BSGEMM_ERR_CUDA if the
 * synchronisation itself failed. */
bsgemm_status bsgemm_get_last_device_status(bsgemm_stream_t stream);

/* Frees every split-K workspace the library holds on the current device
 * (those of destroyed streams included), after waiting for the device to
 * finish its work.  Later calls allocate again as needed.  Returns
 * BSGEMM_ERR_CUDA if the device wait or a free fails. */
bsgemm_status bsgemm_release_workspaces(void);

/* Raw device status word (0, or the timeout code in the low byte and the
 * place of the wait that gave up in bits 8..15), without clearing it. */
int bsgemm_last_device_status_detail(void);

/* Diagnostic: launches one CTA that waits on an mbarrier nothing completes,
 * with a wait limit of `timeout_ns` (1 ns .. 10 s). The wait must give up,
 * record BSGEMM_ERR_DEVICE_TIMEOUT and return; read it back with
 * bsgemm_get_last_device_status. Exercises the bounded-wait path of the
 * GEMM kernels without hanging or faulting the GPU. */
bsgemm_status bsgemm_diag_wait_timeout(unsigned long long timeout_ns, bsgemm_stream_t stream);

/* ---- allocation-free variant --------------------------------------------
 * The pages have no counterpart to this entry point; it serves callers that
 * cannot allocate device memory: code running inside an allocator callback,
 * under a framework that owns every byte of device memory and hands the
 * library only the tensors of the call, or in a process that must not grow
 * its device footprint after start-up.  The entry points above create their
 * split-K workspace with cudaMallocAsync on first use; this one never allocates
 * (no cudaMalloc, cudaFree or allocating library call, torch's included).
 *
 * It computes exactly what bsgemm_fp8_nt computes, with the same arguments,
 * rules and errors, and with the same single-CTA kernels.  It takes the same
 * plan when that plan's scratch fits the array; otherwise it keeps the plan's
 * variant and tile width, drops stream-K and lowers the split-K count until
 * the partial tiles fit (one split needs no scratch, so every problem
 * bsgemm_fp8_nt accepts runs here too, possibly with fewer K splits).  Where
 * the regular plan pairs CTAs (large g = 256 problems) it takes 128-row
 * data-parallel tiles instead.
 * Its split-K / stream-K scratch is a fixed array inside the library's device
 * memory: each GPU that loads the library holds BSGEMM_NOALLOC_SCRATCH_BYTES
 * of FP32 partial tiles plus BSGEMM_NOALLOC_MAX_TILES tile counters until the
 * process exits.  A plan needs split-K: tiles x splits partial tiles and one
 * counter per tile; stream-K: 2 x sk_ctas partial tiles and one counter per
 * stream-K tile; a partial tile is tile width x 128 x 4 bytes.  A launch
 * whose plan needed more than the array holds would be refused with
 * BSGEMM_ERR_SCRATCH_LIMIT before anything is launched; the plan choice
 * above keeps every plan within it.
 *
 * The first call on each device looks up the array's device address (once,
 * with that device current); make that first call before any stream capture.
 * Every call shares the array, which keeps the previous call's contents:
 * each call clears the tile counters on its stream before its kernel.  Calls
 * whose kernels overlap on the GPU (other streams, other host threads on the
 * same device) race on the array and corrupt each other's results, so the
 * caller must serialise them. */
#define BSGEMM_NOALLOC_SCRATCH_BYTES (16u << 20)
#define BSGEMM_NOALLOC_MAX_TILES 4096

bsgemm_status bsgemm_fp8_nt_noalloc(const void *a, const void *b, const float *scale_a,
                                    const float *scale_b, void *out, int64_t M, int64_t N,
                                    int64_t K, int gran, bsgemm_stream_t stream);

/* Library version as major*10000 + minor*100 + patch. */
int bsgemm_version(void);

#ifdef __cplusplus
}
#endif

#endif /* BSGEMM_H */
