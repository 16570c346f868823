/*
 * Plain CPU oracle for block-scaled FP8 GEMM.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may call, link or load
 * this file: only the tests, the smoke check and the bench's CPU-baseline leg
 * use it. It shares no code, header, table or constant with the CUDA library.
 *
 * What it computes (hncyxsy.com/news/191052, "DeepGEMM实战: FP8矩阵乘法加速与
 * Hopper架构优化指南"):
 *   - inputs are FP8 E4M3 codes, accumulation is FP32 or wider (§2.2, §3.2);
 *   - each operand carries one FP32 scale per g x g block, g in {64,128,256},
 *     default 128 (§2.2, §3.1 table);
 *   - dequantisation multiplies by the scale (§5.2: "quantise divides,
 *     dequantise multiplies");
 *   - K is cut into segments that are accumulated separately and then added
 *     (§3.2), which is where the per-block scales enter;
 *   - out is BF16 [M,N], A is [M,K] and B is [N,K] in the "NT" layout, and the
 *     NT/TN/NN/TT flags say how A and B are stored (§3.3, §4.2).
 *
 * The exact definition written out here, for every (m, n):
 *
 *   ref[m,n] = sum_{kb=0}^{Kb-1} sA[m/g][kb] * sB[n/g][kb]
 *                                * sum_{k in block kb} dec(A[m,k]) * dec(B[n,k])
 *   out[m,n] = bf16_rne(ref[m,n])          (one rounding, straight from FP64)
 *
 * The pages name two FP8 formats, E4M3 and E5M2 (§2.2); either operand may
 * use either one (the _fmt entry points; the plain ones are E4M3 x E4M3).
 *
 * Arithmetic, chosen so that every step is exact or one FP64 rounding:
 *   - dec(code) is an integer count of the format's smallest subnormal:
 *     2^-9 for E4M3 (|value| <= 448 = 229376 * 2^-9), 2^-16 for E5M2
 *     (|value| <= 57344 = 7 * 2^29 * 2^-16);
 *   - the inner block sum is an exact 128-bit integer count of
 *     2^-(qa + qb) (qa, qb = 9 or 16): |product| < 2^64, at most 256 terms;
 *   - the block sum is converted to FP64: exact for E4M3 x E4M3 (|sum| <
 *     2^44), otherwise exact whenever it has at most 53 significant bits and
 *     else one rounding of relative size <= 2^-53;
 *   - sA*sB is exact in FP64 (24 + 24 significant bits <= 53);
 *   - term = blocksum * 2^-(qa+qb) * (sA*sB) is one FP64 rounding, and the
 *     terms are added in ascending kb in FP64.
 *
 * Readings of points the pages leave open: both operands use g x g blocks; the scale tensors are
 * row-major FP32 [ceil(rows/g)][ceil(K/g)] in logical block coordinates for
 * every storage layout; a partial last block (rows or K not a multiple of g)
 * simply has fewer terms; for the layout flags the first letter is A and the
 * second is B, "N" for A means stored [M,K], "T" for A means stored [K,M],
 * "T" for B means stored [N,K] and "N" for B means stored [K,N].
 *
 * parity pins: see tests/test_oracle_pins.py (closed forms, power-of-two
 * invariants, exact-rational brute force, hand-worked cases in tests/golden/).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define OR_LAYOUT_NT 0
#define OR_LAYOUT_TN 1
#define OR_LAYOUT_NN 2
#define OR_LAYOUT_TT 3

#define OR_OK 0
#define OR_ERR_ARG 1
#define OR_ERR_NAN_INPUT 2

/* ---- E4M3 ("fn": no infinities) decode -------------------------------------
 * Bit layout: s eeee mmm, exponent bias 7.
 *   eeee == 0            : subnormal, value = (-1)^s * m/8 * 2^-6 = m * 2^-9
 *   eeee == 1111, mmm=111: NaN (the only non-finite code)
 *   otherwise            : value = (-1)^s * (1 + m/8) * 2^(e-7)
 *                                = (-1)^s * (8 + m) * 2^(e-1) * 2^-9
 * The result is the value as a signed integer count of 2^-9.               */
static int e4m3_units(uint8_t code, int64_t *units)
{
    int s = code >> 7;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    int64_t mag;
    if (e == 0xF && m == 0x7)
        return 0; /* NaN */
    if (e == 0)
        mag = m;
    else
        mag = (int64_t)(8 + m) << (e - 1);
    *units = s ? -mag : mag;
    return 1;
}

/* ---- E5M2 (IEEE-like: infinities and NaNs) decode ---------------------------
 * Bit layout: s eeeee mm, exponent bias 15.
 *   eeeee == 0      : subnormal, value = (-1)^s * m/4 * 2^-14 = m * 2^-16
 *   eeeee == 11111  : +-Inf (mm == 0) or NaN (mm != 0)
 *   otherwise       : value = (-1)^s * (1 + m/4) * 2^(e-15)
 *                           = (-1)^s * (4 + m) * 2^(e-1) * 2^-16
 * The result is the value as a signed integer count of 2^-16.              */
static int e5m2_units(uint8_t code, int64_t *units)
{
    int s = code >> 7;
    int e = (code >> 2) & 0x1F;
    int m = code & 0x3;
    int64_t mag;
    if (e == 0x1F)
        return 0; /* Inf or NaN: not a finite input */
    if (e == 0)
        mag = m;
    else
        mag = (int64_t)(4 + m) << (e - 1);
    *units = s ? -mag : mag;
    return 1;
}

#define OR_FMT_E4M3 0
#define OR_FMT_E5M2 1

/* Decode one code of format fmt: units of 2^-quantum_log2(fmt). */
static inline int fp8_units(int fmt, uint8_t code, int64_t *units)
{
    return fmt == OR_FMT_E5M2 ? e5m2_units(code, units) : e4m3_units(code, units);
}

static inline int quantum_log2(int fmt)
{
    return fmt == OR_FMT_E5M2 ? 16 : 9;
}

/* Value of one E4M3 code as a double (NaN for the NaN codes). */
double oracle_e4m3_value(uint8_t code)
{
    int64_t u;
    if (!e4m3_units(code, &u))
        return NAN;
    return ldexp((double)u, -9);
}

/* Value of one code of format fmt (0 E4M3, 1 E5M2) as a double. E5M2's
 * infinities decode to +-Inf and its NaN codes to NaN.                     */
double oracle_fp8_value(int fmt, uint8_t code)
{
    int64_t u = 0;
    if (fmt == OR_FMT_E5M2) {
        if (((code >> 2) & 0x1F) == 0x1F)
            return (code & 0x3) ? NAN : ((code >> 7) ? -INFINITY : INFINITY);
        e5m2_units(code, &u);
        return ldexp((double)u, -16);
    }
    return oracle_e4m3_value(code);
}

/* ---- FP64 -> BF16, round to nearest, ties to even --------------------------
 * BF16 keeps 8 significant bits and FP32's exponent range (normal minimum
 * 2^-126, subnormal quantum 2^-133, largest finite (2 - 2^-7) * 2^127).
 * The rounding is done once, on the exact double, with no detour through
 * FP32 (which would round twice).                                         */
uint16_t oracle_bf16_rne(double x)
{
    double r;
    float f;
    uint32_t bits;
    if (isnan(x))
        return 0x7FC0;
    if (x == 0.0)
        return signbit(x) ? 0x8000 : 0x0000;
    if (isinf(x))
        return signbit(x) ? 0xFF80 : 0x7F80;
    if (fabs(x) < ldexp(1.0, -126)) {
        /* subnormal range: quantum 2^-133 */
        r = ldexp(nearbyint(ldexp(x, 133)), -133);
    } else {
        int e;
        double fr = frexp(x, &e);            /* x = fr * 2^e, 0.5 <= |fr| < 1 */
        double q = nearbyint(ldexp(fr, 8));  /* 8 significant bits, ties-to-even */
        r = ldexp(q, e - 8);                 /* q == +-256 carries into the next binade */
    }
    if (fabs(r) > ldexp(255.0, 120)) /* 255 * 2^120 = (2 - 2^-7) * 2^127 */
        r = x > 0 ? INFINITY : -INFINITY;
    f = (float)r; /* exact: r has <= 8 significant bits in FP32's range */
    memcpy(&bits, &f, sizeof bits);
    return (uint16_t)(bits >> 16);
}

/* ---- element access by layout (§3.3 / §4.2 flags) ---------------------- */
static inline uint8_t elem_a(int layout, const uint8_t *a, int64_t M, int64_t K, int64_t m, int64_t k)
{
    /* first letter: N -> A stored [M,K]; T -> A stored [K,M] */
    if (layout == OR_LAYOUT_NT || layout == OR_LAYOUT_NN)
        return a[m * K + k];
    return a[k * M + m];
}

static inline uint8_t elem_b(int layout, const uint8_t *b, int64_t N, int64_t K, int64_t n, int64_t k)
{
    /* second letter: T -> B stored [N,K]; N -> B stored [K,N] */
    if (layout == OR_LAYOUT_NT || layout == OR_LAYOUT_TT)
        return b[n * K + k];
    return b[k * N + n];
}

/* One output element: the definition above, term by term.
 * Returns 0 on success, OR_ERR_NAN_INPUT if a non-finite code was met.   */
static int one_element(int layout, int fa, int fb, const uint8_t *a, const uint8_t *b,
                       const float *sa, const float *sb, int64_t M, int64_t N, int64_t K,
                       int64_t g, int64_t m, int64_t n, double *ref)
{
    int64_t Kb = (K + g - 1) / g;
    int shift = quantum_log2(fa) + quantum_log2(fb);
    double acc = 0.0;
    for (int64_t kb = 0; kb < Kb; ++kb) {
        int64_t k0 = kb * g;
        int64_t k1 = k0 + g < K ? k0 + g : K;
        __int128 blocksum = 0; /* exact, units of 2^-shift */
        for (int64_t k = k0; k < k1; ++k) {
            int64_t ua, ub;
            if (!fp8_units(fa, elem_a(layout, a, M, K, m, k), &ua) ||
                !fp8_units(fb, elem_b(layout, b, N, K, n, k), &ub)) {
                *ref = NAN;
                return OR_ERR_NAN_INPUT;
            }
            blocksum += (__int128)ua * ub;
        }
        double scale = (double)sa[(m / g) * Kb + kb] * (double)sb[(n / g) * Kb + kb]; /* exact */
        acc += ldexp((double)blocksum, -shift) * scale;
    }
    *ref = acc;
    return OR_OK;
}

static int check_args(int layout, const void *a, const void *b, const float *sa, const float *sb,
                      int64_t M, int64_t N, int64_t K, int64_t g)
{
    if (layout < OR_LAYOUT_NT || layout > OR_LAYOUT_TT)
        return OR_ERR_ARG;
    if (!a || !b || !sa || !sb || M <= 0 || N <= 0 || K <= 0 || g <= 0)
        return OR_ERR_ARG;
    return OR_OK;
}

/* Full output. ref: FP64 [M*N] (may be NULL); out: BF16 bits [M*N] (may be NULL).
 * Parallel over rows with OpenMP when compiled with it; each element is
 * computed independently, so the result does not depend on the thread count. */
int oracle_bsgemm_fmt(int layout, int fa, int fb, const uint8_t *a, const uint8_t *b,
                      const float *sa, const float *sb, int64_t M, int64_t N, int64_t K, int64_t g,
                      double *ref, uint16_t *out)
{
    int rc = check_args(layout, a, b, sa, sb, M, N, K, g);
    int bad = 0;
    if (rc)
        return rc;
    if ((fa != OR_FMT_E4M3 && fa != OR_FMT_E5M2) || (fb != OR_FMT_E4M3 && fb != OR_FMT_E5M2))
        return OR_ERR_ARG;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t n = 0; n < N; ++n) {
            double r;
            bad |= one_element(layout, fa, fb, a, b, sa, sb, M, N, K, g, m, n, &r);
            if (ref)
                ref[m * N + n] = r;
            if (out)
                out[m * N + n] = oracle_bf16_rne(r);
        }
    }
    return bad ? OR_ERR_NAN_INPUT : OR_OK;
}

/* Selected outputs only: element i is (mi[i], ni[i]). For parity checks at
 * sizes where the full product would take the oracle too long.            */
int oracle_bsgemm_at_fmt(int layout, int fa, int fb, const uint8_t *a, const uint8_t *b,
                         const float *sa, const float *sb, int64_t M, int64_t N, int64_t K,
                         int64_t g, int64_t count, const int64_t *mi, const int64_t *ni,
                         double *ref, uint16_t *out)
{
    int rc = check_args(layout, a, b, sa, sb, M, N, K, g);
    int bad = 0;
    if (rc)
        return rc;
    if ((fa != OR_FMT_E4M3 && fa != OR_FMT_E5M2) || (fb != OR_FMT_E4M3 && fb != OR_FMT_E5M2))
        return OR_ERR_ARG;
    if (count < 0 || (count > 0 && (!mi || !ni)))
        return OR_ERR_ARG;
    for (int64_t i = 0; i < count; ++i)
        if (mi[i] < 0 || mi[i] >= M || ni[i] < 0 || ni[i] >= N)
            return OR_ERR_ARG;
#pragma omp parallel for schedule(dynamic, 16) reduction(| : bad)
    for (int64_t i = 0; i < count; ++i) {
        double r;
        bad |= one_element(layout, fa, fb, a, b, sa, sb, M, N, K, g, mi[i], ni[i], &r);
        if (ref)
            ref[i] = r;
        if (out)
            out[i] = oracle_bf16_rne(r);
    }
    return bad ? OR_ERR_NAN_INPUT : OR_OK;
}

/* E4M3 x E4M3 forms of the two entry points above. */
int oracle_bsgemm(int layout, const uint8_t *a, const uint8_t *b, const float *sa, const float *sb,
                  int64_t M, int64_t N, int64_t K, int64_t g, double *ref, uint16_t *out)
{
    return oracle_bsgemm_fmt(layout, OR_FMT_E4M3, OR_FMT_E4M3, a, b, sa, sb, M, N, K, g, ref, out);
}

int oracle_bsgemm_at(int layout, const uint8_t *a, const uint8_t *b, const float *sa,
                     const float *sb, int64_t M, int64_t N, int64_t K, int64_t g, int64_t count,
                     const int64_t *mi, const int64_t *ni, double *ref, uint16_t *out)
{
    return oracle_bsgemm_at_fmt(layout, OR_FMT_E4M3, OR_FMT_E4M3, a, b, sa, sb, M, N, K, g, count,
                                mi, ni, ref, out);
}

/* Number of OpenMP threads the oracle would use (1 without OpenMP). */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ---- per-block FP8 quantisation (§4.4 granularity must match, §5.2
 * "quantise divides, dequantise multiplies") ------------------------------
 * For each g x g block of a row-major [rows, cols] FP32 matrix x:
 *   amax  = max |x| over the block's elements (partial blocks: the elements
 *           that exist);
 *   s     = amax / FMAX in FP32 (FMAX = 448 for E4M3, 57344 for E5M2), or
 *           1.0 when amax is 0;
 *   q     = the format's code nearest to the FP32 quotient x / s, ties to the
 *           code with an even mantissa, saturating to +-FMAX.
 * FP32 arithmetic is used for s and x / s because that is where the decision
 * of each integer code is taken; it is IEEE division, correctly rounded.   */
/* Nearest finite code to v (finite FP32), ties to even mantissa, saturating. */
uint8_t oracle_fp8_encode(int fmt, float v)
{
    double fmax = fmt == OR_FMT_E5M2 ? 57344.0 : 448.0;
    double x = (double)v; /* exact */
    int neg = signbit(x) ? 1 : 0;
    double ax = fabs(x);
    int best = -1;
    double best_err = 0.0;
    if (ax >= fmax)
        ax = fmax;
    /* non-negative codes 0x00..0x7F: finite ones, increasing in value */
    for (int c = 0; c < 0x80; ++c) {
        double cv = oracle_fp8_value(fmt, (uint8_t)c);
        double err;
        if (!isfinite(cv))
            continue;
        err = fabs(cv - ax);
        /* a tie is between two neighbouring codes; the even one (mantissa
         * LSB = code LSB = 0) wins */
        if (best < 0 || err < best_err || (err == best_err && (c & 1) == 0)) {
            best = c;
            best_err = err;
        }
    }
    if (neg)
        best |= 0x80; /* the sign is kept, zero included */
    return (uint8_t)best;
}

int oracle_quantize_blocks(int fmt, const float *x, int64_t rows, int64_t cols, int64_t g,
                           uint8_t *q, float *scales)
{
    int64_t Rb, Cb;
    float fmax;
    if ((fmt != OR_FMT_E4M3 && fmt != OR_FMT_E5M2) || !x || !q || !scales || rows <= 0 ||
        cols <= 0 || g <= 0)
        return OR_ERR_ARG;
    Rb = (rows + g - 1) / g;
    Cb = (cols + g - 1) / g;
    fmax = fmt == OR_FMT_E5M2 ? 57344.0f : 448.0f;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t blk = 0; blk < Rb * Cb; ++blk) {
        int64_t rb = blk / Cb, cb = blk % Cb;
        int64_t r0 = rb * g, r1 = r0 + g < rows ? r0 + g : rows;
        int64_t c0 = cb * g, c1 = c0 + g < cols ? c0 + g : cols;
        float amax = 0.0f, s;
        for (int64_t r = r0; r < r1; ++r)
            for (int64_t c = c0; c < c1; ++c) {
                float a = fabsf(x[r * cols + c]);
                if (a > amax)
                    amax = a;
            }
        s = amax > 0.0f ? amax / fmax : 1.0f;
        scales[rb * Cb + cb] = s;
        for (int64_t r = r0; r < r1; ++r)
            for (int64_t c = c0; c < c1; ++c)
                q[r * cols + c] = oracle_fp8_encode(fmt, x[r * cols + c] / s);
    }
    return OR_OK;
}

/* ---- fused epilogue (§2.3, §6: bias and activation applied before the
 * result is written back) ----------------------------------------------------
 *   v[m,n] = act(ref[m,n] + bias[n])      in FP64, bias may be NULL
 *   act: 0 none, 1 ReLU = max(v, 0), 2 GELU = 0.5 v (1 + erf(v / sqrt 2))
 * epi_ref receives v (FP64); out receives bf16_rne(v) (may be NULL).      */
int oracle_epilogue(const double *ref, int64_t M, int64_t N, const float *bias, int act,
                    double *epi_ref, uint16_t *out)
{
    if (!ref || !epi_ref || M <= 0 || N <= 0 || act < 0 || act > 2)
        return OR_ERR_ARG;
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double v = ref[m * N + n] + (bias ? (double)bias[n] : 0.0);
            if (act == 1)
                v = v > 0.0 ? v : 0.0;
            else if (act == 2)
                v = 0.5 * v * (1.0 + erf(v / sqrt(2.0)));
            epi_ref[m * N + n] = v;
            if (out)
                out[m * N + n] = oracle_bf16_rne(v);
        }
    return OR_OK;
}
