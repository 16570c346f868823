/* Exhaustive check of the quantiser's fast quotient for BF16 input.
 *
 * The GPU quantiser divides every element x of a block by the block's scale
 * s = RN(amax / FMAX). For BF16 input with s >= 2^-60 it does not divide.
 * It applies Markstein's correction step to the correctly rounded
 * reciprocal rs = RN(1 / s), with the residual taken negated:
 *     q0 = RN(x * rs);  en = RN(fma(q0, s, -x));  q = RN(fma(-en, rs, q0))
 * (en = q0 * s - x is exact where it matters; negated, the correction keeps
 * the sign of a zero x: -0 gives -0)
 * This program runs those steps in IEEE single precision for every finite
 * BF16 amax >= 0 and every BF16 x of either sign with |x| <= amax, for E4M3
 * (FMAX 448) and E5M2 (FMAX 57344). It checks q against the correctly rounded
 * RN(x / s):
 *   - where |x / s| >= 2^-18: bit for bit;
 *   - below that: |q| < 2^-17 with the same sign. Both FP8 formats then give
 *     the code +-0 for both values: the smallest E5M2 step is 2^-16, and the
 *     smallest E4M3 step is 2^-9.
 * Blocks with s < 2^-60 keep the division in the kernel and are skipped here.
 * Exit status 0 means no pair differs. Build with -ffp-contract=off, so the
 * compiler keeps every product and sum rounded on its own.
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

static float from_bf16(uint32_t b) {
  uint32_t u = b << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

static uint32_t bits_of(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  return u;
}

int main(void) {
  const float fmax_of[2] = {448.0f, 57344.0f};
  int failed = 0;
  for (int fi = 0; fi < 2; ++fi) {
    const float fmax_v = fmax_of[fi];
    long long bad = 0, pairs = 0, divided = 0;
#pragma omp parallel for schedule(dynamic, 64) reduction(+ : bad, pairs, divided)
    for (uint32_t ab = 0; ab < 0x7F80u; ++ab) {   /* every finite BF16 amax */
      const float amax = from_bf16(ab);
      volatile float fm = fmax_v;                  /* a run-time division */
      const float s = amax > 0.0f ? amax / fm : 1.0f;   /* an all-zero block takes s = 1 */
      if (!(s >= 0x1p-60f)) {
        divided++;
        continue;
      }
      volatile float one = 1.0f;
      const float rs = one / s;
      for (uint32_t xb = 0; xb <= ab; ++xb) {
        for (int neg = 0; neg < 2; ++neg) {
          const float x = from_bf16(xb | (neg ? 0x8000u : 0u));
          volatile float sv = s;
          const float want = x / sv;
          const float q0 = x * rs;
          const float en = fmaf(q0, s, -x);
          const float q = fmaf(-en, rs, q0);
          pairs++;
          int same;
          if (fabsf(want) >= 0x1p-18f)
            same = bits_of(q) == bits_of(want);
          else
            same = fabsf(q) < 0x1p-17f && (signbit(q) != 0) == (signbit(want) != 0);
          if (!same) {
            bad++;
            if (bad <= 4)
              printf("FMAX %g: amax %a x %a: x/s %a, fast %a\n", fmax_v, amax, x, want, q);
          }
        }
      }
    }
    printf("FMAX %g: %lld pairs, %lld differ; %lld amax values left to the division\n", fmax_v,
           pairs, bad, divided);
    failed |= bad != 0 || pairs < 900000000LL;
  }
  return failed;
}
