/*
 * A plain C99 client of the library: it includes only bsgemm.h, links
 * libbsgemm.so, and calls the entry points that run on the host alone (plan,
 * status strings, version, and argument checks that return before any CUDA
 * call). tests/test_abi_c_client.py compiles it with -std=c99 -pedantic
 * -Werror and runs it without a GPU. Exit status 0 means every check passed.
 */
#include <stdio.h>
#include <string.h>

#include "bsgemm.h"

static int failures = 0;

#define CHECK(cond)                                                       \
    do {                                                                  \
        if (!(cond)) {                                                    \
            fprintf(stderr, "%s:%d: check failed: %s\n", __FILE__, __LINE__, #cond); \
            ++failures;                                                   \
        }                                                                 \
    } while (0)

int main(void)
{
    bsgemm_plan plan;
    bsgemm_tuning tuning;
    bsgemm_epilogue epi;
    /* a 16-byte aligned stand-in address: the checks below reject the call
     * before anything is dereferenced or launched */
    static float dummy[64] __attribute__((aligned(16)));
    const void *p = dummy;
    int code;

    CHECK(bsgemm_version() > 0); /* major*10000 + minor*100 + patch */

    for (code = BSGEMM_OK; code <= BSGEMM_ERR_SCRATCH_LIMIT; ++code) {
        const char *s = bsgemm_status_string((bsgemm_status)code);
        CHECK(s != NULL && strlen(s) > 0);
    }
    CHECK(bsgemm_status_string((bsgemm_status)99) != NULL);

    /* the square 4096^3 NT g=128 plan on 148 SMs: 128 x 256 tiles, one wave of
     * persistent CTAs, no split */
    memset(&plan, 0, sizeof plan);
    CHECK(bsgemm_make_plan(BSGEMM_LAYOUT_NT, 4096, 4096, 4096, 128, 148, NULL, &plan) == BSGEMM_OK);
    CHECK(plan.swap_ab == 0 && plan.bnq == 256);
    CHECK(plan.tiles_p == 32 && plan.tiles_q == 16);
    CHECK(plan.splits == 1 && plan.grid == 148 && plan.kernels == 1);

    /* decode-sized M goes to swap-AB */
    CHECK(bsgemm_make_plan(BSGEMM_LAYOUT_NT, 1, 7168, 7168, 128, 148, NULL, &plan) == BSGEMM_OK);
    CHECK(plan.swap_ab == 1 && plan.bnq == 16);

    /* tuning: forced CTA pairs, and a rejected combination */
    memset(&tuning, 0, sizeof tuning);
    tuning.variant = BSGEMM_VARIANT_CTA_PAIR;
    CHECK(bsgemm_make_plan(BSGEMM_LAYOUT_TN, 4096, 4096, 4096, 256, 148, &tuning, &plan) == BSGEMM_OK);
    CHECK(plan.cta_pair == 1 && plan.tiles_p == 16 && plan.tiles_q == 16);
    tuning.splits = 2;
    CHECK(bsgemm_make_plan(BSGEMM_LAYOUT_NT, 4096, 4096, 4096, 128, 148, &tuning, &plan) ==
          BSGEMM_ERR_INVALID_ARG);

    /* host-side argument errors, reported before any launch */
    CHECK(bsgemm_make_plan(BSGEMM_LAYOUT_NT, 256, 256, 256, 96, 148, NULL, &plan) ==
          BSGEMM_ERR_UNSUPPORTED_GRAN);
    CHECK(bsgemm_make_plan(BSGEMM_LAYOUT_NT, 0, 256, 256, 128, 148, NULL, &plan) == BSGEMM_ERR_INVALID_ARG);
    CHECK(bsgemm_fp8_nt(NULL, p, p, p, dummy, 16, 16, 16, 128, NULL) == BSGEMM_ERR_INVALID_ARG);
    CHECK(bsgemm_fp8_nt(p, p, p, p, dummy, 16, 16, 16, 32, NULL) == BSGEMM_ERR_UNSUPPORTED_GRAN);
    CHECK(bsgemm_fp8_nt(p, p, p, p, dummy, 16, 16, 24, 128, NULL) == BSGEMM_ERR_MISALIGNED); /* K % 16 */
    CHECK(bsgemm_fp8_tn(p, p, p, p, dummy, 8, 16, 16, 128, NULL) == BSGEMM_ERR_MISALIGNED);  /* M % 16 */
    CHECK(bsgemm_fp8_nn(p, p, p, p, dummy, 16, 8, 16, 128, NULL) == BSGEMM_ERR_MISALIGNED);  /* N % 16 */
    CHECK(bsgemm_fp8_tt(p, p, p, p, dummy, 16, 12, 16, 128, NULL) == BSGEMM_ERR_MISALIGNED); /* N % 8 */
    CHECK(bsgemm_fp8_gemm_fmt(BSGEMM_LAYOUT_NT, 2, BSGEMM_FP8_E4M3, p, p, p, p, dummy, 16, 16, 16, 128,
                              NULL, NULL) == BSGEMM_ERR_INVALID_ARG);
    memset(&epi, 0, sizeof epi);
    epi.activation = 7;
    CHECK(bsgemm_fp8_gemm_fused(BSGEMM_LAYOUT_NT, BSGEMM_FP8_E4M3, BSGEMM_FP8_E4M3, p, p, p, p, &epi,
                                dummy, 16, 16, 16, 128, NULL, NULL) == BSGEMM_ERR_INVALID_ARG);
    CHECK(bsgemm_fp8_grouped_nt(BSGEMM_FP8_E4M3, BSGEMM_FP8_E4M3, p, p, p, p, dummy, NULL, 1, 16, 16, 16,
                                128, NULL) == BSGEMM_ERR_INVALID_ARG);
    CHECK(bsgemm_quantize_fp8(BSGEMM_SRC_F32, BSGEMM_FP8_E4M3, p, 16, 16, 100, dummy, dummy, NULL) ==
          BSGEMM_ERR_UNSUPPORTED_GRAN);
    CHECK(bsgemm_fp8_nt_noalloc(p, p, NULL, p, dummy, 16, 16, 16, 128, NULL) == BSGEMM_ERR_INVALID_ARG);

    if (failures == 0)
        printf("abi_c_client: all checks passed\n");
    return failures == 0 ? 0 : 1;
}
