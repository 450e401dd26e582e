/* A plain C99 consumer of the C ABI: includes include/razer.h, links
 * librazer.so and exercises the host-side calls (no GPU is needed: every
 * call below returns before any launch).  Exit status 0 when all checks hold. */
#include <stdio.h>
#include <string.h>

#include "razer.h"

static int failures = 0;

static void check(int cond, const char *what)
{
    if (!cond) {
        fprintf(stderr, "FAILED: %s\n", what);
        failures++;
    }
}

int main(void)
{
    check(razer_version() >= 100, "version");
    check(strcmp(razer_status_string(RAZER_ERR_ALIGN), "misaligned pointer") == 0, "status string");
    /* GEMV workspace: 0 for empty sizes, positive for a decode shape */
    check(razer_workspace_size(RAZER_OP_GEMV, 1, 0, 4096) == 0, "empty GEMV workspace");
    check(razer_workspace_size(RAZER_OP_GEMV, 1, 4096, 4096) > 0, "GEMV workspace");
    /* argument validation before any launch */
    unsigned char buf[64];
    void *p = (void *)(((size_t)buf + 15) & ~(size_t)15);
    check(razer_gemv(p, RAZER_F16, 1, p, p, NULL, RAZER_FMT_WEIGHT, 64, 128, p, RAZER_F32, NULL, 0, NULL) ==
              RAZER_ERR_INVALID_ARG,
          "gemv without ts");
    check(razer_gemv(p, RAZER_F16, 33, p, p, (const float *)p, RAZER_FMT_WEIGHT, 64, 128, p, RAZER_F32, NULL, 0, NULL) ==
              RAZER_ERR_SHAPE,
          "gemv with B = 33");
    check(razer_quantize_weights(p, RAZER_F16, 4, 24, p, p, (float *)p, RAZER_FMT_WEIGHT, NULL) == RAZER_ERR_SHAPE,
          "quantize with K % 16 != 0");
    const float v[2] = {5.0f, 3.0f}; /* 3 is an E2M1 magnitude: not a special value */
    check(razer_quantize_variant(p, RAZER_F16, 4, 128, 32, RAZER_FMT_WEIGHT, v, 2, p, p, (float *)p, NULL) ==
              RAZER_ERR_INVALID_ARG,
          "variant with a grid value");
    if (failures == 0) printf("abi consumer: all checks passed\n");
    return failures ? 1 : 0;
}
