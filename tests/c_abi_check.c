/*
 * A plain C11 caller of the library, built against the three public headers
 * and linked with liblittlebit.so.  It makes only calls that end in the
 * library's host-side argument checks, so it runs without a GPU; it shows
 * that the headers are valid C, that the symbols link from C, and that the
 * status codes documented in the headers come back through the C ABI.
 * Prints "OK" and exits 0 when every check holds.
 */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "littlebit.h"
#include "littlebit_backward.h"
#include "littlebit_init.h"

static int fails = 0;
#define CHECK(c)                                                                  \
    do {                                                                          \
        if (!(c)) {                                                               \
            printf("FAIL line %d: %s\n", __LINE__, #c);                           \
            ++fails;                                                              \
        }                                                                         \
    } while (0)

int main(void)
{
    /* status strings and the packed layout size */
    CHECK(strcmp(lb_status_string(LB_OK), "LB_OK") == 0);
    CHECK(strstr(lb_status_string(LB_ERR_INVALID_ARG), "INVALID") != NULL);
    CHECK(lb_packed_words(10, 33) == 20);
    CHECK(lb_packed_words(-1, 3) == 0);

    /* packing: invalid sizes, an empty request, a misaligned factor */
    CHECK(lb_pack_signs(NULL, -1, 4, NULL, NULL) == LB_ERR_INVALID_ARG);
    CHECK(lb_pack_signs(NULL, 3, 0, NULL, NULL) == LB_ERR_INVALID_ARG);
    CHECK(lb_pack_signs(NULL, 0, 4, NULL, NULL) == LB_OK);
    CHECK(lb_pack_signs((const float *)(uintptr_t)2, 5, 4, (uint32_t *)(uintptr_t)64, NULL) == LB_ERR_INVALID_ARG);

    /* layers and stacks */
    lb_layer *L = NULL;
    CHECK(lb_layer_create(&L, 8, 8, 4, 3, NULL, NULL, NULL, NULL, NULL, NULL) == LB_ERR_UNSUPPORTED);
    CHECK(lb_layer_create(&L, 0, 8, 4, 2, NULL, NULL, NULL, NULL, NULL, NULL) == LB_ERR_INVALID_ARG);
    CHECK(lb_layer_create(&L, 8, 8, LB_MAX_RANK + 1, 2, NULL, NULL, NULL, NULL, NULL, NULL) == LB_ERR_INVALID_ARG);
    CHECK(lb_layer_create(NULL, 8, 8, 4, 2, NULL, NULL, NULL, NULL, NULL, NULL) == LB_ERR_INVALID_ARG);
    CHECK(L == NULL);
    CHECK(lb_linear_forward(NULL, 1, NULL, NULL, NULL) == LB_ERR_INVALID_ARG);
    lb_stack *S = NULL;
    CHECK(lb_stack_create(&S, NULL, 0, NULL) == LB_ERR_INVALID_ARG);
    CHECK(lb_stack_forward(NULL, NULL, NULL, 1, NULL) == LB_ERR_INVALID_ARG);
    CHECK(lb_layer_bpw(NULL) == 0.0);
    lb_layer_destroy(NULL);
    lb_stack_destroy(NULL);

    /* initialisation: workspace sizes and argument checks */
    CHECK(lb_dual_svid_workspace_bytes(8, 8, 9) == 0);
    const size_t ws = lb_dual_svid_workspace_bytes(96, 40, 6);
    CHECK(ws > (size_t)96 * 40 * 8);
    CHECK(lb_littlebit2_workspace_bytes(96, 40, 6) > ws);
    void *dev = (void *)(uintptr_t)256;
    uint32_t *const u1[1] = {(uint32_t *)dev};
    float *const f1[1] = {(float *)dev};
    CHECK(lb_dual_svid_init((const float *)dev, 96, 40, 6, 3, 24, u1, u1, f1, f1, f1, NULL, dev, ws, NULL) ==
          LB_ERR_UNSUPPORTED);
    CHECK(lb_dual_svid_init(NULL, 96, 40, 6, 1, 24, u1, u1, f1, f1, f1, NULL, dev, ws, NULL) == LB_ERR_INVALID_ARG);
    CHECK(lb_dual_svid_init((const float *)dev, 96, 40, 6, 1, 24, u1, u1, f1, f1, f1, NULL, dev, ws - 8, NULL) ==
          LB_ERR_INVALID_ARG);

    /* QAT backward */
    const uint32_t *const cu1[1] = {(const uint32_t *)dev};
    const uint16_t *const ch1[1] = {(const uint16_t *)dev};
    lb_backward *B = NULL;
    CHECK(lb_backward_create(NULL, 64, 64, 8, 1, cu1, cu1, ch1, ch1, ch1, NULL) == LB_ERR_INVALID_ARG);
    CHECK(lb_backward_create(&B, 64, 64, 8, 3, cu1, cu1, ch1, ch1, ch1, NULL) == LB_ERR_UNSUPPORTED);
    CHECK(lb_backward_create(&B, 64, 60, 8, 1, cu1, cu1, ch1, ch1, ch1, NULL) == LB_ERR_UNSUPPORTED);
    lb_backward_destroy(NULL);
    /* its dense-product GEMM: argument checks happen before any device work */
    const uint16_t *h16 = (const uint16_t *)dev;
    float *f32 = (float *)dev;
    CHECK(lb_gemm_at_b(NULL, 64, h16, 64, f32, 64, 8, 64, 64, (const float *)dev, (int *)dev, NULL) ==
          LB_ERR_INVALID_ARG);
    CHECK(lb_gemm_at_b(h16, 64, h16, 48, f32, 48, 8, 64, 48, (const float *)dev, (int *)dev, NULL) ==
          LB_ERR_UNSUPPORTED);
    CHECK(lb_gemm_at_b(h16, 64, h16, 64, f32, 64, 8, 0, 64, (const float *)dev, (int *)dev, NULL) == LB_OK);

    printf(fails ? "FAILED (%d)\n" : "OK\n", fails);
    return fails != 0;
}
