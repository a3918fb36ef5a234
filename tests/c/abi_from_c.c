/* The C ABI of libmoe_dispatch.so used from plain C (no C++, no Python):
 * compiled with a C compiler against include/moe_dispatch.h and linked to the
 * library.  Exercises only calls that return before touching a device: the
 * size helpers, the strings, and the host-side argument checks (fake,
 * never-dereferenced addresses).  Exit status 0 = every check held. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "moe_dispatch.h"

static int failures = 0;

#define CHECK(cond)                                                        \
    do {                                                                   \
        if (!(cond)) {                                                     \
            fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #cond); \
            ++failures;                                                    \
        }                                                                  \
    } while (0)

int main(void) {
    void* const A = (void*)(uintptr_t)0x10000;     /* aligned, never dereferenced */
    cudaStream_t s = NULL;

    /* sizes */
    CHECK(moe_worst_case_rows(16384, 8, 128, 16) == 16384LL * 8 + 128 * 15);
    CHECK(moe_worst_case_rows(10, 0, 8, 8) == -1);
    CHECK(moe_layout_workspace_bytes(16384, 8, 128, 8) > 16384u * 8 * 2);
    CHECK(moe_layout_workspace_bytes(64, 2, 7, 2) == 0);          /* E % R */
    CHECK(moe_layout_workspace_bytes(64, 2, 8, 2) % 256 == 0);

    /* strings */
    CHECK(strcmp(moe_strerror(MOE_OK), "ok") == 0);
    CHECK(strstr(moe_strerror(MOE_ERR_INVALID_ARG), "invalid") != NULL);
    CHECK(strstr(moe_status_bit_name(MOE_ST_COVERAGE), "cover") != NULL);
    CHECK(strstr(moe_version(), "sm_100a") != NULL);
    CHECK(strcmp(moe_last_cuda_error(), "none") == 0);     /* no CUDA failure on this thread */

    /* host checks: each call is refused before any CUDA call */
    CHECK(moe_dispatch_layout((const int64_t*)A, 64, 2, 8, 3, 4, (int32_t*)A, (int32_t*)A,
                              (int32_t*)A, (int32_t*)A, (uint8_t*)A, (int32_t*)A, A,
                              (int32_t*)A, s) == MOE_ERR_INVALID_ARG);          /* E % R */
    CHECK(moe_permute((const uint16_t*)A, (const int64_t*)A, 64, 2, 8, 60, (const int32_t*)A, A,
                      1, 128, (uint16_t*)A, (int32_t*)A, (int32_t*)A, (int32_t*)A,
                      s) == MOE_ERR_INVALID_ARG);                               /* H % 8 */
    CHECK(moe_combine_weighted((const uint16_t*)A, 256, (const int32_t*)A, (const int32_t*)A, A,
                               2, 64, 2, 64, 0, (uint16_t*)A, (int32_t*)A,
                               s) == MOE_ERR_INVALID_ARG);                      /* dtype */
    CHECK(moe_combine_backward((const uint16_t*)A, (const uint16_t*)A, 256, (const int32_t*)A,
                               (const int32_t*)A, NULL, MOE_DTYPE_F32, 64, 2, 64,
                               (const int32_t*)A, 8, 1, (uint16_t*)A, A, (int32_t*)A,
                               s) == MOE_ERR_INVALID_ARG);                      /* null w */
    CHECK(moe_segment_labels((const int32_t*)A, 0, 8, 10, (int64_t*)A, (int32_t*)A,
                             s) == MOE_ERR_INVALID_ARG);                        /* n = 0 */
    CHECK(moe_combine_from_ranks((const uint16_t* const*)A, NULL, 3, 0, 256, (const int32_t*)A,
                                 (const int64_t*)A, 8, A, MOE_DTYPE_F32, 64, 2, 64,
                                 (uint16_t*)A, (int32_t*)A, s) == MOE_ERR_INVALID_ARG);
    CHECK(moe_dispatch_layout_noalloc((const int64_t*)A, 1 << 20, 32, 1024, 1, 1, (int32_t*)A,
                                      (int32_t*)A, (int32_t*)A, (int32_t*)A, (uint8_t*)A,
                                      (int32_t*)A, (int32_t*)A, s) == MOE_ERR_SCRATCH);

    if (failures == 0) printf("C ABI checks passed\n");
    return failures == 0 ? 0 : 1;
}
