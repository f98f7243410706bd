/*
 * A plain C11 caller of libfa2.so: include/fa2.h compiles as C (no CUDA or
 * C++ headers needed), the library links and loads without a GPU, and the
 * host-side validation answers with the documented status codes before
 * anything reaches a device.  Pointers are fake, aligned and never read.
 * Prints "ok" and returns 0 when every check holds, else names the first
 * failure and returns 1.
 */
#include <math.h>
#include <stdio.h>
#include <string.h>

#include "fa2.h"

static int failures = 0;

#define CHECK(cond)                                                     \
    do {                                                                \
        if (!(cond)) {                                                  \
            fprintf(stderr, "check failed (line %d): %s\n", __LINE__, #cond); \
            failures++;                                                 \
        }                                                               \
    } while (0)

static void* const P = (void*)0x10000;     /* 256-byte aligned, fake */

static fa2_status fwd(void* q, int N, int d, int causal, float scale, int dtype) {
    return fa2_forward(q, P, P, P, (float*)P, 1, 2, N, d, causal, scale, (fa2_dtype)dtype, NULL);
}

int main(void) {
    for (int code = FA2_OK; code <= FA2_ERR_SCRATCH_TOO_SMALL; ++code) {
        const char* s = fa2_status_string((fa2_status)code);
        CHECK(s != NULL && strncmp(s, "FA2_", 4) == 0);
    }
    CHECK(strcmp(fa2_status_string(FA2_OK), "FA2_OK") == 0);

    /* Workspace: two fp32 [B*H][ceil(N/128)*128] regions and, with more than
     * one key tile, the fp32 dQ accumulator [B*H][ceil(N/128)*128][d], each
     * rounded up to 256 bytes, for 16-bit inputs; the _ex form agrees with
     * MHA shapes. */
    size_t ws = fa2_backward_workspace_bytes(2, 3, 200, 80, FA2_BF16);
    CHECK(ws == 2 * (size_t)(2 * 3 * 256 * 4) + (size_t)(2 * 3 * 256 * 80 * 4));
    CHECK(fa2_backward_workspace_bytes(2, 3, 128, 80, FA2_BF16) == 2 * (size_t)(2 * 3 * 128 * 4));
    CHECK(fa2_backward_workspace_bytes_ex(2, 3, 3, 200, 200, 80, FA2_BF16) == ws);
    CHECK(fa2_backward_workspace_bytes(2, 3, 200, 80, FA2_FP16) == ws);
    CHECK(fa2_backward_workspace_bytes(2, 3, 200, 24, FA2_BF16) == 0);

    /* Forward validation, in the header's order of checks. */
    CHECK(fwd(NULL, 128, 64, 1, 0.125f, FA2_BF16) == FA2_ERR_NULL_PTR);
    CHECK(fwd(P, 0, 64, 1, 0.125f, FA2_BF16) == FA2_ERR_BAD_SHAPE);
    CHECK(fwd(P, 128, 48, 1, 0.125f, FA2_BF16) == FA2_ERR_UNSUPPORTED_HEAD_DIM);
    CHECK(fwd(P, 128, 64, 1, 0.125f, 7) == FA2_ERR_UNSUPPORTED_DTYPE);
    CHECK(fwd((char*)P + 2, 128, 64, 1, 0.125f, FA2_BF16) == FA2_ERR_MISALIGNED);
    CHECK(fwd(P, 128, 64, 2, 0.125f, FA2_BF16) == FA2_ERR_BAD_ARGUMENT);
    CHECK(fwd(P, 128, 64, 1, NAN, FA2_BF16) == FA2_ERR_BAD_ARGUMENT);

    /* Backward: a workspace one byte short, and a misaligned workspace. */
    size_t need = fa2_backward_workspace_bytes(1, 2, 128, 64, FA2_BF16);
    CHECK(fa2_backward(P, P, P, P, (const float*)P, P, P, P, P, 1, 2, 128, 64, 1, 0.125f,
                       FA2_BF16, P, need - 1, NULL) == FA2_ERR_WORKSPACE_TOO_SMALL);
    CHECK(fa2_backward(P, P, P, P, (const float*)P, P, P, P, P, 1, 2, 128, 64, 1, 0.125f,
                       FA2_BF16, (char*)P + 16, need, NULL) == FA2_ERR_MISALIGNED);

    /* Backward options: unknown flag bits are rejected before anything else. */
    CHECK(fa2_backward_opts(P, P, P, P, (const float*)P, P, P, P, P, 1, 2, 2, 128, 128, 64, 1,
                            0.125f, FA2_BF16, NULL, 4u, P, need, NULL) == FA2_ERR_BAD_ARGUMENT);
    CHECK(fa2_backward_opts(P, P, P, P, (const float*)P, P, P, P, P, 1, 2, 2, 128, 128, 64, 1,
                            0.125f, FA2_BF16, NULL, FA2_BWD_DETERMINISTIC | FA2_BWD_ONE_PASS, P,
                            need, NULL) == FA2_ERR_BAD_ARGUMENT);
    CHECK(fa2_backward_opts(P, P, P, P, (const float*)P, P, P, P, P, 1, 2, 2, 128, 128, 64, 1,
                            0.125f, FA2_BF16, NULL, FA2_BWD_DETERMINISTIC, P, need - 1, NULL) ==
          FA2_ERR_WORKSPACE_TOO_SMALL);

    /* Grouped-query shapes: H must be a multiple of H_kv. */
    CHECK(fa2_forward_ex(P, P, P, P, (float*)P, 1, 6, 4, 128, 128, 64, 1, 0.125f, FA2_BF16,
                         NULL) == FA2_ERR_BAD_SHAPE);

    /* Block-sparse: a NULL mask is a NULL pointer. */
    CHECK(fa2_forward_block_sparse(P, P, P, P, (float*)P, 1, 2, 2, 128, 128, 64, 1, 0.125f,
                                   FA2_BF16, NULL, NULL) == FA2_ERR_NULL_PTR);

    /* Watchdog self-test: the wait limit must lie in [1e3, 1e10] ns. */
    CHECK(fa2_watchdog_selftest(0ull, NULL) == FA2_ERR_BAD_ARGUMENT);
    CHECK(fa2_watchdog_selftest(20000000000ull, NULL) == FA2_ERR_BAD_ARGUMENT);

    if (failures) return 1;
    printf("ok\n");
    return 0;
}
