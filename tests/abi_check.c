/*
 * abi_check.c -- the C ABI used from plain C99 (no C++, no Python): the header compiles
 * with -std=c99 -pedantic -Werror, the library links, and every host-side check of every
 * entry point returns its documented status before anything touches the device.  The
 * pointers below are never dereferenced: each call fails a host check.
 *
 * Built and run by tests/test_c_abi.py; exits 0 when every check passes, else prints the
 * failing check and exits 1.  The Kronecker-sparse factor's header (ks_linear.h) is
 * compiled and checked the same way.
 */
#include "kron_linear.h"
#include "ks_linear.h"

#include <stdint.h>
#include <stdio.h>
#include <string.h>

static int failures = 0;

#define CHECK(cond)                                                          \
    do {                                                                     \
        if (!(cond)) {                                                       \
            printf("FAILED line %d: %s (last error: %s)\n", __LINE__, #cond, \
                   kron_last_error());                                       \
            ++failures;                                                      \
        }                                                                    \
    } while (0)

int main(void) {
    void *const P = (void *)(uintptr_t)0x10000;     /* 16-byte aligned, never read */
    void *const MIS = (void *)(uintptr_t)0x10004;   /* misaligned */
    void *const WS = (void *)(uintptr_t)0x100000;   /* 256-byte aligned, never read */
    size_t need;
    int st;

    CHECK(kron_linear_abi_version() == KRON_LINEAR_ABI_VERSION);
    for (st = KRON_OK; st <= KRON_ERR_TIMEOUT; ++st)
        CHECK(strncmp(kron_status_string((kron_status_t)st), "KRON_", 5) == 0);

    /* workspace size: a function of the arguments only; 0 for invalid ones */
    need = kron_linear_workspace_size(20000, 32, 32, 32, 32, 4, KRON_TF32);
    CHECK(need > 0 && need % 256 == 0);
    CHECK(need == kron_linear_workspace_size(20000, 32, 32, 32, 32, 4, KRON_TF32));
    CHECK(kron_linear_workspace_size(20000, 0, 32, 32, 32, 4, KRON_TF32) == 0);
    CHECK(kron_linear_workspace_size(-1, 32, 32, 32, 32, 4, KRON_F32) == 0);
    CHECK(kron_linear_workspace_size(8, 2, 2, 4, 4, 1, (kron_dtype_t)9) == 0);

    /* forward */
    CHECK(kron_linear_forward(P, P, P, P, NULL, P, 8, 2, 2, 4, 4, 1, (kron_dtype_t)9, 0, NULL) ==
          KRON_ERR_INVALID_ARG);
    CHECK(strlen(kron_last_error()) > 0);
    CHECK(kron_linear_forward(P, P, P, P, NULL, P, 8, 2, 2, 4, 4, 1, KRON_F32, 8u, NULL) ==
          KRON_ERR_INVALID_ARG);                                            /* unknown flag */
    CHECK(kron_linear_forward(NULL, P, P, P, NULL, P, 8, 2, 2, 4, 4, 1, KRON_F32, 0, NULL) ==
          KRON_ERR_INVALID_ARG);                                            /* x missing */
    CHECK(kron_linear_forward(MIS, P, P, P, NULL, P, 8, 2, 2, 4, 4, 1, KRON_F32, 0, NULL) ==
          KRON_ERR_ALIGNMENT);
    CHECK(kron_linear_forward(P, P, P, P, NULL, P, 8, 2, 2, 6, 4, 1, KRON_F32, 0, NULL) ==
          KRON_ERR_UNSUPPORTED);                                            /* m1 % 4 */
    CHECK(kron_linear_forward(P, P, P, P, NULL, P, 8, 2, 2, 4, 4, 1, KRON_BF16, 0, NULL) ==
          KRON_ERR_UNSUPPORTED);                                            /* m1 % 8 */
    /* N == 0 is a no-op that needs no device at all */
    CHECK(kron_linear_forward(NULL, P, P, P, NULL, NULL, 0, 2, 2, 4, 4, 1, KRON_F32, 0, NULL) ==
          KRON_OK);
    CHECK(strlen(kron_last_error()) == 0);

    /* backward */
    need = kron_linear_workspace_size(8, 2, 2, 4, 4, 1, KRON_F32);
    CHECK(kron_linear_backward(P, P, P, P, P, P, NULL, P, P, NULL, 8, 2, 2, 4, 4, 1, KRON_F32, 0,
                               WS, need, NULL) == KRON_ERR_INVALID_ARG);   /* dS missing */
    CHECK(kron_linear_backward(P, P, P, P, P, P, P, P, P, NULL, 8, 2, 2, 4, 4, 1, KRON_F32, 0,
                               NULL, 0, NULL) == KRON_ERR_WORKSPACE);
    CHECK(kron_linear_backward(P, P, P, P, P, P, P, P, P, NULL, 8, 2, 2, 4, 4, 1, KRON_F32, 0,
                               WS, need - 4, NULL) == KRON_ERR_WORKSPACE);
    CHECK(kron_linear_backward(P, P, P, P, P, P, P, P, P, NULL, 8, 2, 2, 4, 4, 1, KRON_F32, 0,
                               (char *)WS + 16, need, NULL) == KRON_ERR_ALIGNMENT);
    CHECK(kron_linear_backward(P, P, P, P, MIS, P, P, P, P, NULL, 8, 2, 2, 4, 4, 1, KRON_F32, 0,
                               WS, need, NULL) == KRON_ERR_ALIGNMENT);     /* dY misaligned */

    /* backward with the fused l1 term: the weight is checked like every other argument */
    CHECK(kron_linear_backward_l1(P, P, P, P, P, P, P, P, P, NULL, 8, 2, 2, 4, 4, 1, KRON_F32, 0,
                                  -0.5, WS, need, NULL) == KRON_ERR_INVALID_ARG);
    CHECK(kron_linear_backward_l1(P, P, P, P, P, P, P, P, P, NULL, 8, 2, 2, 4, 4, 1, KRON_F32, 0,
                                  1e31, WS, need, NULL) == KRON_ERR_INVALID_ARG);
    CHECK(kron_linear_backward_l1(P, P, P, P, P, P, P, P, P, NULL, 8, 2, 2, 4, 4, 1, KRON_F32, 0,
                                  0.5, NULL, 0, NULL) == KRON_ERR_WORKSPACE);

    /* backward without a workspace: invalid arguments and oversized problems are refused
       on the host, before the scratch array's address is looked up */
    CHECK(kron_linear_backward_noalloc(P, P, P, P, P, P, P, P, P, NULL, 8, 2, 2, 4, 4, 1,
                                       (kron_dtype_t)9, 0, NULL) == KRON_ERR_INVALID_ARG);
    CHECK(kron_linear_backward_noalloc(P, P, P, P, P, P, P, P, P, NULL, 8, 2, 2, 6, 4, 1,
                                       KRON_F32, 0, NULL) == KRON_ERR_UNSUPPORTED);
    /* 20000 rows of the 4096^2 layer with 64x64 blocks and rank 8 need ~41 MB of scratch */
    CHECK(kron_linear_workspace_size(20000, 64, 64, 64, 64, 8, KRON_F32) >
          KRON_NOALLOC_SCRATCH_BYTES);
    CHECK(kron_linear_backward_noalloc(P, P, P, P, P, P, P, P, P, NULL, 20000, 64, 64, 64, 64, 8,
                                       KRON_F32, 0, NULL) == KRON_ERR_WORKSPACE);
    CHECK(strstr(kron_last_error(), "scratch") != NULL);
    /* an oversized problem with a bad argument: the argument's own status comes first */
    CHECK(kron_linear_backward_noalloc(P, P, P, P, P, P, NULL, P, P, NULL, 20000, 64, 64, 64, 64,
                                       8, KRON_F32, 0, NULL) == KRON_ERR_INVALID_ARG);
    CHECK(kron_linear_backward_noalloc(P, P, P, P, MIS, P, P, P, P, NULL, 20000, 64, 64, 64, 64,
                                       8, KRON_F32, 0, NULL) == KRON_ERR_ALIGNMENT);
    CHECK(kron_linear_backward_noalloc(NULL, P, P, P, P, P, P, P, P, NULL, 8, 2, 2, 4, 4, 1,
                                       KRON_F32, 0, NULL) == KRON_ERR_INVALID_ARG);

    /* the tensor-core paths refuse shapes they have no kernel for (no silent FP32 run):
       1024^2 with 16x16 blocks (p = q = 64) and rank 2 on TF32; a 15x24 layer on BF16 */
    CHECK(kron_linear_forward(P, P, P, P, NULL, P, 8, 64, 64, 16, 16, 2, KRON_TF32, 0, NULL) ==
          KRON_ERR_UNSUPPORTED);
    CHECK(strstr(kron_last_error(), "tensor-core") != NULL);
    CHECK(kron_linear_forward(P, P, P, P, NULL, P, 8, 3, 5, 8, 8, 3, KRON_BF16, 0, NULL) ==
          KRON_ERR_UNSUPPORTED);
    CHECK(kron_linear_workspace_size(8, 64, 64, 16, 16, 2, KRON_TF32) == 0);
    CHECK(kron_linear_backward(P, P, P, P, P, P, P, P, P, NULL, 8, 64, 64, 16, 16, 2, KRON_TF32,
                               0, WS, 1u << 20, NULL) == KRON_ERR_UNSUPPORTED);
    CHECK(kron_linear_backward_noalloc(P, P, P, P, P, P, P, P, P, NULL, 8, 3, 5, 8, 8, 3,
                                       KRON_BF16, 0, NULL) == KRON_ERR_UNSUPPORTED);
    /* the same shapes run on the exact-FP32 path */
    CHECK(kron_linear_workspace_size(8, 64, 64, 16, 16, 2, KRON_F32) > 0);

    /* Van Loan fit: sizes, rank and pointers are checked on the host */
    CHECK(kron_vanloan_workspace_size(32, 32, 32, 32, 12) > 0);
    CHECK(kron_vanloan_workspace_size(32, 32, 32, 32, 65) == 0);
    CHECK(kron_vanloan_fit(P, 4, 4, 4, 4, 9, P, 8, 2, 1, P, P, P, P, WS, 1u << 24, NULL) ==
          KRON_ERR_INVALID_ARG);                                        /* r > k */
    CHECK(kron_vanloan_fit(MIS, 4, 4, 4, 4, 2, P, 8, 2, 1, P, P, P, P, WS, 1u << 24, NULL) ==
          KRON_ERR_ALIGNMENT);
    CHECK(kron_vanloan_fit(P, 4, 4, 4, 4, 2, P, 8, 2, 1, P, P, P, P, NULL, 0, NULL) ==
          KRON_ERR_WORKSPACE);

    /* Kronecker-sparse factor: FP32 only, natural 4-byte alignment, host checks first */
    {
        void *const MIS2 = (void *)(uintptr_t)0x10002; /* not 4-byte aligned */
        size_t ks_need = ks_linear_workspace_size(20000, 1, 32, 32, 32, KRON_F32);
        CHECK(ks_need > 0 && ks_need % 256 == 0);
        CHECK(ks_need == ks_linear_workspace_size(20000, 1, 32, 32, 32, KRON_F32));
        CHECK(ks_linear_workspace_size(20000, 1, 32, 32, 32, KRON_TF32) == 0);
        CHECK(ks_linear_workspace_size(-1, 1, 32, 32, 32, KRON_F32) == 0);
        CHECK(ks_linear_workspace_size(8, 0, 32, 32, 32, KRON_F32) == 0);
        CHECK(ks_linear_forward(P, P, NULL, P, 8, 2, 3, 4, 5, (kron_dtype_t)9, 0, NULL) ==
              KRON_ERR_INVALID_ARG);
        CHECK(ks_linear_forward(P, P, NULL, P, 8, 2, 3, 4, 5, KRON_TF32, 0, NULL) ==
              KRON_ERR_UNSUPPORTED);
        CHECK(ks_linear_forward(P, P, NULL, P, 8, 2, 3, 4, 5, KRON_BF16, 0, NULL) ==
              KRON_ERR_UNSUPPORTED);
        CHECK(ks_linear_forward(P, P, NULL, P, 8, 2, 3, 4, 5, KRON_F32, 1u, NULL) ==
              KRON_ERR_INVALID_ARG);                                        /* no flags */
        CHECK(ks_linear_forward(P, P, NULL, P, 8, 0, 3, 4, 5, KRON_F32, 0, NULL) ==
              KRON_ERR_INVALID_ARG);
        CHECK(ks_linear_forward(NULL, P, NULL, P, 8, 2, 3, 4, 5, KRON_F32, 0, NULL) ==
              KRON_ERR_INVALID_ARG);
        CHECK(ks_linear_forward(MIS2, P, NULL, P, 8, 2, 3, 4, 5, KRON_F32, 0, NULL) ==
              KRON_ERR_ALIGNMENT);
        CHECK(ks_linear_forward(NULL, P, NULL, NULL, 0, 2, 3, 4, 5, KRON_F32, 0, NULL) ==
              KRON_OK);                                                     /* N == 0 */
        ks_need = ks_linear_workspace_size(8, 2, 3, 4, 5, KRON_F32);
        CHECK(ks_linear_backward(P, P, P, P, NULL, NULL, 8, 2, 3, 4, 5, KRON_F32, 0, WS,
                                 ks_need, NULL) == KRON_ERR_INVALID_ARG);   /* dw missing */
        CHECK(ks_linear_backward(P, P, P, P, P, NULL, 8, 2, 3, 4, 5, KRON_F32, 0, NULL, 0,
                                 NULL) == KRON_ERR_WORKSPACE);
        CHECK(ks_linear_backward(P, P, P, P, P, NULL, 8, 2, 3, 4, 5, KRON_F32, 0, WS,
                                 ks_need - 4, NULL) == KRON_ERR_WORKSPACE);
        CHECK(ks_linear_backward(P, P, P, P, P, NULL, 8, 2, 3, 4, 5, KRON_F32, 0,
                                 (char *)WS + 16, ks_need, NULL) == KRON_ERR_ALIGNMENT);
        CHECK(ks_linear_backward(P, P, MIS2, P, P, NULL, 8, 2, 3, 4, 5, KRON_F32, 0, WS,
                                 ks_need, NULL) == KRON_ERR_ALIGNMENT);     /* dY */
    }

    if (failures) return 1;
    printf("abi_check: all checks passed\n");
    return 0;
}
