/*
 * ks_linear.h -- C ABI of the Kronecker-sparse (KS) factor in libkronlinear.so.
 *
 * A KS matrix (page "Fast Inference with Kronecker-Sparse Matrices", abstract) has a
 * support that is a Kronecker product of identity and all-ones blocks.  The pattern
 * (a, b, c, d) names the support kron(I_a, kron(1_{b x c}, I_d)) of an (a*b*d) x (a*c*d)
 * matrix K, which this library applies as the weight of a linear layer with row vectors
 * (the orientation of kron_linear.h):
 *
 *     y = x K + bias,
 *     K[(al*b + be)*d + de][(al*c + ga)*d + de] = w[al][de][be][ga],   zero elsewhere.
 *
 * Read per row: y[n][(al*c + ga)*d + de] = sum_be x[n][(al*b + be)*d + de] w[al][de][be][ga]
 * (+ bias), i.e. a*d independent b x c products whose inputs and outputs are strided by d
 * inside the row.  The kernels gather those strided slices on chip (one read of x, one
 * write of y, no permuted copies in memory), output-stationary: each CTA owns a tile of
 * y and runs the whole contraction for it.  Butterfly and Monarch matrices are products
 * of such factors; a chain is a sequence of calls.
 *
 * Layouts (row-major, contiguous):
 *   x, dX   [N][a*b*d]
 *   y, dY   [N][a*c*d]
 *   w, dw   [a][d][b][c]    the a*b*c*d free entries of K
 *   bias, dbias [a*c*d]
 *
 * Path: KRON_F32 only (every tensor float32, exact FP32 arithmetic on the CUDA cores);
 * KRON_TF32 and KRON_BF16 return KRON_ERR_UNSUPPORTED and launch nothing.
 *
 * Ownership, streams and errors as in kron_linear.h: every pointer except `stream` is a
 * device pointer owned by the caller, nothing is allocated or synchronised, all work is
 * enqueued on `stream`, and argument checks run on the host before any launch.  Tensors
 * need only their natural 4-byte alignment (KRON_ERR_ALIGNMENT otherwise).  Results are
 * bitwise reproducible for the same inputs and device: the row split of the backward's
 * sums depends on the sizes only and the partial sums are added in a fixed order.
 */
#ifndef KS_LINEAR_H
#define KS_LINEAR_H

#include "kron_linear.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Forward: y = x K + bias.
 *   N >= 0 rows (N == 0 is a no-op; x and y may then be NULL); a, b, c, d >= 1 with
 *   a*b*d and a*c*d at most 2^24.  bias may be NULL (no bias).
 */
KRON_API kron_status_t ks_linear_forward(const void *x, const void *w, const void *bias, void *y,
                                         int64_t N, int a, int b, int c, int d,
                                         kron_dtype_t dtype, unsigned flags, void *stream);

/*
 * Backward: gradients of L = <dY, y>.
 *   dX    [N][a*b*d] = dY K^T                                     (may be NULL: skipped)
 *   dw    [a][d][b][c]: dw[al][de][be][ga] = sum_n x[n][(al*b + be)*d + de] dY[n][(al*c + ga)*d + de]
 *   dbias [a*c*d]    = sum_n dY[n]                                 (may be NULL: skipped)
 * Gradients overwrite their outputs.  With N == 0, x, dY and dX may be NULL and dw and
 * dbias are set to zero.  `workspace` holds ks_linear_workspace_size(...) bytes, is
 * 256-byte aligned and owned by the caller (KRON_ERR_WORKSPACE if NULL or smaller).
 * flags must be 0.
 */
KRON_API kron_status_t ks_linear_backward(const void *x, const void *w, const void *dY, void *dX,
                                          void *dw, void *dbias, int64_t N, int a, int b, int c,
                                          int d, kron_dtype_t dtype, unsigned flags,
                                          void *workspace, size_t workspace_bytes, void *stream);

/* Bytes of workspace ks_linear_backward needs (a multiple of 256; 0 if the arguments are
 * invalid or the dtype is not KRON_F32).  Depends only on the arguments. */
KRON_API size_t ks_linear_workspace_size(int64_t N, int a, int b, int c, int d,
                                         kron_dtype_t dtype);

#ifdef __cplusplus
}
#endif

#endif /* KS_LINEAR_H */
