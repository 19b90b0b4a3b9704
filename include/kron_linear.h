/*
 * kron_linear.h -- C ABI of libkronlinear.so, the B200 (sm_100a) implementation of
 * the sum-of-Kronecker-products linear layer
 *
 *     y = x W + bias,   W = sum_{i<r} kron(C_i, B_i),   C_i = S (.) A_i,
 *
 * as defined on the page "kronecker-layer-benchmark" (section "1. Build W, then
 * multiply", KronLinear.weight/forward; rectangular B_i as in section "2. The vec
 * trick").  W is never formed: each row x_n is viewed as X_n (p x m1) and
 * Y_n = sum_i C_i^T X_n B_i (section "2. The vec trick" and "3. The vec trick
 * without the loop"), with both contractions fused on chip.
 *
 * Layouts (all row-major, contiguous, no padding):
 *   x, dX   [N][p*m1]      X_n[a][j]  = x[n][a*m1 + j]
 *   y, dY   [N][q*m2]      Y_n[c][k]  = y[n][c*m2 + k]
 *   S, dS   [p][q]
 *   A, dA   [r][p][q]
 *   B, dB   [r][m1][m2]
 *   bias, dbias [q*m2]
 *
 * Element types by path (kron_dtype_t):
 *   KRON_F32   every tensor is float32; exact FP32 arithmetic on the CUDA cores.
 *   KRON_TF32  every tensor is float32; both contractions run on the tcgen05 tensor
 *              cores with TF32 operands and FP32 accumulation.
 *   KRON_BF16  x, y, dY, dX, S, A, B and bias are bfloat16; dS, dA, dB and dbias are
 *              float32.  tcgen05 tensor cores with BF16 operands, FP32 accumulation.
 *   KRON_TF32 and KRON_BF16 run only where a tensor-core kernel exists for the shape;
 *   a call of any other shape returns KRON_ERR_UNSUPPORTED and launches nothing (it is
 *   never run on another path).  KRON_F32 takes any shape whose FP32 tile fits shared
 *   memory.  kron_linear_workspace_size returns 0 for a shape the requested path does
 *   not take, so it also answers whether a backward is supported.
 *
 * Ownership and synchronisation: every pointer except `stream` is a DEVICE pointer
 * owned by the caller.  The library allocates no memory and never synchronises; all
 * work is enqueued on `stream` (a cudaStream_t passed as void*, NULL = legacy default
 * stream).  No result depends on an earlier call.  The only device memory of its own
 * is compiled in: the error word of kron_linear_device_error and the scratch array of
 * kron_linear_backward_noalloc.
 *
 * Errors: arguments, shapes, alignment and workspace size are checked on the host
 * before anything is launched; a failing check returns its status and launches
 * nothing.  Shapes the requested path has no kernel for return KRON_ERR_UNSUPPORTED;
 * nothing ever falls back to another path or to the CPU.  A failed launch returns KRON_ERR_CUDA;
 * faults during execution surface at the caller's next synchronisation.
 * kron_last_error() gives a one-line description of the last failure on the
 * calling host thread.
 */
#ifndef KRON_LINEAR_H
#define KRON_LINEAR_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define KRON_LINEAR_ABI_VERSION 2

#if defined(__GNUC__)
#define KRON_API __attribute__((visibility("default")))
#else
#define KRON_API
#endif

typedef enum {
    KRON_F32 = 0,   /* exact FP32 (FFMA)                          */
    KRON_TF32 = 1,  /* FP32 I/O, TF32 tensor cores, FP32 accumulate */
    KRON_BF16 = 2   /* BF16 I/O, BF16 tensor cores, FP32 accumulate */
} kron_dtype_t;

typedef enum {
    KRON_OK = 0,
    KRON_ERR_INVALID_ARG = 1,  /* null pointer, non-positive size, bad dtype or flag   */
    KRON_ERR_UNSUPPORTED = 2,  /* valid shape that this path does not implement          */
    KRON_ERR_ALIGNMENT = 3,    /* a pointer is not 16-byte aligned                       */
    KRON_ERR_WORKSPACE = 4,    /* workspace NULL or smaller than kron_linear_workspace_size */
    KRON_ERR_CUDA = 5,         /* a CUDA runtime call or kernel launch failed            */
    KRON_ERR_TIMEOUT = 6       /* a bounded device-side wait gave up (kron_linear_device_error) */
} kron_status_t;

/* Skip the work of (a, c) blocks where S is zero (the m1 x m2 block of W is zero,
 * page "kronecker-layer-benchmark", introduction).  Only provably-zero products are
 * skipped: dS stays exact at zero entries of S.  Results equal the unflagged call
 * up to rounding. */
#define KRON_FLAG_SKIP_ZERO_BLOCKS 1u

/*
 * Forward: y = x W + bias.
 *   x     [N][p*m1]  input rows
 *   S, A, B          factors as above
 *   bias  [q*m2]     may be NULL (no bias)
 *   y     [N][q*m2]  output, overwritten
 *   N >= 0 rows (N == 0 is a no-op and x, y may then be NULL); p, q, m1, m2, r >= 1.
 * Requirements: x, y, S, A, B, bias 16-byte aligned (KRON_ERR_ALIGNMENT);
 * m1 and m2 multiples of 4 (F32/TF32) or 8 (BF16), else KRON_ERR_UNSUPPORTED.
 */
KRON_API kron_status_t kron_linear_forward(const void *x, const void *S, const void *A, const void *B,
                                  const void *bias, void *y,
                                  int64_t N, int p, int q, int m1, int m2, int r,
                                  kron_dtype_t dtype, unsigned flags, void *stream);

/*
 * Backward: gradients of L = <dY, y> (dY = dL/dy).
 *   dX    [N][p*m1]   = dY W^T                                   (may be NULL: skipped)
 *   dS    [p][q]      = sum_i dC_i (.) A_i
 *   dA    [r][p][q]   = dC_i (.) S,   dC_i = sum_n (X_n B_i) dY_n^T
 *   dB    [r][m1][m2] = sum_n X_n^T C_i dY_n
 *   dbias [q*m2]      = sum_n dY_n                                (may be NULL: skipped)
 * With N == 0, x, dY and dX may be NULL and the factor gradients are set to zero.
 * Gradients OVERWRITE their outputs.  T = X_n B_i is recomputed, nothing is kept
 * from the forward call.  The sums over rows are split into a fixed number of
 * contiguous row ranges whose partials are added in a fixed order, so results are
 * bitwise identical across calls with the same inputs on the same GPU model.
 * `workspace` is device scratch of at least kron_linear_workspace_size(...) bytes,
 * 256-byte aligned, owned by the caller; its contents on entry are ignored.
 * On the tensor-core paths of the tutorial layer's shape (p = q = m1 = m2 = 32, r = 4)
 * the parameter-gradient kernel sums the row ranges itself after a grid-wide barrier:
 * it is a cooperative launch of one CTA per row range (at most 148), all of which must
 * be resident at once.  On a device or partition that cannot hold them (fewer SMs, or
 * SMs taken by other work under MPS) the launch fails and the call returns
 * KRON_ERR_CUDA; the other paths add the ranges with a separate reduction kernel.
 */
KRON_API kron_status_t kron_linear_backward(const void *x, const void *S, const void *A, const void *B,
                                   const void *dY, void *dX, void *dS, void *dA, void *dB,
                                   void *dbias,
                                   int64_t N, int p, int q, int m1, int m2, int r,
                                   kron_dtype_t dtype, unsigned flags,
                                   void *workspace, size_t workspace_bytes, void *stream);

/*
 * Backward with the l1 penalty on S fused into the dS epilogue.
 *
 * The layer is trained with the loss plus l1 * sum_{a,c} |S[a][c]| (page
 * "kronecker-layer-benchmark", introduction: an l1 penalty on S makes S sparse and with it
 * W block-sparse; section "Setup": the step's loss is the cross-entropy plus the model's
 * penalty).  The gradient of that term, l1 * sign(S), is added to dS inside the kernel that
 * writes dS, so the caller launches nothing for it:
 *   dS [p][q] = sum_i dC_i (.) A_i + l1 * sign(S)
 * sign(0) = 0: at S[a][c] = 0 the term is 0, the subgradient that autograd takes for |.|.
 * The sum is formed in double and rounded once to float32.
 *   l1   the penalty's weight, 0 <= l1 <= 1e30 (else KRON_ERR_INVALID_ARG); with l1 == 0
 *        the results are bit for bit those of kron_linear_backward.
 * With N == 0 the factor gradients are zero except dS = l1 * sign(S).
 * Every other argument, output and rule is kron_linear_backward's.  (The penalty's value is
 * not computed: the caller adds l1 * sum|S| to the loss it reports if it wants it.)
 */
KRON_API kron_status_t kron_linear_backward_l1(const void *x, const void *S, const void *A,
                                               const void *B, const void *dY, void *dX,
                                               void *dS, void *dA, void *dB, void *dbias,
                                               int64_t N, int p, int q, int m1, int m2, int r,
                                               kron_dtype_t dtype, unsigned flags, double l1,
                                               void *workspace, size_t workspace_bytes,
                                               void *stream);

/*
 * Backward without a caller-provided workspace.  (An addition of this library: the
 * paper has no counterpart.)
 *
 * Some callers cannot allocate device memory at the moment they run the backward: a
 * real-time loop in which cudaMalloc's device-wide synchronisation is not acceptable,
 * a host whose device memory is entirely owned by another allocator, or plain C code
 * with no allocator of its own.  This entry point takes the same arguments as
 * kron_linear_backward without the workspace and uses instead a fixed scratch array
 * of KRON_NOALLOC_SCRATCH_BYTES compiled into the library; it allocates nothing.
 *   - Every GPU that loads the library holds that array until the process exits.
 *   - Problems whose kron_linear_workspace_size exceeds KRON_NOALLOC_SCRATCH_BYTES are
 *     rejected with KRON_ERR_WORKSPACE before anything is launched.
 *   - All calls share the one array per device: calls that overlap on the GPU (for
 *     example on two streams) race on it and must be serialised by the caller.
 *   - The first call on a device looks up the array's device address (with that device
 *     current); make that first call before any stream capture.  The address belongs to
 *     the current CUDA context: it is looked up again after the context changes (after
 *     cudaDeviceReset, or under a context made current through the driver API), so the
 *     first call under a new context must also come before any capture.
 * Results are the same as kron_linear_backward's.
 */
#define KRON_NOALLOC_SCRATCH_BYTES (8u << 20)
KRON_API kron_status_t kron_linear_backward_noalloc(const void *x, const void *S, const void *A,
                                                    const void *B, const void *dY, void *dX,
                                                    void *dS, void *dA, void *dB, void *dbias,
                                                    int64_t N, int p, int q, int m1, int m2, int r,
                                                    kron_dtype_t dtype, unsigned flags,
                                                    void *stream);

/*
 * Triple Kronecker layer (page "LLM Compression via Kronecker Product Decomposition",
 * section "Triple Kronecker -- AxBxC (Extreme Compression)"), with r terms:
 *
 *     y = x W + bias,   W = sum_i kron(A_i, kron(B_i, C_i)),
 *     A [r][p][q], B [r][m1][m2], C [r][s1][s2], x [N][p*m1*s1], y [N][q*m2*s2],
 *     W[(a*m1 + j)*s1 + u][(c*m2 + k)*s2 + v] = sum_i A_i[a][c] B_i[j][k] C_i[u][v].
 *
 * It runs as the two-factor layer above with S = ones and the block factor
 * kron(B_i, C_i) ((m1*s1) x (m2*s2)), formed in the workspace by each call, so the shapes,
 * paths, dtypes (KRON_BF16: x, y, dY, dX, A, B, C, bias bf16; gradients fp32) and errors
 * are those of kron_linear_forward / kron_linear_backward for (p, q, m1*s1, m2*s2, r); in
 * BF16 the block factor is rounded once to bf16.  The backward returns dA = dC' and chains
 * the block factor's gradient to dB and dC (fixed-order double sums); dX and dbias may be
 * NULL.  `workspace` is kron3_linear_workspace_size(..., backward) bytes (forward: 0, backward:
 * 1), 256-byte aligned, owned by the caller; 0 means the arguments are invalid or the
 * backward has no kernel for the block shape on this path.
 */
KRON_API size_t kron3_linear_workspace_size(int64_t N, int p, int q, int m1, int m2, int s1,
                                            int s2, int r, kron_dtype_t dtype, int backward);
KRON_API kron_status_t kron3_linear_forward(const void *x, const void *A, const void *B,
                                            const void *C, const void *bias, void *y, int64_t N,
                                            int p, int q, int m1, int m2, int s1, int s2, int r,
                                            kron_dtype_t dtype, unsigned flags, void *workspace,
                                            size_t workspace_bytes, void *stream);
KRON_API kron_status_t kron3_linear_backward(const void *x, const void *A, const void *B,
                                             const void *C, const void *dY, void *dX, void *dA,
                                             void *dB, void *dC, void *dbias, int64_t N, int p,
                                             int q, int m1, int m2, int s1, int s2, int r,
                                             kron_dtype_t dtype, unsigned flags, void *workspace,
                                             size_t workspace_bytes, void *stream);

/*
 * Rank-r Kronecker fit of a dense matrix, to initialise the layer's factors from a dense
 * layer (page "LLM Compression via Kronecker Product Decomposition", sections "Van Loan
 * Rearrangement (1993)", "Rank-K" and "Adaptive Normalization"):
 *
 *   Wt[a*q + c][j*m2 + k] = W[a*m1 + j][c*m2 + k]            ((p*q) x (m1*m2))
 *   Wt ~ sum_{i<r} sigma_i u_i v_i^T                           (r leading singular pairs)
 *   A_i = sqrt(sigma_i) reshape(u_i, p, q),  B_i = sqrt(sigma_i) reshape(v_i, m1, m2)
 *   alpha = |W|_F / |sum_i kron(A_i, B_i)|_F; with normalize != 0, A_i and B_i are both
 *   scaled by sqrt(alpha) (the fit then has the Frobenius norm of W).
 *
 * With S = ones, (S, A, B) are factors of this layer: sum_i kron(S (.) A_i, B_i) is the
 * best Kronecker sum of r terms to W in the Frobenius norm (times alpha when normalized).
 * The singular pairs come from randomized subspace iteration (Halko, Martinsson and Tropp,
 * 2011): Q = orth(Wt Omega), then power_iters times Q = orth(Wt orth(Wt^T Q)), and the
 * eigenpairs of (Q^T Wt)(Q^T Wt)^T.  The fit is exact (to rounding) when W has Kronecker
 * rank <= k; otherwise more power iterations and a larger k bring it closer to the exact
 * truncated SVD.  Sums run in double in a fixed order: results are bitwise reproducible.
 *   W       [p*m1][q*m2] float32, device
 *   omega   [k][m1*m2]  float32, device: the random test matrix (e.g. standard normal),
 *           drawn by the caller; 1 <= r <= k <= 64, k <= p*q, k <= m1*m2
 *   power_iters  0..16
 *   A [r][p][q], B [r][m1][m2], sigma [k] (estimated singular values of Wt, largest
 *   first), alpha [1]: float32 outputs, device, overwritten
 *   workspace of kron_vanloan_workspace_size(p, q, m1, m2, k) bytes, 256-byte aligned
 * Every pointer is 16-byte aligned (KRON_ERR_ALIGNMENT).  Bad sizes or pointers return
 * KRON_ERR_INVALID_ARG before anything is launched; all work is enqueued on `stream`.
 */
KRON_API size_t kron_vanloan_workspace_size(int p, int q, int m1, int m2, int k);
KRON_API kron_status_t kron_vanloan_fit(const void *W, int p, int q, int m1, int m2, int r,
                                        const void *omega, int k, int power_iters,
                                        int normalize, void *A, void *B, void *sigma,
                                        void *alpha, void *workspace, size_t workspace_bytes,
                                        void *stream);

/* Bytes of device workspace kron_linear_backward needs for this problem (0 if the
 * arguments are invalid).  Depends only on the arguments, not on the device. */
KRON_API size_t kron_linear_workspace_size(int64_t N, int p, int q, int m1, int m2, int r,
                                  kron_dtype_t dtype);

/* Static description of a status code. */
KRON_API const char *kron_status_string(kron_status_t status);

/* One-line description of the last failure on this host thread ("" if none). */
KRON_API const char *kron_last_error(void);

/* Device-side error state of the tensor-core kernels.  Every wait inside those
 * kernels is bounded: if one makes no progress for 2 s the kernel raises an error
 * word in device memory and returns instead of hanging.  This call synchronises the
 * current device, reads that word and returns KRON_ERR_TIMEOUT if it is set
 * (KRON_OK otherwise); clear != 0 resets it. */
KRON_API kron_status_t kron_linear_device_error(int clear);

/* KRON_LINEAR_ABI_VERSION of the loaded library. */
KRON_API int kron_linear_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KRON_LINEAR_H */
