/*
 * kron_oracle.c -- plain, slow, fp64 CPU oracle for the sum-of-Kronecker-products
 * linear layer.  TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the
 * benchmark's CPU-baseline leg call it; the product path never does.  It shares
 * no code, header or constant with the CUDA library.
 *
 * What it computes (page "kronecker-layer-benchmark", section "1. Build W, then
 * multiply", the `weight()` and `forward()` methods of KronLinear):
 *
 *     C_i = S (.) A_i                         (elementwise, p x q)
 *     W   = sum_i kron(C_i, B_i)              ((p*m1) x (q*m2), torch.kron order)
 *     y   = x W + bias                        (row vectors, x is N x (p*m1))
 *
 * i.e. W[a*m1 + j][c*m2 + k] = sum_i C_i[a][c] * B_i[j][k].  B_i is m1 x m2
 * (the section "2. The vec trick" allows a rectangular B: `m, n = B.shape[1:]`).
 *
 * The backward pass is the gradient of L = <G, y> for an upstream gradient
 * G = dL/dy, by the chain rule through the explicit W (the page leaves the
 * backward to autograd, section "Setup", "Training step"):
 *
 *     dX        = G W^T
 *     dW        = x^T G
 *     dC_i[a,c] = sum_{j,k} dW[a*m1+j][c*m2+k] * B_i[j][k]
 *     dB_i[j,k] = sum_{a,c} dW[a*m1+j][c*m2+k] * C_i[a][c]
 *     dA_i      = dC_i (.) S
 *     dS        = sum_i dC_i (.) A_i
 *     dbias     = sum_n G[n]
 *
 * The tutorial trains S under an l1 penalty lam * sum|S| (same page, introduction);
 * oracle_l1_grad gives that term's gradient, lam * sign(S), which the library can add
 * to dS.
 *
 * Everything is double precision, row-major and contiguous:
 *   x [N][p*m1], y and G [N][q*m2], S [p][q], A [r][p][q], B [r][m1][m2],
 *   bias [q*m2], W [p*m1][q*m2].
 * Loops are the definitions written out; OpenMP only splits independent output
 * rows across threads, the summation order inside one output stays sequential.
 */
#include <stddef.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

void oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int oracle_get_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* W = sum_i kron(S (.) A_i, B_i), built entry by entry. */
void oracle_build_weight(const double *S, const double *A, const double *B,
                         int p, int q, int m1, int m2, int r, double *W)
{
    const long in = (long)p * m1, out = (long)q * m2;
    memset(W, 0, sizeof(double) * (size_t)(in * out));
    for (int i = 0; i < r; ++i)
        for (int a = 0; a < p; ++a)
            for (int c = 0; c < q; ++c) {
                const double Cac = S[(long)a * q + c] * A[((long)i * p + a) * q + c];
                for (int j = 0; j < m1; ++j)
                    for (int k = 0; k < m2; ++k)
                        W[((long)a * m1 + j) * out + (long)c * m2 + k] +=
                            Cac * B[((long)i * m1 + j) * m2 + k];
            }
}

/* y = x W + bias (bias may be NULL).  Naive triple loop, one output row per task. */
void oracle_matmul_bias(const double *x, const double *W, const double *bias,
                        long N, long in, long out, double *y)
{
    #pragma omp parallel for schedule(static)
    for (long n = 0; n < N; ++n) {
        double *yn = y + n * out;
        for (long o = 0; o < out; ++o) yn[o] = bias ? bias[o] : 0.0;
        const double *xn = x + n * in;
        for (long u = 0; u < in; ++u) {
            const double xv = xn[u];
            const double *Wu = W + u * out;
            for (long o = 0; o < out; ++o) yn[o] += xv * Wu[o];
        }
    }
}

/* Forward: builds W, then y = x W + bias. */
void oracle_forward(const double *x, const double *S, const double *A, const double *B,
                    const double *bias, long N, int p, int q, int m1, int m2, int r,
                    double *y)
{
    const long in = (long)p * m1, out = (long)q * m2;
    double *W = (double *)malloc(sizeof(double) * (size_t)(in * out));
    oracle_build_weight(S, A, B, p, q, m1, m2, r, W);
    oracle_matmul_bias(x, W, bias, N, in, out, y);
    free(W);
}

/*
 * Backward through the explicit W.  Any output pointer may be NULL to skip it
 * (dX is the costly one; dW is needed by dS, dA and dB).
 */
void oracle_backward(const double *x, const double *S, const double *A, const double *B,
                     const double *G, long N, int p, int q, int m1, int m2, int r,
                     double *dX, double *dS, double *dA, double *dB, double *dbias)
{
    const long in = (long)p * m1, out = (long)q * m2;
    double *W = (double *)malloc(sizeof(double) * (size_t)(in * out));
    oracle_build_weight(S, A, B, p, q, m1, m2, r, W);

    if (dX) {
        /* dX[n][u] = sum_o G[n][o] * W[u][o] */
        #pragma omp parallel for schedule(static)
        for (long n = 0; n < N; ++n) {
            const double *Gn = G + n * out;
            for (long u = 0; u < in; ++u) {
                const double *Wu = W + u * out;
                double s = 0.0;
                for (long o = 0; o < out; ++o) s += Gn[o] * Wu[o];
                dX[n * in + u] = s;
            }
        }
    }

    if (dS || dA || dB) {
        /* dW[u][o] = sum_n x[n][u] * G[n][o] */
        double *dW = (double *)calloc((size_t)(in * out), sizeof(double));
        #pragma omp parallel for schedule(static)
        for (long u = 0; u < in; ++u) {
            double *dWu = dW + u * out;
            for (long n = 0; n < N; ++n) {
                const double xv = x[n * in + u];
                const double *Gn = G + n * out;
                for (long o = 0; o < out; ++o) dWu[o] += xv * Gn[o];
            }
        }
        /* dC_i[a][c] = sum_{j,k} dW[a*m1+j][c*m2+k] * B_i[j][k] */
        double *dC = (double *)calloc((size_t)r * p * q, sizeof(double));
        for (int i = 0; i < r; ++i)
            for (int a = 0; a < p; ++a)
                for (int c = 0; c < q; ++c) {
                    double s = 0.0;
                    for (int j = 0; j < m1; ++j)
                        for (int k = 0; k < m2; ++k)
                            s += dW[((long)a * m1 + j) * out + (long)c * m2 + k] *
                                 B[((long)i * m1 + j) * m2 + k];
                    dC[((long)i * p + a) * q + c] = s;
                }
        if (dB) {
            /* dB_i[j][k] = sum_{a,c} dW[a*m1+j][c*m2+k] * C_i[a][c] */
            for (int i = 0; i < r; ++i)
                for (int j = 0; j < m1; ++j)
                    for (int k = 0; k < m2; ++k) {
                        double s = 0.0;
                        for (int a = 0; a < p; ++a)
                            for (int c = 0; c < q; ++c)
                                s += dW[((long)a * m1 + j) * out + (long)c * m2 + k] *
                                     S[(long)a * q + c] * A[((long)i * p + a) * q + c];
                        dB[((long)i * m1 + j) * m2 + k] = s;
                    }
        }
        if (dA) {
            for (int i = 0; i < r; ++i)
                for (long ac = 0; ac < (long)p * q; ++ac)
                    dA[(long)i * p * q + ac] = dC[(long)i * p * q + ac] * S[ac];
        }
        if (dS) {
            for (long ac = 0; ac < (long)p * q; ++ac) {
                double s = 0.0;
                for (int i = 0; i < r; ++i)
                    s += dC[(long)i * p * q + ac] * A[(long)i * p * q + ac];
                dS[ac] = s;
            }
        }
        free(dC);
        free(dW);
    }

    if (dbias) {
        for (long o = 0; o < out; ++o) {
            double s = 0.0;
            for (long n = 0; n < N; ++n) s += G[n * out + o];
            dbias[o] = s;
        }
    }
    free(W);
}

/*
 * Gradient of the l1 penalty lam * sum_{a,c} |S[a][c]| that the page
 * "kronecker-layer-benchmark" (introduction) puts on S, added to the step's loss
 * (section "Setup"): out[a][c] = lam * sign(S[a][c]).  |.| has no derivative at 0; the
 * value taken there is 0, the subgradient autograd uses for abs().
 */
void oracle_l1_grad(const double *S, int p, int q, double lam, double *out)
{
    for (long ac = 0; ac < (long)p * q; ++ac) {
        const double v = S[ac];
        out[ac] = v > 0.0 ? lam : (v < 0.0 ? -lam : 0.0);
    }
}

/*
 * Van Loan rearrangement (page "LLM Compression via Kronecker Product Decomposition",
 * section "Van Loan Rearrangement (1993)"): the (p*m1) x (q*m2) matrix W becomes the
 * (p*q) x (m1*m2) matrix Wt whose row (a, c) is block (a, c) of W read row by row:
 *
 *     Wt[a*q + c][j*m2 + k] = W[a*m1 + j][c*m2 + k]
 *
 * so that W = sum_i kron(C_i, B_i) exactly when Wt = sum_i vec(C_i) vec(B_i)^T.
 */
void oracle_vanloan_rearrange(const double *W, int p, int q, int m1, int m2, double *Wt)
{
    for (int a = 0; a < p; ++a)
        for (int c = 0; c < q; ++c)
            for (int j = 0; j < m1; ++j)
                for (int k = 0; k < m2; ++k)
                    Wt[((size_t)a * q + c) * ((size_t)m1 * m2) + (size_t)j * m2 + k] =
                        W[((size_t)a * m1 + j) * ((size_t)q * m2) + (size_t)c * m2 + k];
}

/*
 * Triple Kronecker layer (page "LLM Compression via Kronecker Product Decomposition",
 * section "Triple Kronecker -- AxBxC (Extreme Compression)"), with r terms:
 *
 *     W = sum_i kron(A_i, kron(B_i, C_i)),   A_i p x q,  B_i m1 x m2,  C_i s1 x s2,
 *     W[(a*m1 + j)*s1 + u][(c*m2 + k)*s2 + v] = sum_i A_i[a][c] B_i[j][k] C_i[u][v],
 *     y = x W + bias,
 *
 * built entry by entry; the backward is the chain rule through that W (dX = G W^T,
 * dW = x^T G, dA_i[a][c] = sum dW[..] B_i[j][k] C_i[u][v], and likewise for B_i and C_i).
 * A [r][p][q], B [r][m1][m2], C [r][s1][s2]; x [N][p*m1*s1]; y, G [N][q*m2*s2].
 */
void oracle_build_weight3(const double *A, const double *B, const double *C, int p, int q,
                          int m1, int m2, int s1, int s2, int r, double *W)
{
    const long in = (long)p * m1 * s1, out = (long)q * m2 * s2;
    memset(W, 0, sizeof(double) * (size_t)in * out);
    for (int i = 0; i < r; ++i)
        for (int a = 0; a < p; ++a)
            for (int c = 0; c < q; ++c) {
                const double av = A[((long)i * p + a) * q + c];
                for (int j = 0; j < m1; ++j)
                    for (int k = 0; k < m2; ++k) {
                        const double bv = B[((long)i * m1 + j) * m2 + k];
                        for (int u = 0; u < s1; ++u)
                            for (int v = 0; v < s2; ++v)
                                W[(((long)a * m1 + j) * s1 + u) * out + ((long)c * m2 + k) * s2 + v] +=
                                    av * bv * C[((long)i * s1 + u) * s2 + v];
                    }
            }
}

void oracle_forward3(const double *x, const double *A, const double *B, const double *C,
                     const double *bias, long N, int p, int q, int m1, int m2, int s1, int s2,
                     int r, double *y)
{
    const long in = (long)p * m1 * s1, out = (long)q * m2 * s2;
    double *W = (double *)malloc(sizeof(double) * (size_t)in * out);
    oracle_build_weight3(A, B, C, p, q, m1, m2, s1, s2, r, W);
    oracle_matmul_bias(x, W, bias, N, in, out, y);
    free(W);
}

void oracle_backward3(const double *x, const double *A, const double *B, const double *C,
                      const double *G, long N, int p, int q, int m1, int m2, int s1, int s2,
                      int r, double *dX, double *dA, double *dB, double *dC, double *dbias)
{
    const long in = (long)p * m1 * s1, out = (long)q * m2 * s2;
    double *W = (double *)malloc(sizeof(double) * (size_t)in * out);
    double *dW = (double *)calloc((size_t)in * out, sizeof(double));
    oracle_build_weight3(A, B, C, p, q, m1, m2, s1, s2, r, W);
    /* dX = G W^T */
#pragma omp parallel for
    for (long n = 0; n < N; ++n)
        for (long u = 0; u < in; ++u) {
            double s = 0.0;
            for (long o = 0; o < out; ++o) s += G[n * out + o] * W[u * out + o];
            dX[n * in + u] = s;
        }
    /* dW = x^T G */
#pragma omp parallel for
    for (long u = 0; u < in; ++u)
        for (long n = 0; n < N; ++n) {
            const double xv = x[n * in + u];
            for (long o = 0; o < out; ++o) dW[u * out + o] += xv * G[n * out + o];
        }
    for (int i = 0; i < r; ++i) {
        for (int a = 0; a < p; ++a)
            for (int c = 0; c < q; ++c) {
                double s = 0.0;
                for (int j = 0; j < m1; ++j)
                    for (int k = 0; k < m2; ++k)
                        for (int u = 0; u < s1; ++u)
                            for (int v = 0; v < s2; ++v)
                                s += dW[(((long)a * m1 + j) * s1 + u) * out + ((long)c * m2 + k) * s2 + v] *
                                     B[((long)i * m1 + j) * m2 + k] * C[((long)i * s1 + u) * s2 + v];
                dA[((long)i * p + a) * q + c] = s;
            }
        for (int j = 0; j < m1; ++j)
            for (int k = 0; k < m2; ++k) {
                double s = 0.0;
                for (int a = 0; a < p; ++a)
                    for (int c = 0; c < q; ++c)
                        for (int u = 0; u < s1; ++u)
                            for (int v = 0; v < s2; ++v)
                                s += dW[(((long)a * m1 + j) * s1 + u) * out + ((long)c * m2 + k) * s2 + v] *
                                     A[((long)i * p + a) * q + c] * C[((long)i * s1 + u) * s2 + v];
                dB[((long)i * m1 + j) * m2 + k] = s;
            }
        for (int u = 0; u < s1; ++u)
            for (int v = 0; v < s2; ++v) {
                double s = 0.0;
                for (int a = 0; a < p; ++a)
                    for (int c = 0; c < q; ++c)
                        for (int j = 0; j < m1; ++j)
                            for (int k = 0; k < m2; ++k)
                                s += dW[(((long)a * m1 + j) * s1 + u) * out + ((long)c * m2 + k) * s2 + v] *
                                     A[((long)i * p + a) * q + c] * B[((long)i * m1 + j) * m2 + k];
                dC[((long)i * s1 + u) * s2 + v] = s;
            }
    }
    for (long o = 0; o < out; ++o) {
        double s = 0.0;
        for (long n = 0; n < N; ++n) s += G[n * out + o];
        dbias[o] = s;
    }
    free(W);
    free(dW);
}

/*
 * Kronecker-sparse (KS) factor (page "Fast Inference with Kronecker-Sparse Matrices",
 * abstract): a matrix whose support is a Kronecker product of identity and all-ones blocks.
 * Pattern (a, b, c, d) names the support kron(I_a, kron(1_{b x c}, I_d)) of an
 * (a*b*d) x (a*c*d) matrix K, used here as the weight of y = x K + bias.  Its a*b*c*d free
 * entries are the values w [a][d][b][c]:
 *
 *     K[(al*b + be)*d + de][(al*c + ga)*d + de] = w[al][de][be][ga],   zero elsewhere.
 *
 * The oracle builds K entry by entry and multiplies naively (oracle_matmul_bias); the
 * backward is the chain rule through that explicit K:
 *     dX = G K^T,   dK = x^T G,   dw[al][de][be][ga] = dK at the entry w fills,
 *     dbias = sum_n G[n].
 * x [N][a*b*d], y and G [N][a*c*d], bias [a*c*d].
 */
void oracle_ks_build(const double *w, int a, int b, int c, int d, double *K)
{
    const long in = (long)a * b * d, out = (long)a * c * d;
    memset(K, 0, sizeof(double) * (size_t)in * out);
    for (int al = 0; al < a; ++al)
        for (int de = 0; de < d; ++de)
            for (int be = 0; be < b; ++be)
                for (int ga = 0; ga < c; ++ga)
                    K[(((long)al * b + be) * d + de) * out + ((long)al * c + ga) * d + de] =
                        w[(((long)al * d + de) * b + be) * c + ga];
}

void oracle_ks_forward(const double *x, const double *w, const double *bias, long N, int a,
                       int b, int c, int d, double *y)
{
    const long in = (long)a * b * d, out = (long)a * c * d;
    double *K = (double *)malloc(sizeof(double) * (size_t)in * out);
    oracle_ks_build(w, a, b, c, d, K);
    oracle_matmul_bias(x, K, bias, N, in, out, y);
    free(K);
}

void oracle_ks_backward(const double *x, const double *w, const double *G, long N, int a, int b,
                        int c, int d, double *dX, double *dw, double *dbias)
{
    const long in = (long)a * b * d, out = (long)a * c * d;
    double *K = (double *)malloc(sizeof(double) * (size_t)in * out);
    double *dK = (double *)calloc((size_t)in * out, sizeof(double));
    oracle_ks_build(w, a, b, c, d, K);
    /* dX = G K^T */
#pragma omp parallel for
    for (long n = 0; n < N; ++n)
        for (long u = 0; u < in; ++u) {
            double s = 0.0;
            for (long o = 0; o < out; ++o) s += G[n * out + o] * K[u * out + o];
            dX[n * in + u] = s;
        }
    /* dK = x^T G */
#pragma omp parallel for
    for (long u = 0; u < in; ++u)
        for (long n = 0; n < N; ++n) {
            const double xv = x[n * in + u];
            for (long o = 0; o < out; ++o) dK[u * out + o] += xv * G[n * out + o];
        }
    for (int al = 0; al < a; ++al)
        for (int de = 0; de < d; ++de)
            for (int be = 0; be < b; ++be)
                for (int ga = 0; ga < c; ++ga)
                    dw[(((long)al * d + de) * b + be) * c + ga] =
                        dK[(((long)al * b + be) * d + de) * out + ((long)al * c + ga) * d + de];
    for (long o = 0; o < out; ++o) {
        double s = 0.0;
        for (long n = 0; n < N; ++n) s += G[n * out + o];
        dbias[o] = s;
    }
    free(K);
    free(dK);
}
