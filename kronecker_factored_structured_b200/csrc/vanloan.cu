// vanloan.cu -- rank-r Kronecker fit of a dense matrix on the GPU (the page "LLM Compression
// via Kronecker Product Decomposition", sections "Van Loan Rearrangement (1993)", "Rank-K"
// and "Adaptive Normalization"), to initialise this layer's factors from a dense W.
//
//   1. Wt = R(W): Wt[a*q + c][j*m2 + k] = W[a*m1 + j][c*m2 + k]  ((p*q) x (m1*m2)); then
//      W = sum_i kron(C_i, B_i) exactly when Wt = sum_i vec(C_i) vec(B_i)^T, so the best
//      Kronecker sum of r terms comes from the r leading singular pairs of Wt.
//   2. Those pairs by randomized subspace iteration (Halko, Martinsson and Tropp, "Finding
//      structure with randomness", 2011, the range finder with power iterations): Q = orth(Wt
//      Omega), then `power_iters` times Q = orth(Wt orth(Wt^T Q)); Bs = Q^T Wt (k x n); the
//      eigenpairs of the k x k Gram matrix Bs Bs^T = V diag(lambda) V^T give sigma = sqrt(lambda),
//      u = Q V and v = Bs^T V / sigma.  Omega (n x k, k >= r) is the caller's random matrix.
//   3. C_i = sqrt(sigma_i) reshape(u_i, p, q), B_i = sqrt(sigma_i) reshape(v_i, m1, m2), i < r.
//   4. alpha = |W|_F / |sum_i kron(C_i, B_i)|_F, and with `normalize` both factors of every
//      term are scaled by sqrt(alpha).
// Sums run in double in a fixed order (no atomics), so the fit is bitwise reproducible.
// Dense products are small next to a layer pass; they run on the CUDA cores.
#include "../../include/kron_linear.h"
#include "internal.h"

#include <math.h>
#include <stdarg.h>
#include <stdio.h>

namespace kron {
kron_status_t report_failure(kron_status_t st, const char *msg);
}

namespace {

constexpr int kMaxK = 64;
constexpr int kNormParts = 256;   // CTAs of the |W|_F^2 partial sums

struct VLSizes {
    int p, q, m1, m2, r, k;
    int64_t m() const { return (int64_t)p * q; }
    int64_t n() const { return (int64_t)m1 * m2; }
};

// workspace layout (byte offsets, 256-aligned)
struct VLLayout {
    size_t wt, qm, zn, gram, vec, lam, norm, total;
};
inline size_t al256(size_t x) { return (x + 255) & ~(size_t)255; }
VLLayout vl_layout(const VLSizes &s) {
    VLLayout L;
    size_t o = 0;
    L.wt = o;   o = al256(o + (size_t)s.m() * s.n() * sizeof(float));
    L.qm = o;   o = al256(o + (size_t)s.k * s.m() * sizeof(double));
    L.zn = o;   o = al256(o + (size_t)s.k * s.n() * sizeof(double));
    L.gram = o; o = al256(o + (size_t)kMaxK * kMaxK * sizeof(double));
    L.vec = o;  o = al256(o + (size_t)kMaxK * kMaxK * sizeof(double));
    L.lam = o;  o = al256(o + (size_t)kMaxK * sizeof(double));
    L.norm = o; o = al256(o + (size_t)(kNormParts + 2) * sizeof(double));
    L.total = o;
    return L;
}

__global__ void k_rearrange(const float *__restrict__ W, float *__restrict__ Wt, int p, int q,
                            int m1, int m2) {
    const int64_t n = (int64_t)m1 * m2, total = (int64_t)p * q * n;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t row = e / n, col = e % n;
        const int a = (int)(row / q), c = (int)(row % q);
        const int j = (int)(col / m2), kk = (int)(col % m2);
        Wt[e] = W[((int64_t)a * m1 + j) * ((int64_t)q * m2) + (int64_t)c * m2 + kk];
    }
}

// Y[c][row] = sum_j Wt[row][j] X[c][j]   (Wt: m x n fp32; X: k x n; Y: k x m, double)
// A CTA takes 32 rows; the j range is walked in tiles of 32 staged in shared memory.
template <typename TX>
__global__ void __launch_bounds__(256) k_mul_rows(const float *__restrict__ Wt,
                                                  const TX *__restrict__ X, double *__restrict__ Y,
                                                  int64_t m, int64_t n, int k) {
    __shared__ float ws[32][33];
    __shared__ double xs[kMaxK][33];
    const int t = threadIdx.x, r = t / 8, cg = t % 8;
    const int64_t row0 = (int64_t)blockIdx.x * 32;
    double acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int64_t j0 = 0; j0 < n; j0 += 32) {
        for (int e = t; e < 32 * 32; e += 256) {
            const int rr = e / 32, jj = e % 32;
            ws[rr][jj] = (row0 + rr < m && j0 + jj < n) ? Wt[(row0 + rr) * n + j0 + jj] : 0.f;
        }
        for (int e = t; e < k * 32; e += 256) {
            const int c = e / 32, jj = e % 32;
            xs[c][jj] = j0 + jj < n ? (double)X[(int64_t)c * n + j0 + jj] : 0.0;
        }
        __syncthreads();
        for (int jj = 0; jj < 32; ++jj) {
            const double w = ws[r][jj];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int c = cg + 8 * u;
                if (c < k) acc[u] += w * xs[c][jj];
            }
        }
        __syncthreads();
    }
    if (row0 + r < m) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int c = cg + 8 * u;
            if (c < k) Y[(int64_t)c * m + row0 + r] = acc[u];
        }
    }
}

// Z[c][j] = sum_row Wt[row][j] Q[c][row]   (Z: k x n, double).  A CTA takes 32 columns j.
__global__ void __launch_bounds__(256) k_mul_cols(const float *__restrict__ Wt,
                                                  const double *__restrict__ Q,
                                                  double *__restrict__ Z, int64_t m, int64_t n,
                                                  int k) {
    __shared__ float ws[32][33];    // [row][j]
    __shared__ double qs[kMaxK][33];
    const int t = threadIdx.x, jl = t / 8, cg = t % 8;
    const int64_t j0 = (int64_t)blockIdx.x * 32;
    double acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int64_t r0 = 0; r0 < m; r0 += 32) {
        for (int e = t; e < 32 * 32; e += 256) {
            const int rr = e / 32, jj = e % 32;
            ws[rr][jj] = (r0 + rr < m && j0 + jj < n) ? Wt[(r0 + rr) * n + j0 + jj] : 0.f;
        }
        for (int e = t; e < k * 32; e += 256) {
            const int c = e / 32, rr = e % 32;
            qs[c][rr] = r0 + rr < m ? Q[(int64_t)c * m + r0 + rr] : 0.0;
        }
        __syncthreads();
        for (int rr = 0; rr < 32; ++rr) {
            const double w = ws[rr][jl];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int c = cg + 8 * u;
                if (c < k) acc[u] += w * qs[c][rr];
            }
        }
        __syncthreads();
    }
    if (j0 + jl < n) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int c = cg + 8 * u;
            if (c < k) Z[(int64_t)c * n + j0 + jl] = acc[u];
        }
    }
}

// Sum over a block of 1024 threads in a fixed order (warp shuffles, then warp 0).
__device__ double block_sum(double v, double *red) {
    for (int o = 16; o > 0; o >>= 1) v += __shfl_down_sync(0xffffffffu, v, o);
    const int w = threadIdx.x / 32, l = threadIdx.x % 32;
    __syncthreads();
    if (l == 0) red[w] = v;
    __syncthreads();
    double s = 0.0;
    if (w == 0) {
        s = l < (int)(blockDim.x / 32) ? red[l] : 0.0;
        for (int o = 16; o > 0; o >>= 1) s += __shfl_down_sync(0xffffffffu, s, o);
        if (l == 0) red[32] = s;
    }
    __syncthreads();
    return red[32];
}

// Orthonormal columns in place: X is k vectors of length len (X[c][*]), by classical
// Gram-Schmidt applied twice per vector; a vector with nothing left after the projections
// (the range of X has fewer than k dimensions) becomes zero.
__global__ void __launch_bounds__(1024) k_orthonormalize(double *X, int64_t len, int k) {
    __shared__ double red[33];
    __shared__ double dots[kMaxK];
    const int t = threadIdx.x, w = t / 32, l = t % 32;
    for (int c = 0; c < k; ++c) {
        double *xc = X + (int64_t)c * len;
        for (int pass = 0; pass < 2; ++pass) {
            // dots with the finished vectors: warp w takes vectors w, w + 32
            for (int i = w; i < c; i += 32) {
                const double *xi = X + (int64_t)i * len;
                double s = 0.0;
                for (int64_t e = l; e < len; e += 32) s += xi[e] * xc[e];
                for (int o = 16; o > 0; o >>= 1) s += __shfl_down_sync(0xffffffffu, s, o);
                if (l == 0) dots[i] = s;
            }
            __syncthreads();
            for (int64_t e = t; e < len; e += blockDim.x) {
                double v = xc[e];
                for (int i = 0; i < c; ++i) v -= dots[i] * X[(int64_t)i * len + e];
                xc[e] = v;
            }
            __syncthreads();
        }
        double s = 0.0;
        for (int64_t e = t; e < len; e += blockDim.x) s += xc[e] * xc[e];
        const double nrm = sqrt(block_sum(s, red));
        const double inv = nrm > 1e-280 ? 1.0 / nrm : 0.0;
        for (int64_t e = t; e < len; e += blockDim.x) xc[e] *= inv;
        __syncthreads();
    }
}

// G[c1][c2] = sum_j Z[c1][j] Z[c2][j]: CTA c1, one warp per c2 >= c1 (mirrored).
__global__ void __launch_bounds__(256) k_gram(const double *__restrict__ Z, double *G, int64_t n,
                                              int k) {
    const int c1 = blockIdx.x, w = threadIdx.x / 32, l = threadIdx.x % 32;
    for (int c2 = c1 + w; c2 < k; c2 += 8) {
        double s = 0.0;
        for (int64_t e = l; e < n; e += 32) s += Z[(int64_t)c1 * n + e] * Z[(int64_t)c2 * n + e];
        for (int o = 16; o > 0; o >>= 1) s += __shfl_down_sync(0xffffffffu, s, o);
        if (l == 0) {
            G[c1 * kMaxK + c2] = s;
            G[c2 * kMaxK + c1] = s;
        }
    }
}

// Eigenpairs of the symmetric k x k matrix G by cyclic Jacobi in parallel (round-robin)
// order: each round rotates k/2 disjoint index pairs.  The rotations accumulate in Vw
// (global scratch); at the end G is overwritten with the eigenvectors in columns, ordered
// by eigenvalue from the largest, and lam receives the eigenvalues in that order.
__global__ void __launch_bounds__(1024) k_jacobi(double *G, double *Vw, double *lam, int k) {
    __shared__ double A[kMaxK][kMaxK + 1];
    __shared__ double cs[kMaxK / 2], sn[kMaxK / 2];
    __shared__ int pp[kMaxK / 2], qq[kMaxK / 2];
    __shared__ double off;
    __shared__ int order[kMaxK];
    const int t = threadIdx.x;
    const int ke = k + (k & 1);   // even number of players (index k is a dummy when k is odd)
    for (int e = t; e < kMaxK * kMaxK; e += blockDim.x) {
        const int i = e / kMaxK, j = e % kMaxK;
        A[i][j] = (i < k && j < k) ? G[i * kMaxK + j] : 0.0;
        Vw[e] = i == j ? 1.0 : 0.0;
    }
    __syncthreads();
    for (int sweep = 0; sweep < 40; ++sweep) {
        if (t == 0) {
            double o = 0.0, d = 0.0;
            for (int i = 0; i < k; ++i)
                for (int j = 0; j < k; ++j) (i == j ? d : o) += A[i][j] * A[i][j];
            off = (o <= 1e-30 * d || d == 0.0) ? -1.0 : o;
        }
        __syncthreads();
        if (off < 0.0) break;
        for (int rd = 0; rd < ke - 1; ++rd) {
            if (t < ke / 2) {
                int a, b;
                if (t == 0) {
                    a = 0;
                    b = 1 + rd;
                } else {
                    a = 1 + (rd + t) % (ke - 1);
                    b = 1 + (rd - t + ke - 1) % (ke - 1);
                }
                if (a > b) { const int x = a; a = b; b = x; }
                double c = 1.0, s = 0.0;
                if (b < k && A[a][b] != 0.0) {
                    const double th = (A[b][b] - A[a][a]) / (2.0 * A[a][b]);
                    const double tt = (th >= 0.0 ? 1.0 : -1.0) / (fabs(th) + sqrt(th * th + 1.0));
                    c = 1.0 / sqrt(tt * tt + 1.0);
                    s = tt * c;
                }
                pp[t] = a; qq[t] = b; cs[t] = c; sn[t] = s;
            }
            __syncthreads();
            // rows: A <- J^T A
            for (int e = t; e < (ke / 2) * kMaxK; e += blockDim.x) {
                const int pr = e / kMaxK, j = e % kMaxK, a = pp[pr], b = qq[pr];
                if (b < k) {
                    const double x = A[a][j], y = A[b][j];
                    A[a][j] = cs[pr] * x - sn[pr] * y;
                    A[b][j] = sn[pr] * x + cs[pr] * y;
                }
            }
            __syncthreads();
            // columns: A <- A J, V <- V J
            for (int e = t; e < (ke / 2) * kMaxK; e += blockDim.x) {
                const int pr = e / kMaxK, i = e % kMaxK, a = pp[pr], b = qq[pr];
                if (b < k) {
                    const double x = A[i][a], y = A[i][b];
                    A[i][a] = cs[pr] * x - sn[pr] * y;
                    A[i][b] = sn[pr] * x + cs[pr] * y;
                    const double vx = Vw[i * kMaxK + a], vy = Vw[i * kMaxK + b];
                    Vw[i * kMaxK + a] = cs[pr] * vx - sn[pr] * vy;
                    Vw[i * kMaxK + b] = sn[pr] * vx + cs[pr] * vy;
                }
            }
            __syncthreads();
        }
    }
    if (t == 0) {   // order by eigenvalue, largest first (stable)
        for (int i = 0; i < k; ++i) order[i] = i;
        for (int i = 1; i < k; ++i) {
            const int x = order[i];
            int j = i - 1;
            while (j >= 0 && A[order[j]][order[j]] < A[x][x]) {
                order[j + 1] = order[j];
                --j;
            }
            order[j + 1] = x;
        }
    }
    __syncthreads();
    for (int e = t; e < k * k; e += blockDim.x) {
        const int i = e / k, j = e % k;
        G[i * kMaxK + j] = Vw[i * kMaxK + order[j]];
    }
    if (t < k) lam[t] = A[order[t]][order[t]];
}

// C_i = sqrt(sigma_i) Q V[:, i]  (reshaped p x q)  and  B_i = Z^T V[:, i] / sqrt(sigma_i)
// (= sqrt(sigma_i) v_i), i < r; sigma_c = sqrt(max(lambda_c, 0)) for every c < k.
__global__ void k_assemble(const double *__restrict__ Q, const double *__restrict__ Z,
                           const double *__restrict__ V, const double *__restrict__ lam,
                           float *A, float *B, float *sigma, int64_t m, int64_t n, int r, int k) {
    const int64_t tot = (int64_t)r * (m + n);
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < tot;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int i = (int)(e / (m + n));
        const int64_t o = e % (m + n);
        const double sg = sqrt(fmax(lam[i], 0.0));
        double s = 0.0;
        if (o < m) {
            for (int c = 0; c < k; ++c) s += Q[(int64_t)c * m + o] * V[c * kMaxK + i];
            A[(int64_t)i * m + o] = (float)(sqrt(sg) * s);
        } else {
            const int64_t j = o - m;
            for (int c = 0; c < k; ++c) s += Z[(int64_t)c * n + j] * V[c * kMaxK + i];
            B[(int64_t)i * n + j] = sg > 0.0 ? (float)(s / sqrt(sg)) : 0.f;
        }
    }
    if (blockIdx.x == 0 && threadIdx.x < k)
        sigma[threadIdx.x] = (float)sqrt(fmax(lam[threadIdx.x], 0.0));
}

// |W|_F^2 in kNormParts fixed slices (one per CTA)
__global__ void __launch_bounds__(1024) k_sumsq_parts(const float *__restrict__ W, int64_t total,
                                                      double *parts) {
    __shared__ double red[33];
    const int64_t per = (total + gridDim.x - 1) / gridDim.x;
    const int64_t e0 = (int64_t)blockIdx.x * per, e1 = e0 + per < total ? e0 + per : total;
    double s = 0.0;
    for (int64_t e = e0 + threadIdx.x; e < e1; e += blockDim.x) s += (double)W[e] * W[e];
    s = block_sum(s, red);
    if (threadIdx.x == 0) parts[blockIdx.x] = s;
}

// alpha = |W|_F / |sum_i kron(C_i, B_i)|_F, with |sum_i kron(C_i, B_i)|_F^2 =
// sum_{i,l} <C_i, C_l> <B_i, B_l>; with normalize, C and B are scaled by sqrt(alpha).
__global__ void __launch_bounds__(1024) k_alpha(const double *parts, int nparts, float *A, float *B,
                                                int64_t m, int64_t n, int r, int normalize,
                                                float *alpha_out) {
    __shared__ double red[33];
    __shared__ double alpha_s;
    double f2 = 0.0;   // meaningful in thread 0
    for (int i = 0; i < r; ++i)
        for (int l = i; l < r; ++l) {
            double sc = 0.0, sb = 0.0;
            for (int64_t e = threadIdx.x; e < m; e += blockDim.x)
                sc += (double)A[(int64_t)i * m + e] * A[(int64_t)l * m + e];
            for (int64_t e = threadIdx.x; e < n; e += blockDim.x)
                sb += (double)B[(int64_t)i * n + e] * B[(int64_t)l * n + e];
            sc = block_sum(sc, red);
            sb = block_sum(sb, red);
            f2 += (i == l ? 1.0 : 2.0) * sc * sb;
        }
    if (threadIdx.x == 0) {
        double w2 = 0.0;
        for (int b = 0; b < nparts; ++b) w2 += parts[b];
        alpha_s = f2 > 0.0 ? sqrt(w2 / f2) : 1.0;
        *alpha_out = (float)alpha_s;
    }
    __syncthreads();
    if (normalize) {
        const float sa = (float)sqrt(alpha_s);
        for (int64_t e = threadIdx.x; e < (int64_t)r * m; e += blockDim.x) A[e] *= sa;
        for (int64_t e = threadIdx.x; e < (int64_t)r * n; e += blockDim.x) B[e] *= sa;
    }
}

bool al16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

kron_status_t vl_fail(kron_status_t st, const char *fmt, ...) __attribute__((format(printf, 2, 3)));
kron_status_t vl_fail(kron_status_t st, const char *fmt, ...) {
    char msg[256];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(msg, sizeof(msg), fmt, ap);
    va_end(ap);
    return kron::report_failure(st, msg);
}

kron_status_t vl_check_sizes(int p, int q, int m1, int m2, int k) {
    if (p < 1 || q < 1 || m1 < 1 || m2 < 1)
        return vl_fail(KRON_ERR_INVALID_ARG, "p, q, m1, m2 must be >= 1");
    if ((int64_t)p * q > (1 << 22) || (int64_t)m1 * m2 > (1 << 22) ||
        (int64_t)p * q * m1 * m2 > ((int64_t)1 << 32))
        return vl_fail(KRON_ERR_INVALID_ARG, "sizes out of range");
    if (k < 1 || k > kMaxK)
        return vl_fail(KRON_ERR_INVALID_ARG, "k must be in [1, %d] (got %d)", kMaxK, k);
    if ((int64_t)k > (int64_t)p * q || (int64_t)k > (int64_t)m1 * m2)
        return vl_fail(KRON_ERR_INVALID_ARG, "k must not exceed p*q or m1*m2 (got %d)", k);
    return KRON_OK;
}

}  // namespace

extern "C" {

size_t kron_vanloan_workspace_size(int p, int q, int m1, int m2, int k) {
    if (vl_check_sizes(p, q, m1, m2, k) != KRON_OK) return 0;
    return vl_layout(VLSizes{p, q, m1, m2, 1, k}).total;
}

kron_status_t kron_vanloan_fit(const void *W, int p, int q, int m1, int m2, int r,
                               const void *omega, int k, int power_iters, int normalize,
                               void *A, void *B, void *sigma, void *alpha, void *workspace,
                               size_t workspace_bytes, void *stream) {
    kron_status_t st = vl_check_sizes(p, q, m1, m2, k);
    if (st != KRON_OK) return st;
    if (r < 1 || r > k) return vl_fail(KRON_ERR_INVALID_ARG, "r must be in [1, k] (got %d)", r);
    if (power_iters < 0 || power_iters > 16)
        return vl_fail(KRON_ERR_INVALID_ARG, "power_iters must be in [0, 16] (got %d)",
                       power_iters);
    if (!W || !omega || !A || !B || !sigma || !alpha)
        return vl_fail(KRON_ERR_INVALID_ARG, "W, omega, A, B, sigma and alpha must be non-null");
    if (!al16(W) || !al16(omega) || !al16(A) || !al16(B) || !al16(sigma) || !al16(alpha))
        return vl_fail(KRON_ERR_ALIGNMENT, "all tensors must be 16-byte aligned");
    const VLSizes s{p, q, m1, m2, r, k};
    const VLLayout L = vl_layout(s);
    if (!workspace || workspace_bytes < L.total)
        return vl_fail(KRON_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", L.total,
                       workspace ? workspace_bytes : (size_t)0);
    if ((uintptr_t)workspace & 255u)
        return vl_fail(KRON_ERR_ALIGNMENT, "workspace must be 256-byte aligned");
    cudaStream_t cs = (cudaStream_t)stream;
    char *ws = static_cast<char *>(workspace);
    float *Wt = reinterpret_cast<float *>(ws + L.wt);
    double *Qm = reinterpret_cast<double *>(ws + L.qm);
    double *Zn = reinterpret_cast<double *>(ws + L.zn);
    double *G = reinterpret_cast<double *>(ws + L.gram);
    double *V = reinterpret_cast<double *>(ws + L.vec);
    double *lam = reinterpret_cast<double *>(ws + L.lam);
    double *nrm = reinterpret_cast<double *>(ws + L.norm);
    const int64_t m = s.m(), n = s.n();
    const float *Wf = static_cast<const float *>(W);
    const int rows_blocks = (int)((m + 31) / 32), cols_blocks = (int)((n + 31) / 32);
    k_rearrange<<<1184, 256, 0, cs>>>(Wf, Wt, p, q, m1, m2);
    k_mul_rows<float><<<rows_blocks, 256, 0, cs>>>(Wt, static_cast<const float *>(omega), Qm, m, n, k);
    k_orthonormalize<<<1, 1024, 0, cs>>>(Qm, m, k);
    for (int it = 0; it < power_iters; ++it) {
        k_mul_cols<<<cols_blocks, 256, 0, cs>>>(Wt, Qm, Zn, m, n, k);
        k_orthonormalize<<<1, 1024, 0, cs>>>(Zn, n, k);
        k_mul_rows<double><<<rows_blocks, 256, 0, cs>>>(Wt, Zn, Qm, m, n, k);
        k_orthonormalize<<<1, 1024, 0, cs>>>(Qm, m, k);
    }
    k_mul_cols<<<cols_blocks, 256, 0, cs>>>(Wt, Qm, Zn, m, n, k);   // Bs^T = Wt^T Q
    k_gram<<<k, 256, 0, cs>>>(Zn, G, n, k);
    k_jacobi<<<1, 1024, 0, cs>>>(G, V, lam, k);   // eigenvectors end up in G
    k_assemble<<<592, 256, 0, cs>>>(Qm, Zn, G, lam, static_cast<float *>(A),
                                    static_cast<float *>(B), static_cast<float *>(sigma), m, n, r, k);
    k_sumsq_parts<<<kNormParts, 1024, 0, cs>>>(Wf, m * n, nrm);
    k_alpha<<<1, 1024, 0, cs>>>(nrm, kNormParts, static_cast<float *>(A), static_cast<float *>(B),
                                m, n, r, normalize, static_cast<float *>(alpha));
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return vl_fail(KRON_ERR_CUDA, "Van Loan fit launch: %s", cudaGetErrorString(e));
    return KRON_OK;
}

}  // extern "C"
