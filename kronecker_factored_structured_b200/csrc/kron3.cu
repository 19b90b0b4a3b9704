// kron3.cu -- the triple Kronecker layer of the page "LLM Compression via Kronecker Product
// Decomposition" (section "Triple Kronecker -- AxBxC (Extreme Compression)"), with r terms:
//
//     y = x W + bias,   W = sum_i kron(A_i, kron(B_i, C_i)),
//     A_i p x q,  B_i m1 x m2,  C_i s1 x s2,  W (p*m1*s1) x (q*m2*s2).
//
// kron(A_i, kron(B_i, C_i)) is this library's two-factor layer with S = ones and the block
// factor B'_i = kron(B_i, C_i) ((m1*s1) x (m2*s2)).  B' is block-sized (kilobytes), so it is
// formed once per call and the two-factor kernels (tensor cores where the shape has them)
// run unchanged: the vec trick's two on-chip stages with the inner Kronecker folded into the
// block.  The backward takes dA = dC' (S = ones) and dB' from the two-factor backward and
// chains dB' back to the inner factors:
//     dB_i[j][k] = sum_{u,v} dB'_i[j*s1+u][k*s2+v] C_i[u][v]
//     dC_i[u][v] = sum_{j,k} dB'_i[j*s1+u][k*s2+v] B_i[j][k]
// (fixed-order double sums: bitwise reproducible).
#include "../../include/kron_linear.h"
#include "internal.h"

#include <cuda_bf16.h>
#include <stdarg.h>
#include <stdio.h>

namespace kron {
kron_status_t report_failure(kron_status_t st, const char *msg);
}

namespace {

struct K3Layout {
    size_t s, bp, ds, dbp, ws2, total;
};

inline size_t a256(size_t x) { return (x + 255) & ~(size_t)255; }

K3Layout k3_layout(int64_t N, int p, int q, int m1, int m2, int s1, int s2, int r,
                   kron_dtype_t dtype, bool backward) {
    const size_t e = dtype == KRON_BF16 ? 2 : 4;
    const size_t bpn = (size_t)r * m1 * s1 * m2 * s2;
    K3Layout L;
    size_t o = 0;
    L.s = o;   o = a256(o + (size_t)p * q * e);
    L.bp = o;  o = a256(o + bpn * e);
    L.ds = o;  o = backward ? a256(o + (size_t)p * q * 4) : o;
    L.dbp = o; o = backward ? a256(o + bpn * 4) : o;
    L.ws2 = o;
    if (backward) o += kron_linear_workspace_size(N, p, q, m1 * s1, m2 * s2, r, dtype);
    L.total = o;
    return L;
}

template <typename T> __device__ __forceinline__ float ldv(const T *p, size_t i);
template <> __device__ __forceinline__ float ldv<float>(const float *p, size_t i) { return p[i]; }
template <> __device__ __forceinline__ float ldv<__nv_bfloat16>(const __nv_bfloat16 *p, size_t i) {
    return __bfloat162float(p[i]);
}
template <typename T> __device__ __forceinline__ T cvt(float v);
template <> __device__ __forceinline__ float cvt<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 cvt<__nv_bfloat16>(float v) {
    return __float2bfloat16_rn(v);
}

// S = ones (p x q) and B'_i[j*s1+u][k*s2+v] = B_i[j][k] C_i[u][v] (rounded once to T)
template <typename T>
__global__ void k3_prepare(const T *B, const T *C, T *S, T *Bp, int p, int q, int m1, int m2,
                           int s1, int s2, int r) {
    const int64_t nb = (int64_t)r * m1 * s1 * m2 * s2, ns = (int64_t)p * q;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < nb + ns;
         e += (int64_t)gridDim.x * blockDim.x) {
        if (e >= nb) {
            S[e - nb] = cvt<T>(1.f);
            continue;
        }
        const int64_t cols = (int64_t)m2 * s2;
        const int64_t blk = (int64_t)m1 * s1 * cols;
        const int i = (int)(e / blk);
        const int64_t rem = e % blk, row = rem / cols, col = rem % cols;
        const int j = (int)(row / s1), u = (int)(row % s1), k = (int)(col / s2), v = (int)(col % s2);
        Bp[e] = cvt<T>(ldv(B, ((size_t)i * m1 + j) * m2 + k) * ldv(C, ((size_t)i * s1 + u) * s2 + v));
    }
}

// dB and dC from dB' by the chain rule through B' = kron(B, C)
template <typename T>
__global__ void k3_chain(const float *dBp, const T *B, const T *C, float *dB, float *dC, int m1,
                         int m2, int s1, int s2, int r) {
    const int64_t nb = (int64_t)r * m1 * m2, nc = (int64_t)r * s1 * s2;
    const int64_t cols = (int64_t)m2 * s2, blk = (int64_t)m1 * s1 * cols;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < nb + nc;
         e += (int64_t)gridDim.x * blockDim.x) {
        double s = 0.0;
        if (e < nb) {
            const int i = (int)(e / ((int64_t)m1 * m2)), j = (int)(e / m2 % m1), k = (int)(e % m2);
            for (int u = 0; u < s1; ++u)
                for (int v = 0; v < s2; ++v)
                    s += (double)dBp[(size_t)i * blk + ((size_t)j * s1 + u) * cols + (size_t)k * s2 + v] *
                         ldv(C, ((size_t)i * s1 + u) * s2 + v);
            dB[e] = (float)s;
        } else {
            const int64_t f = e - nb;
            const int i = (int)(f / ((int64_t)s1 * s2)), u = (int)(f / s2 % s1), v = (int)(f % s2);
            for (int j = 0; j < m1; ++j)
                for (int k = 0; k < m2; ++k)
                    s += (double)dBp[(size_t)i * blk + ((size_t)j * s1 + u) * cols + (size_t)k * s2 + v] *
                         ldv(B, ((size_t)i * m1 + j) * m2 + k);
            dC[f] = (float)s;
        }
    }
}

kron_status_t k3_fail(kron_status_t st, const char *fmt, ...) __attribute__((format(printf, 2, 3)));
kron_status_t k3_fail(kron_status_t st, const char *fmt, ...) {
    char msg[256];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(msg, sizeof(msg), fmt, ap);
    va_end(ap);
    return kron::report_failure(st, msg);
}

kron_status_t k3_check(int p, int q, int m1, int m2, int s1, int s2, int r, kron_dtype_t dtype) {
    if (dtype != KRON_F32 && dtype != KRON_TF32 && dtype != KRON_BF16)
        return k3_fail(KRON_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
    if (p < 1 || q < 1 || m1 < 1 || m2 < 1 || s1 < 1 || s2 < 1 || r < 1)
        return k3_fail(KRON_ERR_INVALID_ARG, "sizes must be >= 1");
    if ((int64_t)m1 * s1 > (1 << 16) || (int64_t)m2 * s2 > (1 << 16) || r > 4096)
        return k3_fail(KRON_ERR_INVALID_ARG, "sizes out of range");
    return KRON_OK;
}

bool a16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

}  // namespace

extern "C" {

size_t kron3_linear_workspace_size(int64_t N, int p, int q, int m1, int m2, int s1, int s2, int r,
                                   kron_dtype_t dtype, int backward) {
    if (N < 0 || k3_check(p, q, m1, m2, s1, s2, r, dtype) != KRON_OK) return 0;
    if (backward && kron_linear_workspace_size(N, p, q, m1 * s1, m2 * s2, r, dtype) == 0) return 0;
    return k3_layout(N, p, q, m1, m2, s1, s2, r, dtype, backward != 0).total;
}

kron_status_t kron3_linear_forward(const void *x, const void *A, const void *B, const void *C,
                                   const void *bias, void *y, int64_t N, int p, int q, int m1,
                                   int m2, int s1, int s2, int r, kron_dtype_t dtype,
                                   unsigned flags, void *workspace, size_t workspace_bytes,
                                   void *stream) {
    kron_status_t st = k3_check(p, q, m1, m2, s1, s2, r, dtype);
    if (st != KRON_OK) return st;
    if (!A || !B || !C) return k3_fail(KRON_ERR_INVALID_ARG, "A, B and C must be non-null");
    if (!a16(A) || !a16(B) || !a16(C))
        return k3_fail(KRON_ERR_ALIGNMENT, "all tensors must be 16-byte aligned");
    const K3Layout L = k3_layout(N, p, q, m1, m2, s1, s2, r, dtype, false);
    if (!workspace || workspace_bytes < L.total)
        return k3_fail(KRON_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", L.total,
                       workspace ? workspace_bytes : (size_t)0);
    if ((uintptr_t)workspace & 255u)
        return k3_fail(KRON_ERR_ALIGNMENT, "workspace must be 256-byte aligned");
    char *ws = static_cast<char *>(workspace);
    cudaStream_t cs = (cudaStream_t)stream;
    if (dtype == KRON_BF16)
        k3_prepare<__nv_bfloat16><<<148, 256, 0, cs>>>(
            (const __nv_bfloat16 *)B, (const __nv_bfloat16 *)C, (__nv_bfloat16 *)(ws + L.s),
            (__nv_bfloat16 *)(ws + L.bp), p, q, m1, m2, s1, s2, r);
    else
        k3_prepare<float><<<148, 256, 0, cs>>>((const float *)B, (const float *)C,
                                               (float *)(ws + L.s), (float *)(ws + L.bp), p, q,
                                               m1, m2, s1, s2, r);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return k3_fail(KRON_ERR_CUDA, "block-factor launch: %s", cudaGetErrorString(e));
    return kron_linear_forward(x, ws + L.s, A, ws + L.bp, bias, y, N, p, q, m1 * s1, m2 * s2, r,
                               dtype, flags, stream);
}

kron_status_t kron3_linear_backward(const void *x, const void *A, const void *B, const void *C,
                                    const void *dY, void *dX, void *dA, void *dB, void *dC,
                                    void *dbias, int64_t N, int p, int q, int m1, int m2, int s1,
                                    int s2, int r, kron_dtype_t dtype, unsigned flags,
                                    void *workspace, size_t workspace_bytes, void *stream) {
    kron_status_t st = k3_check(p, q, m1, m2, s1, s2, r, dtype);
    if (st != KRON_OK) return st;
    if (!A || !B || !C || !dA || !dB || !dC)
        return k3_fail(KRON_ERR_INVALID_ARG, "A, B, C, dA, dB and dC must be non-null");
    if (!a16(A) || !a16(B) || !a16(C) || !a16(dA) || !a16(dB) || !a16(dC))
        return k3_fail(KRON_ERR_ALIGNMENT, "all tensors must be 16-byte aligned");
    if (kron_linear_workspace_size(N, p, q, m1 * s1, m2 * s2, r, dtype) == 0)
        return k3_fail(KRON_ERR_UNSUPPORTED,
                       "no backward kernel for the block shape %d x %d (r = %d) on this path",
                       m1 * s1, m2 * s2, r);
    const K3Layout L = k3_layout(N, p, q, m1, m2, s1, s2, r, dtype, true);
    if (!workspace || workspace_bytes < L.total)
        return k3_fail(KRON_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", L.total,
                       workspace ? workspace_bytes : (size_t)0);
    if ((uintptr_t)workspace & 255u)
        return k3_fail(KRON_ERR_ALIGNMENT, "workspace must be 256-byte aligned");
    char *ws = static_cast<char *>(workspace);
    cudaStream_t cs = (cudaStream_t)stream;
    const bool bf = dtype == KRON_BF16;
    if (bf)
        k3_prepare<__nv_bfloat16><<<148, 256, 0, cs>>>(
            (const __nv_bfloat16 *)B, (const __nv_bfloat16 *)C, (__nv_bfloat16 *)(ws + L.s),
            (__nv_bfloat16 *)(ws + L.bp), p, q, m1, m2, s1, s2, r);
    else
        k3_prepare<float><<<148, 256, 0, cs>>>((const float *)B, (const float *)C,
                                               (float *)(ws + L.s), (float *)(ws + L.bp), p, q,
                                               m1, m2, s1, s2, r);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return k3_fail(KRON_ERR_CUDA, "block-factor launch: %s", cudaGetErrorString(e));
    st = kron_linear_backward(x, ws + L.s, A, ws + L.bp, dY, dX, ws + L.ds, dA, ws + L.dbp, dbias,
                              N, p, q, m1 * s1, m2 * s2, r, dtype, flags, ws + L.ws2,
                              workspace_bytes - L.ws2, stream);
    if (st != KRON_OK) return st;
    if (bf)
        k3_chain<__nv_bfloat16><<<148, 256, 0, cs>>>((const float *)(ws + L.dbp),
                                                     (const __nv_bfloat16 *)B,
                                                     (const __nv_bfloat16 *)C, (float *)dB,
                                                     (float *)dC, m1, m2, s1, s2, r);
    else
        k3_chain<float><<<148, 256, 0, cs>>>((const float *)(ws + L.dbp), (const float *)B,
                                             (const float *)C, (float *)dB, (float *)dC, m1, m2,
                                             s1, s2, r);
    e = cudaGetLastError();
    if (e != cudaSuccess)
        return k3_fail(KRON_ERR_CUDA, "inner-factor gradient launch: %s", cudaGetErrorString(e));
    return KRON_OK;
}

}  // extern "C"
