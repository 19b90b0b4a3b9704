// reduce.cu -- deterministic reduction of the backward's row-range partials and the
// factor-gradient epilogue:
//   dC_i = sum over row ranges of the partial dC_i   (fixed order)
//   dA_i = dC_i (.) S,   dS = sum_i dC_i (.) A_i (+ l1 * sign(S)),   dB_i and dbias summed.
// (dA_i and dS follow from C_i = S (.) A_i by the product rule; W = sum_i kron(C_i, B_i)
// as on the page "kronecker-layer-benchmark", section "1. Build W, then multiply".  The
// optional l1 term is the gradient of the penalty l1 * sum|S| that the same page's
// introduction puts on S.)
//
// Workspace layout per range g: ws[g*stride + ...] = [dC: r*p*q][dB: r*m1*m2][dbias: q*m2].
// Each block owns 32 consecutive output columns (for dC: 32 (a,c) positions and all r
// ranks).  Its kWarps warps sum ranges g = w, w+kWarps, ... in double with several
// independent accumulators, which are then added in a fixed order.  The order depends only
// on `parts`, so results are bitwise reproducible.  Many warps per column keep each
// thread's chain of dependent loads short: the kernel is latency-bound, not byte-bound.
#include "internal.h"

#include <cuda_bf16.h>

namespace kron {
namespace {

__device__ __forceinline__ float to_f(float v) { return v; }
__device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }

constexpr int kWarps = 32;

// Sums over the row ranges of up to NC columns off[0..ncols): warp w adds ranges
// g = w, w+kWarps, ... into U independent accumulators per column (so U*ncols loads are
// in flight per thread); then the accumulators and the kWarps warp sums are added in a
// fixed order.
template <int U, int NC>
__device__ __forceinline__ void col_sums(const float *__restrict__ ws, int parts, size_t stride,
                                         const size_t *off, bool valid, int ncols,
                                         double (*red)[33], double *out) {
    const int lane = threadIdx.x, w = threadIdx.y;
    double acc[NC][U];
#pragma unroll
    for (int c = 0; c < NC; ++c)
#pragma unroll
        for (int u = 0; u < U; ++u) acc[c][u] = 0.0;
    if (valid) {
        for (int g = w; g < parts; g += kWarps * U) {
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int gg = g + kWarps * u;
                if (gg < parts) {
#pragma unroll
                    for (int c = 0; c < NC; ++c)
                        if (c < ncols) acc[c][u] += (double)ws[(size_t)gg * stride + off[c]];
                }
            }
        }
    }
#pragma unroll
    for (int c = 0; c < NC; ++c) {
        if (c >= ncols) break;
        double sum = 0.0;
#pragma unroll
        for (int u = 0; u < U; ++u) sum += acc[c][u];
        red[w][lane] = sum;
        __syncthreads();
        if (w == 0) {
            double tot = 0.0;
#pragma unroll
            for (int t = 0; t < kWarps; ++t) tot += red[t][lane];
            out[c] = tot;
        }
        __syncthreads();
    }
}

constexpr int kMaxRanksPerPass = 8;

template <typename TI>
__global__ void __launch_bounds__(32 * kWarps)
kron_reduce_kernel(const float *__restrict__ ws, int parts, size_t stride,
                   const TI *__restrict__ S, const TI *__restrict__ A, float *__restrict__ dS,
                   float *__restrict__ dA, float *__restrict__ dB, float *__restrict__ dbias,
                   Shape s, int blocks_dc, int blocks_db, double l1) {
    __shared__ double red[kWarps][33];
    const size_t pq = (size_t)s.p * s.q;
    const size_t n_dc = (size_t)s.r * pq, n_db = (size_t)s.r * s.m1 * s.m2;
    const size_t n_b = (size_t)s.q * s.m2;
    const int lane = threadIdx.x;
    int blk = blockIdx.x;
    if (blk < blocks_dc) {
        // dC for all ranks of columns (a,c) -> dA = dC (.) S, dS = sum_i dC_i (.) A_i
        const size_t col = (size_t)blk * 32 + lane;
        const bool v = col < pq;
        double ds = 0.0;
        for (int i0 = 0; i0 < s.r; i0 += kMaxRanksPerPass) {
            const int nr = s.r - i0 < kMaxRanksPerPass ? s.r - i0 : kMaxRanksPerPass;
            size_t off[kMaxRanksPerPass];
            double dc[kMaxRanksPerPass];
            for (int ii = 0; ii < kMaxRanksPerPass; ++ii) off[ii] = (size_t)(i0 + ii) * pq + col;
            col_sums<1, kMaxRanksPerPass>(ws, parts, stride, off, v, nr, red, dc);
            if (threadIdx.y == 0 && v) {
                for (int ii = 0; ii < nr; ++ii) {
                    const size_t e = (size_t)(i0 + ii) * pq + col;
                    dA[e] = (float)(dc[ii] * (double)to_f(S[col]));
                    ds += dc[ii] * (double)to_f(A[e]);
                }
            }
        }
        if (threadIdx.y == 0 && v) {
            if (l1 != 0.0) ds += l1 * sign_of(to_f(S[col]));   // d(l1 * sum|S|)/dS
            dS[col] = (float)ds;
        }
        return;
    }
    blk -= blocks_dc;
    if (blk < blocks_db) {
        const size_t col = (size_t)blk * 32 + lane;
        const size_t off = n_dc + col;
        const bool v = col < n_db;
        double out;
        col_sums<4, 1>(ws, parts, stride, &off, v, 1, red, &out);
        if (threadIdx.y == 0 && v) dB[col] = (float)out;
        return;
    }
    blk -= blocks_db;
    const size_t col = (size_t)blk * 32 + lane;
    const size_t off = n_dc + n_db + col;
    const bool v = col < n_b;
    double out;
    col_sums<4, 1>(ws, parts, stride, &off, v, 1, red, &out);
    if (threadIdx.y == 0 && v) dbias[col] = (float)out;
}

}  // namespace

cudaError_t reduce_partials(const float *ws, int parts, const void *S, const void *A,
                            bool is_bf16, float *dS, float *dA, float *dB, float *dbias,
                            const Shape &s, double l1, cudaStream_t st) {
    const size_t pq = (size_t)s.p * s.q;
    const int blocks_dc = (int)((pq + 31) / 32);
    const int blocks_db = (int)(((size_t)s.r * s.m1 * s.m2 + 31) / 32);
    const int blocks_b = dbias ? (int)(((size_t)s.q * s.m2 + 31) / 32) : 0;
    const size_t stride = partial_stride(s);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(blocks_dc + blocks_db + blocks_b));
    cfg.blockDim = dim3(32, kWarps);
    cfg.stream = st;
    if (is_bf16)
        return cudaLaunchKernelEx(&cfg, kron_reduce_kernel<__nv_bfloat16>, ws, parts, stride,
                                  (const __nv_bfloat16 *)S, (const __nv_bfloat16 *)A, dS, dA, dB,
                                  dbias, s, blocks_dc, blocks_db, l1);
    return cudaLaunchKernelEx(&cfg, kron_reduce_kernel<float>, ws, parts, stride, (const float *)S,
                              (const float *)A, dS, dA, dB, dbias, s, blocks_dc, blocks_db, l1);
}

}  // namespace kron
