// reduce.cu -- deterministic reduction of the backward's row-range partials and the
// factor-gradient epilogue:
//   dC_i = sum over row ranges of the partial dC_i   (fixed order)
//   dA_i = dC_i (.) S,   dS = sum_i dC_i (.) A_i,   dB_i and dbias likewise summed.
// (dA_i and dS follow from C_i = S (.) A_i by the product rule; W = sum_i kron(C_i, B_i)
// as on the page "kronecker-layer-benchmark", section "1. Build W, then multiply".)
//
// Workspace layout per range g: ws[g*stride + ...] = [dC: r*p*q][dB: r*m1*m2][dbias: q*m2].
// Each block owns 32 consecutive output columns; its 8 warps sum ranges g = w, w+8, ...
// in double, then warp 0 adds the 8 warp sums in order w = 0..7.  The order depends
// only on `parts`, so results are bitwise reproducible.
#include "internal.h"

#include <cuda_bf16.h>

namespace kron {
namespace {

__device__ __forceinline__ float to_f(float v) { return v; }
__device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }

__device__ __forceinline__ double block_sum(const float *__restrict__ ws, int parts,
                                            size_t stride, size_t off, bool valid,
                                            double (*red)[33]) {
    const int lane = threadIdx.x, w = threadIdx.y;
    double acc = 0.0;
    if (valid)
        for (int g = w; g < parts; g += 8) acc += (double)ws[(size_t)g * stride + off];
    red[w][lane] = acc;
    __syncthreads();
    double tot = 0.0;
    if (w == 0)
#pragma unroll
        for (int t = 0; t < 8; ++t) tot += red[t][lane];
    __syncthreads();
    return tot;
}

template <typename TI>
__global__ void __launch_bounds__(256)
kron_reduce_kernel(const float *__restrict__ ws, int parts, size_t stride,
                   const TI *__restrict__ S, const TI *__restrict__ A, float *__restrict__ dS,
                   float *__restrict__ dA, float *__restrict__ dB, float *__restrict__ dbias,
                   Shape s, int blocks_dc, int blocks_db) {
    __shared__ double red[8][33];
    const size_t pq = (size_t)s.p * s.q;
    const size_t n_dc = (size_t)s.r * pq, n_db = (size_t)s.r * s.m1 * s.m2;
    const size_t n_b = (size_t)s.q * s.m2;
    const int lane = threadIdx.x;
    int blk = blockIdx.x;
    if (blk < blocks_dc) {
        const size_t col = (size_t)blk * 32 + lane;
        const bool valid = col < pq;
        double ds = 0.0;
        for (int i = 0; i < s.r; ++i) {
            const double dc = block_sum(ws, parts, stride, (size_t)i * pq + col, valid, red);
            if (threadIdx.y == 0 && valid) {
                dA[(size_t)i * pq + col] = (float)(dc * (double)to_f(S[col]));
                ds += dc * (double)to_f(A[(size_t)i * pq + col]);
            }
        }
        if (threadIdx.y == 0 && valid) dS[col] = (float)ds;
        return;
    }
    blk -= blocks_dc;
    if (blk < blocks_db) {
        const size_t col = (size_t)blk * 32 + lane;
        const bool valid = col < n_db;
        const double v = block_sum(ws, parts, stride, n_dc + col, valid, red);
        if (threadIdx.y == 0 && valid) dB[col] = (float)v;
        return;
    }
    blk -= blocks_db;
    const size_t col = (size_t)blk * 32 + lane;
    const bool valid = col < n_b;
    const double v = block_sum(ws, parts, stride, n_dc + n_db + col, valid, red);
    if (threadIdx.y == 0 && valid) dbias[col] = (float)v;
}

}  // namespace

cudaError_t reduce_partials(const float *ws, int parts, const void *S, const void *A,
                            bool is_bf16, float *dS, float *dA, float *dB, float *dbias,
                            const Shape &s, cudaStream_t st) {
    const size_t pq = (size_t)s.p * s.q;
    const int blocks_dc = (int)((pq + 31) / 32);
    const int blocks_db = (int)(((size_t)s.r * s.m1 * s.m2 + 31) / 32);
    const int blocks_b = dbias ? (int)(((size_t)s.q * s.m2 + 31) / 32) : 0;
    const dim3 block(32, 8);
    const unsigned grid = (unsigned)(blocks_dc + blocks_db + blocks_b);
    const size_t stride = partial_stride(s);
    if (is_bf16)
        kron_reduce_kernel<__nv_bfloat16><<<grid, block, 0, st>>>(
            ws, parts, stride, (const __nv_bfloat16 *)S, (const __nv_bfloat16 *)A, dS, dA, dB,
            dbias, s, blocks_dc, blocks_db);
    else
        kron_reduce_kernel<float><<<grid, block, 0, st>>>(ws, parts, stride, (const float *)S,
                                                          (const float *)A, dS, dA, dB, dbias,
                                                          s, blocks_dc, blocks_db);
    return cudaGetLastError();
}

}  // namespace kron
