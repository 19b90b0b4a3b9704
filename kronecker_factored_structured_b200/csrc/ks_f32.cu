// ks_f32.cu -- the Kronecker-sparse factor of include/ks_linear.h on the CUDA cores (exact
// FP32).  Pattern (a, b, c, d): y = x K + bias with supp K = kron(I_a, kron(1_{b x c}, I_d))
// (page "Fast Inference with Kronecker-Sparse Matrices", abstract), i.e. per row
//
//     y[n][(al*c + ga)*d + de] = sum_be x[n][(al*b + be)*d + de] * w[al][de][be][ga] + bias,
//
// a*d independent b x c products whose operands sit at stride d inside each row.
//
// Output-stationary, as the page's abstract describes its kernel: a CTA owns a tile of y
// (rows n0.., one block al, deltas de0.., columns ga0..), stages the strided input slices
// it needs in shared memory (the gather happens on chip: x is read once per column tile and
// y written once, no permuted copy of x or y ever reaches HBM) and runs the whole
// contraction for its tile.  The same kernel computes dX = dY K^T with the roles of b and c
// swapped and w read transposed.  dw is a split-N reduction: each CTA sums x^T dY over one
// contiguous row range for one tile of (al, de, be, ga) and writes a partial; a second
// kernel adds the partials in a fixed order (bitwise reproducible; the row split depends on
// the sizes only).  dbias rides along in the dw kernel.
//
// Thread work: a thread owns one delta, kR contiguous rows (dw: be values) and kC columns
// GC apart (GC = column groups of the tile), so that for each of its columns the lanes of a
// warp, which differ first in delta and then in column group, store consecutive addresses.
// The delta stride of each shared array is padded so that those lanes hit distinct banks.
#include "../../include/ks_linear.h"
#include "internal.h"

#include <stdarg.h>
#include <stdio.h>

namespace kron {
kron_status_t report_failure(kron_status_t st, const char *msg);
}

namespace {

constexpr int kThreads = 256;
constexpr int kR = 8;                   // rows (dw: be values) per thread, contiguous
constexpr int kC = 4;                   // columns per thread, GC apart
constexpr int kSmemTile = 32 * 1024;    // bytes of staged operands per CTA
constexpr int64_t kPartTarget = 4 * 148;  // CTAs the backward's row split aims for
constexpr int64_t kMaxWidth = 1 << 24;    // a*b*d and a*c*d

struct KsTile {
    int TD;    // deltas per CTA (d when d <= 8, else 8)
    int GC;    // column groups: TC = GC * kC columns per tile
    int GR;    // row groups: TM = GR * kR rows (forward) or be values (dw) per tile
    int KB;    // reduction chunk staged at once (forward: be or ga values; dw: rows)
    int KG;    // dw: thread groups that split each chunk's rows (forward: 1)
    int padw;  // padding of the column array's delta stride
};

// Largest power of two gr with 2 gr^2 <= maxg, and gc = maxg / gr: a tile with about as
// many columns as rows (TC = 4 gc ~ TM = 8 gr).
void balanced(int maxg, int *gr, int *gc) {
    int r = 1;
    while (2 * (2 * r) * (2 * r) <= maxg) r *= 2;
    *gr = r;
    *gc = maxg / r;
}

int tile_deltas(int d) { return d <= 8 ? d : 8; }
int pad_for(int td) { return (td & (td - 1)) == 0 ? (32 / td) % 32 : 1; }
int cdiv(int64_t x, int64_t y) { return (int)((x + y - 1) / y); }

// Forward / dX tile: kin = contraction length, kout = output block length.
KsTile fwd_tile(int kin, int kout, int d) {
    KsTile t{};
    t.TD = tile_deltas(d);
    t.padw = pad_for(t.TD);
    t.KG = 1;
    const int maxg = kThreads / t.TD;
    int gr, gc;
    balanced(maxg, &gr, &gc);
    const int need_c = cdiv(kout, kC);
    if (gc > need_c) {
        gc = need_c;
        gr = maxg / gc < 64 ? maxg / gc : 64;
    }
    t.GR = gr;
    t.GC = gc;
    const int step = t.TD * (gr * kR + 4 + gc * kC + t.padw) * 4;
    const int kb = kSmemTile / step;
    t.KB = kb < 1 ? 1 : (kb > kin ? kin : kb);
    return t;
}

KsTile dw_tile(int b, int c, int d) {
    KsTile t{};
    t.TD = tile_deltas(d);
    t.padw = pad_for(t.TD);
    const int maxg = kThreads / t.TD;
    int gr, gc;
    balanced(maxg, &gr, &gc);
    const int need_b = cdiv(b, kR), need_c = cdiv(c, kC);
    if (gc > need_c) gc = need_c;
    gr = maxg / gc < need_b ? maxg / gc : need_b;
    gc = maxg / gr < need_c ? maxg / gr : need_c;
    t.GR = gr;
    t.GC = gc;
    t.KG = maxg / (gr * gc);
    const int step = t.TD * (gr * kR + 4 + gc * kC + t.padw) * 4;
    const int kb = kSmemTile / step;
    t.KB = kb < 1 ? 1 : (kb > 256 ? 256 : kb);
    return t;
}

size_t tile_smem(const KsTile &t) {
    const size_t stage =
        (size_t)t.KB * t.TD * ((size_t)t.GR * kR + 4 + (size_t)t.GC * kC + t.padw) * 4;
    const size_t red = t.KG > 1 ? (size_t)kThreads * (kR * kC + kC) * 4 : 0;
    return stage > red ? stage : red;
}

struct DwPlan {
    KsTile t;
    int64_t tiles_per_part, parts, rows_per_part;
    size_t part_stride;  // floats
};

DwPlan dw_plan(int64_t N, int a, int b, int c, int d) {
    DwPlan P;
    P.t = dw_tile(b, c, d);
    P.tiles_per_part = (int64_t)a * cdiv(d, P.t.TD) * cdiv(b, (int64_t)P.t.GR * kR) *
                       cdiv(c, (int64_t)P.t.GC * kC);
    int64_t parts = 0;
    if (N > 0) {
        parts = (kPartTarget + P.tiles_per_part - 1) / P.tiles_per_part;
        const int64_t chunks = (N + P.t.KB - 1) / P.t.KB;
        if (parts > chunks) parts = chunks;
        if (parts < 1) parts = 1;
    }
    P.parts = parts;
    P.rows_per_part = parts ? (N + parts - 1) / parts : 0;
    const size_t nw = (size_t)a * b * c * d, nb = (size_t)a * c * d;
    P.part_stride = (nw + nb + 63) & ~(size_t)63;
    return P;
}

// y (or dX) tiles.  TR = false: in = x [N][a*kin*d], w [a][d][kin][kout].  TR = true (dX):
// in = dY [N][a*kin*d], w [a][d][kout][kin] read transposed.
template <bool TR>
__global__ void __launch_bounds__(kThreads)
ks_fwd_kernel(const float *__restrict__ in, const float *__restrict__ w,
              const float *__restrict__ bias, float *__restrict__ out, int64_t N, int a, int kin,
              int kout, int d, KsTile t, int64_t tiles) {
    extern __shared__ __align__(16) float smem[];
    const int TD = t.TD, GC = t.GC, GR = t.GR, TM = GR * kR, TC = GC * kC;
    const int SX = TM + 4, SW = TC + t.padw;
    float *xs = smem;                             // [KB][TD][SX]: input, rows contiguous
    float *ws = smem + (size_t)t.KB * TD * SX;    // [KB][TD][SW]: values, columns contiguous
    const int tid = threadIdx.x;
    const bool active = tid < TD * GC * GR;
    const int dl = tid % TD, cg = (tid / TD) % GC, rg = tid / (TD * GC);
    const int64_t in_w = (int64_t)a * kin * d, out_w = (int64_t)a * kout * d;
    const int nj = (kout + TC - 1) / TC, nd = (d + TD - 1) / TD;

    for (int64_t tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
        const int jt = (int)(tile % nj);
        int64_t rest = tile / nj;
        const int dt = (int)(rest % nd);
        rest /= nd;
        const int al = (int)(rest % a);
        const int64_t n0 = (rest / a) * TM;
        const int de0 = dt * TD, j0 = jt * TC;

        float acc[kR][kC];
#pragma unroll
        for (int i = 0; i < kR; ++i)
#pragma unroll
            for (int jj = 0; jj < kC; ++jj) acc[i][jj] = 0.f;

        for (int k0 = 0; k0 < kin; k0 += t.KB) {
            const int kb = min(t.KB, kin - k0);
            const int span = kb * TD;  // (k, delta) pairs of one row, contiguous when TD == d
            for (int e = tid; e < span * TM; e += kThreads) {
                const int u = e % span, r = e / span;
                const int de = de0 + u % TD;
                const int64_t n = n0 + r;
                float v = 0.f;
                if (n < N && de < d)
                    v = in[n * in_w + ((int64_t)al * kin + k0 + u / TD) * d + de];
                xs[u * SX + r] = v;
            }
            for (int e = tid; e < span * TC; e += kThreads) {
                int kk, dd, jl;
                if (TR) {
                    kk = e % kb;
                    const int q = e / kb;
                    jl = q % TC;
                    dd = q / TC;
                } else {
                    jl = e % TC;
                    const int q = e / TC;
                    kk = q % kb;
                    dd = q / kb;
                }
                const int de = de0 + dd, j = j0 + jl;
                float v = 0.f;
                if (de < d && j < kout) {
                    const int64_t blk = (int64_t)al * d + de;
                    v = TR ? w[(blk * kout + j) * kin + k0 + kk] : w[(blk * kin + k0 + kk) * kout + j];
                }
                ws[(kk * TD + dd) * SW + jl] = v;
            }
            __syncthreads();
            if (active) {
                for (int kk = 0; kk < kb; ++kk) {
                    const float *xr = xs + (kk * TD + dl) * SX + rg * kR;
                    const float4 x0 = *reinterpret_cast<const float4 *>(xr);
                    const float4 x1 = *reinterpret_cast<const float4 *>(xr + 4);
                    const float xv[kR] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
                    const float *wr = ws + (kk * TD + dl) * SW + cg;
                    float wv[kC];
#pragma unroll
                    for (int jj = 0; jj < kC; ++jj) wv[jj] = wr[jj * GC];
#pragma unroll
                    for (int i = 0; i < kR; ++i)
#pragma unroll
                        for (int jj = 0; jj < kC; ++jj) acc[i][jj] = fmaf(xv[i], wv[jj], acc[i][jj]);
                }
            }
            __syncthreads();
        }

        if (active && de0 + dl < d) {
            const int de = de0 + dl;
#pragma unroll
            for (int jj = 0; jj < kC; ++jj) {
                const int j = j0 + cg + jj * GC;
                if (j >= kout) continue;
                const int64_t col = ((int64_t)al * kout + j) * d + de;
                const float bv = bias ? bias[col] : 0.f;
#pragma unroll
                for (int i = 0; i < kR; ++i) {
                    const int64_t n = n0 + rg * kR + i;
                    if (n < N) out[n * out_w + col] = acc[i][jj] + bv;
                }
            }
        }
    }
}

// Partial sums of dw (and dbias) over one contiguous row range per CTA.  Grid = parts x
// (al, delta tile, be tile, ga tile); part p writes part[p][0 .. a*b*c*d) (dw layout) and,
// from the CTAs of the first be tile, part[p][a*b*c*d + (al*c + ga)*d + de] (dbias).
__global__ void __launch_bounds__(kThreads)
ks_dw_kernel(const float *__restrict__ x, const float *__restrict__ g, float *__restrict__ part,
             int64_t N, int a, int b, int c, int d, KsTile t, int64_t rows_per_part,
             size_t part_stride) {
    extern __shared__ __align__(16) float smem[];
    const int TD = t.TD, GC = t.GC, GR = t.GR, KG = t.KG, TB = GR * kR, TC = GC * kC;
    const int SX = TB + 4, SW = TC + t.padw;
    float *xs = smem;                             // [KB rows][TD][SX]: be contiguous
    float *gs = smem + (size_t)t.KB * TD * SX;    // [KB rows][TD][SW]: ga contiguous
    const int tid = threadIdx.x;
    const int items = TD * GC * GR;
    const bool active = tid < items * KG;
    const int it = tid % items, kg = tid / items;
    const int dl = it % TD, cg = (it / TD) % GC, bg = it / (TD * GC);

    const int nc = (c + TC - 1) / TC, nb = (b + TB - 1) / TB, nd = (d + TD - 1) / TD;
    int64_t rest = blockIdx.x;
    const int ct = (int)(rest % nc);
    rest /= nc;
    const int bt = (int)(rest % nb);
    rest /= nb;
    const int dt = (int)(rest % nd);
    rest /= nd;
    const int al = (int)(rest % a);
    const int64_t p = rest / a;
    const int64_t r0 = p * rows_per_part;
    const int64_t r1 = r0 + rows_per_part < N ? r0 + rows_per_part : N;
    const int de0 = dt * TD, be0 = bt * TB, ga0 = ct * TC;
    const int64_t in_w = (int64_t)a * b * d, out_w = (int64_t)a * c * d;
    const bool with_bias = bt == 0 && bg == 0;

    float acc[kR][kC], bacc[kC];
#pragma unroll
    for (int jj = 0; jj < kC; ++jj) {
        bacc[jj] = 0.f;
#pragma unroll
        for (int i = 0; i < kR; ++i) acc[i][jj] = 0.f;
    }

    for (int64_t n0 = r0; n0 < r1; n0 += t.KB) {
        const int kb = (int)(r1 - n0 < t.KB ? r1 - n0 : t.KB);
        const int spx = TB * TD, spg = TC * TD;
        for (int e = tid; e < kb * spx; e += kThreads) {
            const int u = e % spx, kr = e / spx;
            const int bl = u / TD, dd = u % TD;
            const int be = be0 + bl, de = de0 + dd;
            float v = 0.f;
            if (be < b && de < d) v = x[(n0 + kr) * in_w + ((int64_t)al * b + be) * d + de];
            xs[(kr * TD + dd) * SX + bl] = v;
        }
        for (int e = tid; e < kb * spg; e += kThreads) {
            const int u = e % spg, kr = e / spg;
            const int gl = u / TD, dd = u % TD;
            const int ga = ga0 + gl, de = de0 + dd;
            float v = 0.f;
            if (ga < c && de < d) v = g[(n0 + kr) * out_w + ((int64_t)al * c + ga) * d + de];
            gs[(kr * TD + dd) * SW + gl] = v;
        }
        __syncthreads();
        if (active) {
            for (int kr = kg; kr < kb; kr += KG) {
                const float *xr = xs + (kr * TD + dl) * SX + bg * kR;
                const float4 x0 = *reinterpret_cast<const float4 *>(xr);
                const float4 x1 = *reinterpret_cast<const float4 *>(xr + 4);
                const float xv[kR] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
                const float *gr = gs + (kr * TD + dl) * SW + cg;
                float gv[kC];
#pragma unroll
                for (int jj = 0; jj < kC; ++jj) gv[jj] = gr[jj * GC];
#pragma unroll
                for (int i = 0; i < kR; ++i)
#pragma unroll
                    for (int jj = 0; jj < kC; ++jj) acc[i][jj] = fmaf(xv[i], gv[jj], acc[i][jj]);
                if (with_bias) {
#pragma unroll
                    for (int jj = 0; jj < kC; ++jj) bacc[jj] += gv[jj];
                }
            }
        }
        __syncthreads();
    }

    // The KG row groups' sums, added in group order through shared memory.
    constexpr int RS = kR * kC + kC;
    if (KG > 1) {
        float *red = smem;  // [KG][items][RS]; every read of xs / gs ended at the last sync
        if (active) {
            float *o = red + ((size_t)kg * items + it) * RS;
#pragma unroll
            for (int i = 0; i < kR; ++i)
#pragma unroll
                for (int jj = 0; jj < kC; ++jj) o[i * kC + jj] = acc[i][jj];
#pragma unroll
            for (int jj = 0; jj < kC; ++jj) o[kR * kC + jj] = bacc[jj];
        }
        __syncthreads();
        if (tid < items) {
#pragma unroll
            for (int i = 0; i < kR; ++i)
#pragma unroll
                for (int jj = 0; jj < kC; ++jj) {
                    float s = 0.f;
                    for (int q = 0; q < KG; ++q) s += red[((size_t)q * items + it) * RS + i * kC + jj];
                    acc[i][jj] = s;
                }
#pragma unroll
            for (int jj = 0; jj < kC; ++jj) {
                float s = 0.f;
                for (int q = 0; q < KG; ++q) s += red[((size_t)q * items + it) * RS + kR * kC + jj];
                bacc[jj] = s;
            }
        }
    }

    if (tid < items && de0 + dl < d) {
        const int de = de0 + dl;
        float *pw = part + (size_t)p * part_stride;
#pragma unroll
        for (int i = 0; i < kR; ++i) {
            const int be = be0 + bg * kR + i;
            if (be >= b) continue;
#pragma unroll
            for (int jj = 0; jj < kC; ++jj) {
                const int ga = ga0 + cg + jj * GC;
                if (ga < c) pw[(((int64_t)al * d + de) * b + be) * c + ga] = acc[i][jj];
            }
        }
        if (with_bias) {
            const size_t nw = (size_t)a * b * c * d;
#pragma unroll
            for (int jj = 0; jj < kC; ++jj) {
                const int ga = ga0 + cg + jj * GC;
                if (ga < c) pw[nw + ((size_t)al * c + ga) * d + de] = bacc[jj];
            }
        }
    }
}

// dw[e] = sum_{p < parts} part[p][e] (and dbias likewise), in part order, in double.
__global__ void ks_reduce_kernel(const float *__restrict__ part, int64_t parts, size_t stride,
                                 size_t nw, size_t nb, float *__restrict__ dw,
                                 float *__restrict__ dbias) {
    const size_t total = nw + (dbias ? nb : 0);
    for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
         e += (size_t)gridDim.x * blockDim.x) {
        double s = 0.0;
        for (int64_t p = 0; p < parts; ++p) s += (double)part[(size_t)p * stride + e];
        if (e < nw)
            dw[e] = (float)s;
        else
            dbias[e - nw] = (float)s;
    }
}

kron_status_t ks_fail(kron_status_t st, const char *fmt, ...) __attribute__((format(printf, 2, 3)));
kron_status_t ks_fail(kron_status_t st, const char *fmt, ...) {
    char msg[256];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(msg, sizeof(msg), fmt, ap);
    va_end(ap);
    return kron::report_failure(st, msg);
}

kron_status_t ks_check(int64_t N, int a, int b, int c, int d, kron_dtype_t dtype,
                       unsigned flags) {
    if (dtype != KRON_F32 && dtype != KRON_TF32 && dtype != KRON_BF16)
        return ks_fail(KRON_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
    if (flags)
        return ks_fail(KRON_ERR_INVALID_ARG, "unknown flag bits 0x%x", flags);
    if (N < 0 || a < 1 || b < 1 || c < 1 || d < 1)
        return ks_fail(KRON_ERR_INVALID_ARG,
                       "sizes must be N >= 0 and a, b, c, d >= 1 (got N=%lld a=%d b=%d c=%d d=%d)",
                       (long long)N, a, b, c, d);
    if ((int64_t)a * b * d > kMaxWidth || (int64_t)a * c * d > kMaxWidth ||
        N > ((int64_t)1 << 40))
        return ks_fail(KRON_ERR_INVALID_ARG, "sizes out of range");
    if (dtype != KRON_F32)
        return ks_fail(KRON_ERR_UNSUPPORTED, "the Kronecker-sparse factor runs on KRON_F32 only");
    return KRON_OK;
}

bool a4(const void *p) { return ((uintptr_t)p & 3u) == 0; }

cudaError_t launch_fwd(bool tr, const float *in, const float *w, const float *bias, float *out,
                       int64_t N, int a, int kin, int kout, int d, cudaStream_t st) {
    const KsTile t = fwd_tile(kin, kout, d);
    const int64_t tiles = (N + (int64_t)t.GR * kR - 1) / ((int64_t)t.GR * kR) * a *
                          cdiv(d, t.TD) * cdiv(kout, (int64_t)t.GC * kC);
    const unsigned grid = (unsigned)(tiles < (1 << 30) ? tiles : (1 << 30));
    const size_t smem = tile_smem(t);
    if (tr)
        ks_fwd_kernel<true><<<grid, kThreads, smem, st>>>(in, w, nullptr, out, N, a, kin, kout, d,
                                                          t, tiles);
    else
        ks_fwd_kernel<false><<<grid, kThreads, smem, st>>>(in, w, bias, out, N, a, kin, kout, d,
                                                           t, tiles);
    return cudaGetLastError();
}

}  // namespace

extern "C" {

size_t ks_linear_workspace_size(int64_t N, int a, int b, int c, int d, kron_dtype_t dtype) {
    if (N < 0 || a < 1 || b < 1 || c < 1 || d < 1 || dtype != KRON_F32) return 0;
    if ((int64_t)a * b * d > kMaxWidth || (int64_t)a * c * d > kMaxWidth ||
        N > ((int64_t)1 << 40))
        return 0;
    const DwPlan P = dw_plan(N, a, b, c, d);
    const size_t bytes = (size_t)P.parts * P.part_stride * 4;
    return bytes < 256 ? 256 : bytes;
}

kron_status_t ks_linear_forward(const void *x, const void *w, const void *bias, void *y,
                                int64_t N, int a, int b, int c, int d, kron_dtype_t dtype,
                                unsigned flags, void *stream) {
    kron_status_t st = ks_check(N, a, b, c, d, dtype, flags);
    if (st != KRON_OK) return st;
    if (!w || (N > 0 && (!x || !y)))
        return ks_fail(KRON_ERR_INVALID_ARG, "w, and x and y when N > 0, must be non-null");
    if (!a4(x) || !a4(w) || !a4(bias) || !a4(y))
        return ks_fail(KRON_ERR_ALIGNMENT, "tensors must be 4-byte aligned");
    if (N == 0) return KRON_OK;
    const cudaError_t e = launch_fwd(false, (const float *)x, (const float *)w,
                                     (const float *)bias, (float *)y, N, a, b, c, d,
                                     (cudaStream_t)stream);
    if (e != cudaSuccess) return ks_fail(KRON_ERR_CUDA, "KS forward launch: %s", cudaGetErrorString(e));
    return KRON_OK;
}

kron_status_t ks_linear_backward(const void *x, const void *w, const void *dY, void *dX, void *dw,
                                 void *dbias, int64_t N, int a, int b, int c, int d,
                                 kron_dtype_t dtype, unsigned flags, void *workspace,
                                 size_t workspace_bytes, void *stream) {
    kron_status_t st = ks_check(N, a, b, c, d, dtype, flags);
    if (st != KRON_OK) return st;
    if (!w || !dw || (N > 0 && (!x || !dY)))
        return ks_fail(KRON_ERR_INVALID_ARG, "w and dw, and x and dY when N > 0, must be non-null");
    if (!a4(x) || !a4(w) || !a4(dY) || !a4(dX) || !a4(dw) || !a4(dbias))
        return ks_fail(KRON_ERR_ALIGNMENT, "tensors must be 4-byte aligned");
    const size_t need = ks_linear_workspace_size(N, a, b, c, d, dtype);
    if (!workspace || workspace_bytes < need)
        return ks_fail(KRON_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need,
                       workspace ? workspace_bytes : (size_t)0);
    if ((uintptr_t)workspace & 255u)
        return ks_fail(KRON_ERR_ALIGNMENT, "workspace must be 256-byte aligned");
    cudaStream_t cs = (cudaStream_t)stream;
    const size_t nw = (size_t)a * b * c * d, nb = (size_t)a * c * d;
    cudaError_t e = cudaSuccess;
    if (N == 0) {
        e = cudaMemsetAsync(dw, 0, nw * 4, cs);
        if (e == cudaSuccess && dbias) e = cudaMemsetAsync(dbias, 0, nb * 4, cs);
        if (e != cudaSuccess) return ks_fail(KRON_ERR_CUDA, "KS zero fill: %s", cudaGetErrorString(e));
        return KRON_OK;
    }
    if (dX) {
        e = launch_fwd(true, (const float *)dY, (const float *)w, nullptr, (float *)dX, N, a, c, b,
                       d, cs);
        if (e != cudaSuccess) return ks_fail(KRON_ERR_CUDA, "KS dX launch: %s", cudaGetErrorString(e));
    }
    const DwPlan P = dw_plan(N, a, b, c, d);
    const int64_t grid = P.parts * P.tiles_per_part;
    if (grid > 0x7fffffff)
        return ks_fail(KRON_ERR_UNSUPPORTED, "too many dw tiles (%lld)", (long long)grid);
    float *part = static_cast<float *>(workspace);
    ks_dw_kernel<<<(unsigned)grid, kThreads, tile_smem(P.t), cs>>>(
        (const float *)x, (const float *)dY, part, N, a, b, c, d, P.t, P.rows_per_part,
        P.part_stride);
    e = cudaGetLastError();
    if (e != cudaSuccess) return ks_fail(KRON_ERR_CUDA, "KS dw launch: %s", cudaGetErrorString(e));
    const size_t total = nw + (dbias ? nb : 0);
    const size_t blocks = (total + 255) / 256;
    ks_reduce_kernel<<<(unsigned)(blocks < 4096 ? blocks : 4096), 256, 0, cs>>>(
        part, P.parts, P.part_stride, nw, nb, (float *)dw, (float *)dbias);
    e = cudaGetLastError();
    if (e != cudaSuccess) return ks_fail(KRON_ERR_CUDA, "KS reduce launch: %s", cudaGetErrorString(e));
    return KRON_OK;
}

}  // extern "C"
