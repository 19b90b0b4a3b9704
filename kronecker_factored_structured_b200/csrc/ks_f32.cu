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
// swapped, from a copy of the blocks transposed once per call into the workspace.  dw is a
// split-N reduction: each CTA sums x^T dY over one contiguous row range for one tile of
// (al, de, be, ga) and writes a partial; a second kernel adds the partials in a fixed order
// (bitwise reproducible; the row split depends on the sizes only).  dbias rides along in the
// dw kernel.  Blocks of at most 4 x 4 (butterfly factors) skip the tiles: a register-resident
// stream with one thread per (al, de) runs the forward, dX and the dw partials.
//
// Thread work: a thread owns one delta, kR contiguous rows (dw: be values) and kC contiguous
// columns, read from shared memory as float4 each step.  The lanes of a warp differ first in
// delta (consecutive addresses in y) and then in column group; the delta stride of each
// shared array is padded so that those lanes hit distinct banks.
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
constexpr int kC = 4;                   // columns per thread, contiguous
constexpr int kSmemTile = 32 * 1024;    // bytes of staged operands per CTA
constexpr int64_t kPartTarget = 4 * 148;  // CTAs the backward's row split aims for (a
                                          // constant, not the device's SM count: the split,
                                          // and so the summation order, depend on sizes only)
constexpr int64_t kMaxWidth = 1 << 24;    // a*b*d and a*c*d

struct KsTile {
    int TD;    // deltas per CTA: 1, 2, 4 or 8 (the power of two >= d, at most 8)
    int GC;    // column groups: TC = GC * kC columns per tile
    int GR;    // row groups: TM = GR * kR rows (forward) or be values (dw) per tile
    int KB;    // reduction chunk staged at once (forward: be values; dw: rows)
    int KG;    // dw: thread groups that split each chunk's rows (forward: 1)
    int padw;  // padding of the column array's delta stride
    int vx;    // 1: the row slices are staged with 16-byte loads (alignment allows it)
    int vw;    // 1: the values (forward) / dY slices (dw) likewise
};

// Largest power of two gr with 2 gr^2 <= maxg, and gc = maxg / gr: a tile with about as
// many columns as rows (TC = 4 gc ~ TM = 8 gr).
void balanced(int maxg, int *gr, int *gc) {
    int r = 1;
    while (2 * (2 * r) * (2 * r) <= maxg) r *= 2;
    *gr = r;
    *gc = maxg / r;
}

int tile_deltas(int d) { return d >= 8 ? 8 : (d > 4 ? 8 : (d > 2 ? 4 : d)); }
int pad_for(int td) { return (32 / td) % 32; }
int cdiv(int64_t x, int64_t y) { return (int)((x + y - 1) / y); }
bool a16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

// Whether one CTA's slice of a row -- elements (k, delta) for k in a chunk starting at a
// multiple of `kstep` and delta in a tile of TD -- can move as aligned float4 (all four
// valid or all four outside the matrix): runs of TD (TD < d) need d % 4 == 0; one
// contiguous run (TD == d) needs its start and length to be multiples of 4.
bool slice_vec(int kdim, int kstep, int d, int td) {
    if (td < d) return d % 4 == 0;
    if (td != d) return false;
    return ((int64_t)kdim * d) % 4 == 0 && ((int64_t)kstep * d) % 4 == 0;
}

// Forward / dX tile: kin = contraction length, kout = output block length.
KsTile fwd_tile(int kin, int kout, int d, const void *in, const void *w) {
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
        if (gr >= 4) gr &= ~3;
    }
    t.GR = gr;
    t.GC = gc;
    const int step = t.TD * (gr * kR + 4 + gc * kC + t.padw) * 4;
    int kb = kSmemTile / step;
    kb = kb < 1 ? 1 : (kb > 256 ? 256 : kb);
    if (kb < kin && kb >= 4) kb &= ~3;  // chunk starts stay float4-aligned when d is odd
    t.KB = kb > kin ? kin : kb;
    t.vx = a16(in) && slice_vec(kin, t.KB, d, t.TD);
    t.vw = a16(w) && kout % 4 == 0;
    return t;
}

KsTile dw_tile(int b, int c, int d, const void *x, const void *g) {
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
    t.vx = a16(x) && slice_vec(b, gr * kR, d, t.TD);
    t.vw = a16(g) && slice_vec(c, gc * kC, d, t.TD);
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

DwPlan dw_plan(int64_t N, int a, int b, int c, int d, const void *x, const void *g) {
    DwPlan P;
    P.t = dw_tile(b, c, d, x, g);
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

// Small blocks: row ranges so that about kSmallTarget threads run (sizes only).
constexpr int64_t kSmallTarget = 148 * 1024;
constexpr int kSmallMax = 4;  // largest b and c of the small-block stream
bool small_blocks(int kin, int kout) { return kin <= kSmallMax && kout <= kSmallMax; }
int64_t small_ranges(int64_t N, int a, int d) {
    if (N <= 0) return 0;
    const int64_t threads = (int64_t)cdiv((int64_t)a * d, 128) * 128;
    int64_t r = (kSmallTarget + threads - 1) / threads;
    return r < 1 ? 1 : (r > N ? N : r);
}

// Staging of row slices into shared memory.  Element (row rr, slice position u), with
// u = k*TD + dd for k < kn and dd < TD, comes from
//     src[(row0 + rr) * row_w + (kbase + k) * d + de0 + dd]
// and is zero outside the matrix (row0 + rr >= nmax, kbase + k >= kdim or de0 + dd >= d).
// With vec the slice moves as aligned float4 (4 consecutive u; the host checks that all
// four are inside or all outside).  No division depends on the element: each thread's
// assignment is fixed for the launch.
//
// stage_cols writes dst[u * S + rr] (the forward's input: rows contiguous per position).
// Lane pairs take 8 consecutive positions of one row (a whole 32-byte sector), the 16 pairs
// of a warp 16 consecutive rows; with S = 4 (mod 32) the stores hit 32 distinct banks.
template <int TD>
__device__ __forceinline__ void stage_cols(float *__restrict__ dst, int S,
                                           const float *__restrict__ src, int64_t row_w,
                                           int64_t row0, int64_t nmax, int nrows, int kbase,
                                           int kn, int kdim, int d, int de0, bool vec) {
    const int tid = threadIdx.x;
    const int span = kn * TD;
    if (vec) {
        const int nq = span >> 2;                  // float4 per row slice
        const int qsel = tid & 1, rl = tid >> 1;   // 2 lanes per group, 128 groups
        const int R2 = nrows < 128 ? nrows : 128;  // rows per pass
        const int P2 = 128 / R2;                   // float4 pairs per pass
        const int rr0 = rl % R2, pl = rl / R2;
        if (pl >= P2) return;
        for (int qp = pl; 2 * qp < nq; qp += P2) {
            const int q = 2 * qp + qsel;
            if (q >= nq) continue;
            const int u = 4 * q;
            const int k = u / TD, dd = u % TD;
            const bool inside = kbase + k < kdim && de0 + dd < d;
            const int64_t col = (int64_t)(kbase + k) * d + de0 + dd;
            for (int rr = rr0; rr < nrows; rr += R2) {
                float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                if (inside && row0 + rr < nmax)
                    v = *reinterpret_cast<const float4 *>(src + (row0 + rr) * row_w + col);
                dst[(u + 0) * S + rr] = v.x;
                dst[(u + 1) * S + rr] = v.y;
                dst[(u + 2) * S + rr] = v.z;
                dst[(u + 3) * S + rr] = v.w;
            }
        }
    } else {
        const int esel = tid & 7, rl = tid >> 3;   // 8 lanes per group, 32 groups
        const int R8 = nrows < 32 ? nrows : 32;
        const int P8 = 32 / R8;
        const int rr0 = rl % R8, pl = rl / R8;
        if (pl >= P8) return;
        for (int ep = pl; 8 * ep < span; ep += P8) {
            const int u = 8 * ep + esel;
            if (u >= span) continue;
            const int k = u / TD, dd = u % TD;
            const bool inside = kbase + k < kdim && de0 + dd < d;
            const int64_t col = (int64_t)(kbase + k) * d + de0 + dd;
            for (int rr = rr0; rr < nrows; rr += R8) {
                float v = 0.f;
                if (inside && row0 + rr < nmax) v = src[(row0 + rr) * row_w + col];
                dst[u * S + rr] = v;
            }
        }
    }
}

// stage_rows writes dst[(rr * TD + dd) * S + k] (the dw operands: positions k contiguous per
// row and delta).  Consecutive lanes take consecutive units (float4 or float) of one row, so
// a warp stores within one row wherever a row slice holds 32 units or more; with TD == 1 a
// float4 lands as one 16-byte store.
template <int TD>
__device__ __forceinline__ void stage_rows(float *__restrict__ dst, int S,
                                           const float *__restrict__ src, int64_t row_w,
                                           int64_t row0, int64_t nmax, int nrows, int kbase,
                                           int kn, int kdim, int d, int de0, bool vec) {
    const int tid = threadIdx.x;
    const int span = kn * TD;
    const int nq = vec ? span >> 2 : span;  // units per row slice
    int q0, qstep, r0, rstep;
    if (nq <= kThreads) {
        q0 = tid % nq;
        qstep = nq;  // one unit per thread and row
        r0 = tid / nq;
        rstep = kThreads / nq;
        if (r0 >= rstep) return;
    } else {
        q0 = tid;
        qstep = kThreads;
        r0 = 0;
        rstep = 1;
    }
    for (int q = q0; q < nq; q += qstep) {
        const int u = vec ? 4 * q : q;
        const int k = u / TD, dd = u % TD;
        const bool inside = kbase + k < kdim && de0 + dd < d;
        const int64_t col = (int64_t)(kbase + k) * d + de0 + dd;
        for (int rr = r0; rr < nrows; rr += rstep) {
            const bool ok = inside && row0 + rr < nmax;
            if (vec) {
                float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                if (ok) v = *reinterpret_cast<const float4 *>(src + (row0 + rr) * row_w + col);
                if (TD == 1) {
                    *reinterpret_cast<float4 *>(dst + rr * S + u) = v;
                } else {
                    const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        dst[(rr * TD + (u + e) % TD) * S + (u + e) / TD] = vv[e];
                }
            } else {
                dst[(rr * TD + dd) * S + k] = ok ? src[(row0 + rr) * row_w + col] : 0.f;
            }
        }
    }
}

// y tiles of y = x K + bias, or dX = dY K^T when w holds the transposed blocks.
//   in [N][a*kin*d], w [a][d][kin][kout], out [N][a*kout*d], bias [a*kout*d] or null.
template <int TD>
__global__ void __launch_bounds__(kThreads)
ks_fwd_kernel(const float *__restrict__ in, const float *__restrict__ w,
              const float *__restrict__ bias, float *__restrict__ out, int64_t N, int a, int kin,
              int kout, int d, KsTile t, int64_t tiles) {
    extern __shared__ __align__(16) float smem[];
    const int GC = t.GC, GR = t.GR, TM = GR * kR, TC = GC * kC;
    const int SX = TM + 4, SW = TC + t.padw;
    float *xs = smem;                             // [KB][TD][SX]: input, rows contiguous
    float *ws = smem + (size_t)t.KB * TD * SX;    // [KB][TD][SW]: values, columns contiguous
    const int tid = threadIdx.x;
    const bool active = tid < TD * GC * GR;
    const int dl = tid % TD, cg = (tid / TD) % GC, rg = tid / (TD * GC);
    const int64_t in_w = (int64_t)a * kin * d, out_w = (int64_t)a * kout * d;
    const int nj = (kout + TC - 1) / TC, nd = (d + TD - 1) / TD;
    // fixed per-thread assignment of the value loads: float4 (or float) column jq of rows
    // s = s0, s0 + sstep, ... of the [kb*TD][TC] value slice
    const int wcols = t.vw ? GC : TC;
    const int jq = tid % wcols, s0 = tid / wcols, sstep = kThreads / wcols;

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
            stage_cols<TD>(xs, SX, in, in_w, n0, N, TM, al * kin + k0, kb, al * kin + kin, d,
                           de0, t.vx);
            for (int s = s0; s < kb * TD; s += sstep) {
                const int kk = s / TD, dd = s % TD;
                const int de = de0 + dd;
                const float *wrow = w + (((int64_t)al * d + de) * kin + k0 + kk) * kout + j0;
                if (t.vw) {
                    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (de < d && j0 + 4 * jq < kout)
                        v = *reinterpret_cast<const float4 *>(wrow + 4 * jq);
                    *reinterpret_cast<float4 *>(ws + s * SW + 4 * jq) = v;
                } else {
                    float v = 0.f;
                    if (de < d && j0 + jq < kout) v = wrow[jq];
                    ws[s * SW + jq] = v;
                }
            }
            __syncthreads();
            if (active) {
                const float *xr = xs + dl * SX + rg * kR;
                const float *wr = ws + dl * SW + cg * kC;
                const int xstep = TD * SX, wstep = TD * SW;
#pragma unroll 2
                for (int kk = 0; kk < kb; ++kk) {
                    const float4 x0 = *reinterpret_cast<const float4 *>(xr);
                    const float4 x1 = *reinterpret_cast<const float4 *>(xr + 4);
                    const float4 w4 = *reinterpret_cast<const float4 *>(wr);
                    const float xv[kR] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
                    const float wv[kC] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                    for (int i = 0; i < kR; ++i)
#pragma unroll
                        for (int jj = 0; jj < kC; ++jj)
                            acc[i][jj] = fmaf(xv[i], wv[jj], acc[i][jj]);
                    xr += xstep;
                    wr += wstep;
                }
            }
            __syncthreads();
        }

        if (active && de0 + dl < d) {
            const int de = de0 + dl;
#pragma unroll
            for (int jj = 0; jj < kC; ++jj) {
                const int j = j0 + cg * kC + jj;
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

// wt[al][de][ga][be] = w[al][de][be][ga]: the blocks of K^T, for dX = dY K^T.
__global__ void ks_transpose_kernel(const float *__restrict__ w, float *__restrict__ wt,
                                    int64_t blocks, int b, int c) {
    const int64_t total = blocks * b * c;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t blk = e / ((int64_t)b * c);
        const int rem = (int)(e - blk * b * c);
        const int ga = rem / b, be = rem - ga * b;
        wt[e] = w[(blk * b + be) * c + ga];
    }
}

// Small blocks (b, c <= 4, e.g. the 2 x 2 blocks of butterfly factors): a stream with no
// shared memory.  Thread m = al*d + de keeps the b x c block w[al][de] in registers and runs
// over a range of rows: per row it loads its b inputs (stride d; consecutive threads take
// consecutive de, so each load instruction of a warp reads consecutive addresses wherever
// d >= 32) and stores c outputs.  Grid: x over m in blocks of kSmallThreads, y over row
// ranges of `rows` rows.
constexpr int kSmallThreads = 128;

template <int B, int C>
__global__ void __launch_bounds__(kSmallThreads)
ks_small_fwd_kernel(const float *__restrict__ in, const float *__restrict__ w,
                    const float *__restrict__ bias, float *__restrict__ out, int64_t N, int a,
                    int d, int64_t rows) {
    const int64_t m = (int64_t)blockIdx.x * kSmallThreads + threadIdx.x;
    if (m >= (int64_t)a * d) return;
    const int64_t al = m / d, de = m - al * d;
    float wv[B][C], bv[C];
#pragma unroll
    for (int be = 0; be < B; ++be)
#pragma unroll
        for (int ga = 0; ga < C; ++ga) wv[be][ga] = w[(m * B + be) * C + ga];
#pragma unroll
    for (int ga = 0; ga < C; ++ga) bv[ga] = bias ? bias[(al * C + ga) * d + de] : 0.f;
    const int64_t in_w = (int64_t)a * B * d, out_w = (int64_t)a * C * d;
    const float *src = in + al * B * d + de;
    float *dst = out + al * C * d + de;
    const int64_t n0 = (int64_t)blockIdx.y * rows;
    const int64_t n1 = n0 + rows < N ? n0 + rows : N;
#pragma unroll 4
    for (int64_t n = n0; n < n1; ++n) {
        float xv[B];
#pragma unroll
        for (int be = 0; be < B; ++be) xv[be] = src[n * in_w + (int64_t)be * d];
#pragma unroll
        for (int ga = 0; ga < C; ++ga) {
            float acc = 0.f;
#pragma unroll
            for (int be = 0; be < B; ++be) acc = fmaf(xv[be], wv[be][ga], acc);
            dst[n * out_w + (int64_t)ga * d] = acc + bv[ga];
        }
    }
}

// dw / dbias partials of small blocks: thread m sums x^T dY of its block over the row range
// blockIdx.y (rows [y*rows, (y+1)*rows)) and writes part[y] in the layout of ks_dw_kernel.
template <int B, int C>
__global__ void __launch_bounds__(kSmallThreads)
ks_small_dw_kernel(const float *__restrict__ x, const float *__restrict__ g,
                   float *__restrict__ part, int64_t N, int a, int d, int64_t rows,
                   size_t part_stride) {
    const int64_t m = (int64_t)blockIdx.x * kSmallThreads + threadIdx.x;
    if (m >= (int64_t)a * d) return;
    const int64_t al = m / d, de = m - al * d;
    float acc[B][C], bacc[C];
#pragma unroll
    for (int ga = 0; ga < C; ++ga) {
        bacc[ga] = 0.f;
#pragma unroll
        for (int be = 0; be < B; ++be) acc[be][ga] = 0.f;
    }
    const int64_t in_w = (int64_t)a * B * d, out_w = (int64_t)a * C * d;
    const float *xs = x + al * B * d + de;
    const float *gs = g + al * C * d + de;
    const int64_t n0 = (int64_t)blockIdx.y * rows;
    const int64_t n1 = n0 + rows < N ? n0 + rows : N;
#pragma unroll 4
    for (int64_t n = n0; n < n1; ++n) {
        float xv[B], gv[C];
#pragma unroll
        for (int be = 0; be < B; ++be) xv[be] = xs[n * in_w + (int64_t)be * d];
#pragma unroll
        for (int ga = 0; ga < C; ++ga) gv[ga] = gs[n * out_w + (int64_t)ga * d];
#pragma unroll
        for (int ga = 0; ga < C; ++ga) {
            bacc[ga] += gv[ga];
#pragma unroll
            for (int be = 0; be < B; ++be) acc[be][ga] = fmaf(xv[be], gv[ga], acc[be][ga]);
        }
    }
    float *pw = part + (size_t)blockIdx.y * part_stride;
#pragma unroll
    for (int be = 0; be < B; ++be)
#pragma unroll
        for (int ga = 0; ga < C; ++ga) pw[(m * B + be) * C + ga] = acc[be][ga];
    const size_t nw = (size_t)a * B * C * d;
#pragma unroll
    for (int ga = 0; ga < C; ++ga) pw[nw + (al * C + ga) * d + de] = bacc[ga];
}

// Partial sums of dw (and dbias) over one contiguous row range per CTA.  Grid = parts x
// (al, delta tile, be tile, ga tile); part p writes part[p][0 .. a*b*c*d) (dw layout) and,
// from the CTAs of the first be tile, part[p][a*b*c*d + (al*c + ga)*d + de] (dbias).
template <int TD>
__global__ void __launch_bounds__(kThreads)
ks_dw_kernel(const float *__restrict__ x, const float *__restrict__ g, float *__restrict__ part,
             int64_t N, int a, int b, int c, int d, KsTile t, int64_t rows_per_part,
             size_t part_stride) {
    extern __shared__ __align__(16) float smem[];
    const int GC = t.GC, GR = t.GR, KG = t.KG, TB = GR * kR, TC = GC * kC;
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
        stage_rows<TD>(xs, SX, x, in_w, n0, r1, kb, al * b + be0, TB, al * b + b, d, de0, t.vx);
        stage_rows<TD>(gs, SW, g, out_w, n0, r1, kb, al * c + ga0, TC, al * c + c, d, de0, t.vw);
        __syncthreads();
        if (active) {
            const float *xr = xs + (kg * TD + dl) * SX + bg * kR;
            const float *gr = gs + (kg * TD + dl) * SW + cg * kC;
            const int xstep = KG * TD * SX, gstep = KG * TD * SW;
            for (int kr = kg; kr < kb; kr += KG) {
                const float4 x0 = *reinterpret_cast<const float4 *>(xr);
                const float4 x1 = *reinterpret_cast<const float4 *>(xr + 4);
                const float4 g4 = *reinterpret_cast<const float4 *>(gr);
                const float xv[kR] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
                const float gv[kC] = {g4.x, g4.y, g4.z, g4.w};
                xr += xstep;
                gr += gstep;
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
                    for (int q = 0; q < KG; ++q)
                        s += red[((size_t)q * items + it) * RS + i * kC + jj];
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
                const int ga = ga0 + cg * kC + jj;
                if (ga < c) pw[(((int64_t)al * d + de) * b + be) * c + ga] = acc[i][jj];
            }
        }
        if (with_bias) {
            const size_t nw = (size_t)a * b * c * d;
#pragma unroll
            for (int jj = 0; jj < kC; ++jj) {
                const int ga = ga0 + cg * kC + jj;
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

template <int TD>
void fwd_launch_td(unsigned grid, size_t smem, cudaStream_t st, const float *in, const float *w,
                   const float *bias, float *out, int64_t N, int a, int kin, int kout, int d,
                   const KsTile &t, int64_t tiles) {
    ks_fwd_kernel<TD><<<grid, kThreads, smem, st>>>(in, w, bias, out, N, a, kin, kout, d, t,
                                                    tiles);
}

template <int B, int C>
void small_launch(bool dw, dim3 grid, cudaStream_t st, const float *in, const float *w,
                  const float *bias, float *out, int64_t N, int a, int d, int64_t rows,
                  size_t part_stride) {
    if (dw)
        ks_small_dw_kernel<B, C><<<grid, kSmallThreads, 0, st>>>(in, w, out, N, a, d, rows,
                                                                  part_stride);
    else
        ks_small_fwd_kernel<B, C><<<grid, kSmallThreads, 0, st>>>(in, w, bias, out, N, a, d, rows);
}

template <int B>
void small_launch_c(int c, bool dw, dim3 grid, cudaStream_t st, const float *in, const float *w,
                    const float *bias, float *out, int64_t N, int a, int d, int64_t rows,
                    size_t ps) {
    switch (c) {
    case 1: small_launch<B, 1>(dw, grid, st, in, w, bias, out, N, a, d, rows, ps); break;
    case 2: small_launch<B, 2>(dw, grid, st, in, w, bias, out, N, a, d, rows, ps); break;
    case 3: small_launch<B, 3>(dw, grid, st, in, w, bias, out, N, a, d, rows, ps); break;
    default: small_launch<B, 4>(dw, grid, st, in, w, bias, out, N, a, d, rows, ps); break;
    }
}

// Small-block stream: forward (dw = false: in, w, bias -> out) or dw partials (dw = true:
// in = x, w = dY, out = partials).  b, c <= 4.
cudaError_t launch_small(bool dw, const float *in, const float *w, const float *bias, float *out,
                         int64_t N, int a, int b, int c, int d, size_t part_stride,
                         cudaStream_t st) {
    const int64_t R = small_ranges(N, a, d);
    const int64_t rows = (N + R - 1) / R;
    const dim3 grid((unsigned)cdiv((int64_t)a * d, kSmallThreads), (unsigned)R);
    switch (b) {
    case 1: small_launch_c<1>(c, dw, grid, st, in, w, bias, out, N, a, d, rows, part_stride); break;
    case 2: small_launch_c<2>(c, dw, grid, st, in, w, bias, out, N, a, d, rows, part_stride); break;
    case 3: small_launch_c<3>(c, dw, grid, st, in, w, bias, out, N, a, d, rows, part_stride); break;
    default: small_launch_c<4>(c, dw, grid, st, in, w, bias, out, N, a, d, rows, part_stride); break;
    }
    return cudaGetLastError();
}

// out = in K' (+ bias) for the KS matrix K' with blocks w [a][d][kin][kout].
cudaError_t launch_fwd(const float *in, const float *w, const float *bias, float *out, int64_t N,
                       int a, int kin, int kout, int d, cudaStream_t st) {
    if (small_blocks(kin, kout))
        return launch_small(false, in, w, bias, out, N, a, kin, kout, d, 0, st);
    const KsTile t = fwd_tile(kin, kout, d, in, w);
    const int64_t tiles = (N + (int64_t)t.GR * kR - 1) / ((int64_t)t.GR * kR) * a *
                          cdiv(d, t.TD) * cdiv(kout, (int64_t)t.GC * kC);
    const unsigned grid = (unsigned)(tiles < (1 << 30) ? tiles : (1 << 30));
    const size_t smem = tile_smem(t);
    switch (t.TD) {
    case 1: fwd_launch_td<1>(grid, smem, st, in, w, bias, out, N, a, kin, kout, d, t, tiles); break;
    case 2: fwd_launch_td<2>(grid, smem, st, in, w, bias, out, N, a, kin, kout, d, t, tiles); break;
    case 4: fwd_launch_td<4>(grid, smem, st, in, w, bias, out, N, a, kin, kout, d, t, tiles); break;
    default: fwd_launch_td<8>(grid, smem, st, in, w, bias, out, N, a, kin, kout, d, t, tiles); break;
    }
    return cudaGetLastError();
}

cudaError_t launch_dw(const DwPlan &P, const float *x, const float *g, float *part, int64_t N,
                      int a, int b, int c, int d, cudaStream_t st) {
    const unsigned grid = (unsigned)(P.parts * P.tiles_per_part);
    const size_t smem = tile_smem(P.t);
    const int64_t rpp = P.rows_per_part;
    const size_t ps = P.part_stride;
    switch (P.t.TD) {
    case 1:
        ks_dw_kernel<1><<<grid, kThreads, smem, st>>>(x, g, part, N, a, b, c, d, P.t, rpp, ps);
        break;
    case 2:
        ks_dw_kernel<2><<<grid, kThreads, smem, st>>>(x, g, part, N, a, b, c, d, P.t, rpp, ps);
        break;
    case 4:
        ks_dw_kernel<4><<<grid, kThreads, smem, st>>>(x, g, part, N, a, b, c, d, P.t, rpp, ps);
        break;
    default:
        ks_dw_kernel<8><<<grid, kThreads, smem, st>>>(x, g, part, N, a, b, c, d, P.t, rpp, ps);
        break;
    }
    return cudaGetLastError();
}

// Workspace: [K^T's blocks: a*b*c*d floats, padded to 64][parts x part_stride partials].
size_t wt_floats(int a, int b, int c, int d) {
    return ((size_t)a * b * c * d + 63) & ~(size_t)63;
}

}  // namespace

extern "C" {

size_t ks_linear_workspace_size(int64_t N, int a, int b, int c, int d, kron_dtype_t dtype) {
    if (N < 0 || a < 1 || b < 1 || c < 1 || d < 1 || dtype != KRON_F32) return 0;
    if ((int64_t)a * b * d > kMaxWidth || (int64_t)a * c * d > kMaxWidth ||
        N > ((int64_t)1 << 40))
        return 0;
    const DwPlan P = dw_plan(N, a, b, c, d, nullptr, nullptr);  // sizes do not depend on pointers
    const int64_t parts = small_blocks(b, c) ? small_ranges(N, a, d) : P.parts;
    return (wt_floats(a, b, c, d) + (size_t)parts * P.part_stride) * 4;
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
    const cudaError_t e = launch_fwd((const float *)x, (const float *)w, (const float *)bias,
                                     (float *)y, N, a, b, c, d, (cudaStream_t)stream);
    if (e != cudaSuccess)
        return ks_fail(KRON_ERR_CUDA, "KS forward launch: %s", cudaGetErrorString(e));
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
        if (e != cudaSuccess)
            return ks_fail(KRON_ERR_CUDA, "KS zero fill: %s", cudaGetErrorString(e));
        return KRON_OK;
    }
    float *wt = static_cast<float *>(workspace);
    float *part = wt + wt_floats(a, b, c, d);
    if (dX) {
        const size_t tb = (nw + 255) / 256;
        ks_transpose_kernel<<<(unsigned)(tb < 2048 ? tb : 2048), 256, 0, cs>>>(
            (const float *)w, wt, (int64_t)a * d, b, c);
        e = cudaGetLastError();
        if (e == cudaSuccess)
            e = launch_fwd((const float *)dY, wt, nullptr, (float *)dX, N, a, c, b, d, cs);
        if (e != cudaSuccess)
            return ks_fail(KRON_ERR_CUDA, "KS dX launch: %s", cudaGetErrorString(e));
    }
    const DwPlan P = dw_plan(N, a, b, c, d, x, dY);
    int64_t parts = P.parts;
    if (small_blocks(b, c)) {
        parts = small_ranges(N, a, d);
        e = launch_small(true, (const float *)x, (const float *)dY, nullptr, part, N, a, b, c, d,
                         P.part_stride, cs);
    } else {
        if (P.parts * P.tiles_per_part > 0x7fffffff)
            return ks_fail(KRON_ERR_UNSUPPORTED, "too many dw tiles (%lld)",
                           (long long)(P.parts * P.tiles_per_part));
        e = launch_dw(P, (const float *)x, (const float *)dY, part, N, a, b, c, d, cs);
    }
    if (e != cudaSuccess) return ks_fail(KRON_ERR_CUDA, "KS dw launch: %s", cudaGetErrorString(e));
    const size_t total = nw + (dbias ? nb : 0);
    const size_t blocks = (total + 255) / 256;
    ks_reduce_kernel<<<(unsigned)(blocks < 4096 ? blocks : 4096), 256, 0, cs>>>(
        part, parts, P.part_stride, nw, nb, (float *)dw, (float *)dbias);
    e = cudaGetLastError();
    if (e != cudaSuccess)
        return ks_fail(KRON_ERR_CUDA, "KS reduce launch: %s", cudaGetErrorString(e));
    return KRON_OK;
}

}  // extern "C"
