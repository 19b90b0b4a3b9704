// simt_f32.cu -- exact-FP32 path of the Kronecker layer on the CUDA cores (FFMA).
// The kernels are written for an I/O element type TI (converted to fp32 on load); the
// library instantiates them for fp32 I/O.  All arithmetic is fp32.  Any shape whose
// tiles fit shared memory runs here.
//
// Both contractions of the vec trick (page "kronecker-layer-benchmark", sections
// "2. The vec trick" and "3. The vec trick without the loop") are fused per tile of
// R rows: the intermediate T_i = X_n B_i lives only in shared memory, so the
// permute/reshape copies of the loop-free PyTorch version never touch HBM.
//
// Forward, per tile and rank i:
//   T[(n,a),k]  = sum_j X[(n,a),j] * B_i[j,k]              (stage 1)
//   Y[(n,c),k] += sum_a C_i[a,c]  * T[(n,a),k]              (stage 2)
// Backward, per tile and rank i (G = dY):
//   U[(n,a),k]  = sum_c C_i[a,c]  * G[(n,c),k]
//   T[(n,a),k]  = sum_j X[(n,a),j] * B_i[j,k]              (recomputed)
//   dX[(n,a),j]+= sum_k U[(n,a),k] * B_i[j,k]
//   dB_i[j,k]  += sum_(n,a) X[(n,a),j] * U[(n,a),k]
//   dC_i[a,c]  += sum_(n,k) T[(n,a),k] * G[(n,c),k]
// dB, dC and dbias are accumulated per CTA over one fixed contiguous row range and
// written as partials; reduce.cu adds the partials in a fixed order.
#include "internal.h"

#include <algorithm>

namespace kron {
namespace {

constexpr int kThreads = 512;
constexpr size_t kMaxSmem = 227 * 1024;

// Register-tiled product of shared-memory operands:
//   Cm(m,n) (+)= sum_{k1<K1, k0<K0} Am(m,k1,k0) * Bm(k1,k0,n)   for every batch b
// with Am(m,k1,k0) = A[b*sab + m*sam + k1*sak1 + k0*sak0],
//      Bm(k1,k0,n) = B[b*sbb + k1*sbk1 + k0*sbk0 + n*sbn],
//      Cm(m,n)     = C[b*scb + m*scm + n].
// Thread-owned outputs are the 4x4 grid {tm + u*MT} x {tn + v*NT}: neighbouring
// threads read neighbouring columns of B, and rows of A differ by one row stride
// (odd strides keep those reads on distinct banks).
struct MM {
    const float *A; int sab, sam, sak1, sak0;
    const float *B; int sbb, sbk1, sbk0, sbn;
    float *C; int scb, scm;
    int batch, M, N, K1, K0;
};

// Work item `t` of a product: batch b, and the TM x TN output grid {tm + u*MT} x {tn + v*NT}
// of one thread (MT = ceil(M/TM), NT = ceil(N/TN)).
template <int TM, int TN>
__device__ __forceinline__ int mm_items(const MM &g) {
    return g.batch * ((g.M + TM - 1) / TM) * ((g.N + TN - 1) / TN);
}

template <int TM, int TN>
__device__ __forceinline__ void mm_item(const MM &g, int t, bool accumulate) {
    const int MT = (g.M + TM - 1) / TM, NT = (g.N + TN - 1) / TN;
    const int tiles = MT * NT;
    const int b = t / tiles;
    const int tt = t - b * tiles;
    const int tm = tt / NT, tn = tt - tm * NT;
    int row[TM], col[TN];
    bool rv[TM], cv[TN];
#pragma unroll
    for (int u = 0; u < TM; ++u) {
        row[u] = tm + u * MT;
        rv[u] = row[u] < g.M;
        if (!rv[u]) row[u] = 0;
    }
#pragma unroll
    for (int v = 0; v < TN; ++v) {
        col[v] = tn + v * NT;
        cv[v] = col[v] < g.N;
        if (!cv[v]) col[v] = 0;
    }
    const float *Ab = g.A + (size_t)b * g.sab;
    const float *Bb = g.B + (size_t)b * g.sbb;
    float acc[TM][TN];
#pragma unroll
    for (int u = 0; u < TM; ++u)
#pragma unroll
        for (int v = 0; v < TN; ++v) acc[u][v] = 0.f;
    for (int k1 = 0; k1 < g.K1; ++k1) {
        const float *Ak = Ab + k1 * g.sak1;
        const float *Bk = Bb + k1 * g.sbk1;
#pragma unroll 4
        for (int k0 = 0; k0 < g.K0; ++k0) {
            float a[TM], bb[TN];
#pragma unroll
            for (int u = 0; u < TM; ++u) a[u] = Ak[row[u] * g.sam + k0 * g.sak0];
#pragma unroll
            for (int v = 0; v < TN; ++v) bb[v] = Bk[k0 * g.sbk0 + col[v] * g.sbn];
#pragma unroll
            for (int u = 0; u < TM; ++u)
#pragma unroll
                for (int v = 0; v < TN; ++v) acc[u][v] = fmaf(a[u], bb[v], acc[u][v]);
        }
    }
    float *Cb = g.C + (size_t)b * g.scb;
#pragma unroll
    for (int u = 0; u < TM; ++u)
#pragma unroll
        for (int v = 0; v < TN; ++v)
            if (rv[u] && cv[v]) {
                float *c = Cb + row[u] * g.scm + col[v];
                *c = accumulate ? *c + acc[u][v] : acc[u][v];
            }
}

// One product over the whole CTA with 4 x 4 outputs per work item.
__device__ __forceinline__ void smem_mm(const MM &g, bool accumulate) {
    const int n = mm_items<4, 4>(g);
    for (int t = threadIdx.x; t < n; t += blockDim.x) mm_item<4, 4>(g, t, accumulate);
}

// Two independent products sharing the CTA's threads (items of the first, then of the
// second), each with its own output grid per item: products with few outputs take smaller
// grids, so that every thread has work.
template <int TM1, int TN1, int TM2, int TN2>
__device__ __forceinline__ void smem_mm2(const MM &g1, bool acc1, const MM &g2, bool acc2) {
    const int n1 = mm_items<TM1, TN1>(g1), n2 = mm_items<TM2, TN2>(g2);
    for (int t = threadIdx.x; t < n1 + n2; t += blockDim.x) {
        if (t < n1) mm_item<TM1, TN1>(g1, t, acc1);
        else mm_item<TM2, TN2>(g2, t - n1, acc2);
    }
}

// The same for three independent products.
template <int TM1, int TN1, int TM2, int TN2, int TM3, int TN3>
__device__ __forceinline__ void smem_mm3(const MM &g1, bool acc1, const MM &g2, bool acc2,
                                         const MM &g3, bool acc3) {
    const int n1 = mm_items<TM1, TN1>(g1), n2 = mm_items<TM2, TN2>(g2), n3 = mm_items<TM3, TN3>(g3);
    for (int t = threadIdx.x; t < n1 + n2 + n3; t += blockDim.x) {
        if (t < n1) mm_item<TM1, TN1>(g1, t, acc1);
        else if (t < n1 + n2) mm_item<TM2, TN2>(g2, t - n1, acc2);
        else mm_item<TM3, TN3>(g3, t - n1 - n2, acc3);
    }
}

__device__ __forceinline__ float to_f(float v) { return v; }

// Four consecutive fp32 elements (16 bytes).
__device__ __forceinline__ float4 load4(const float *p) { return *reinterpret_cast<const float4 *>(p); }
__device__ __forceinline__ void store4(float *p, float4 v) { *reinterpret_cast<float4 *>(p) = v; }

// Row r of a [rows][width] global matrix -> shared rows with stride ld; rows at or
// beyond N read as zero.  `width` elements per row (a multiple of 4), aligned rows.
template <typename TI>
__device__ __forceinline__ void load_rows(const TI *__restrict__ g, int64_t n0, int64_t N,
                                          int rows, int width, float *s, int blk, int ld) {
    // width = nblk * blk; shared row (n, b) of length blk starts at ((n*nblk)+b)*ld
    const int nblk = width / blk;
    const int w4 = width >> 2;
    for (int e = threadIdx.x; e < rows * w4; e += blockDim.x) {
        const int n = e / w4, c4 = (e - n * w4) << 2;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (n0 + n < N) v = load4(g + (n0 + n) * width + c4);
        const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const int c = c4 + t, bi = c / blk, j = c - bi * blk;
            s[(n * nblk + bi) * ld + j] = vv[t];
        }
    }
}

struct FwdLayout {
    int R, ldx, ldb, ldc, ldt, skip;
    size_t offX, offB, offC, offT, offY, offI, total;  // in floats (offI: int lists)
};

inline size_t up4(size_t v) { return (v + 3) & ~(size_t)3; }  // 16-byte aligned offsets

FwdLayout fwd_layout(const Shape &s, int R, bool skip) {
    FwdLayout L;
    L.R = R;
    L.skip = skip;
    L.ldx = s.m1 + 1;
    L.ldb = s.m2 + 1;
    L.ldc = s.q + 1;
    L.ldt = s.m2 + 1;
    size_t o = 0;
    L.offX = o; o = up4(o + (size_t)R * s.p * L.ldx);
    L.offB = o; o = up4(o + (size_t)s.m1 * L.ldb);
    L.offC = o; o = up4(o + (size_t)s.p * L.ldc);
    L.offT = o; o = up4(o + (size_t)R * s.p * L.ldt);
    L.offY = o; o = up4(o + (size_t)R * s.q * s.m2);
    // zero-block skip: row map [p], column pointers [q+1], column lists [p*q] (ints)
    L.offI = o; if (skip) o = up4(o + (size_t)s.p + s.q + 1 + (size_t)s.p * s.q);
    L.total = o;
    return L;
}

// acc_smem: the dC/dB/dbias accumulators live in shared memory; otherwise (large
// r*p*q) they are accumulated in place in the CTA's own workspace partial.
struct BwdLayout {
    int R, ldx, ldg, ldb, ldc, ldt, acc_smem, skip, resident;
    size_t offX, offG, offDX, offU, offT, offB, offC, offDC, offDB, offDb, offI, total;
};

// resident: the factors of every rank stay in shared memory for the whole kernel (loaded
// once); otherwise rank i's are reloaded for each tile.
BwdLayout bwd_layout(const Shape &s, int R, bool acc_smem, bool skip, bool resident = false) {
    BwdLayout L;
    L.R = R;
    L.skip = skip;
    L.resident = resident;
    L.acc_smem = acc_smem;
    L.ldx = s.m1 + 1;
    L.ldg = s.m2 + 1;
    L.ldb = s.m2 + 1;
    L.ldc = s.q + 1;
    L.ldt = s.m2 + 1;
    size_t o = 0;
    L.offX = o; o = up4(o + (size_t)R * s.p * L.ldx);
    L.offG = o; o = up4(o + (size_t)R * s.q * L.ldg);
    L.offDX = o; o = up4(o + (size_t)R * s.p * L.ldx);
    L.offU = o; o = up4(o + (size_t)R * s.p * L.ldt);
    L.offT = o; o = up4(o + (size_t)R * s.p * L.ldt);
    const size_t nf = resident ? (size_t)s.r : 1;   // ranks held
    L.offB = o; o = up4(o + nf * s.m1 * L.ldb);
    L.offC = o; o = up4(o + nf * s.p * L.ldc);
    L.offDC = L.offDB = L.offDb = o;
    if (acc_smem) {
        L.offDC = o; o = up4(o + (size_t)s.r * s.p * s.q);
        L.offDB = o; o = up4(o + (size_t)s.r * s.m1 * s.m2);
        L.offDb = o; o = up4(o + (size_t)s.q * s.m2);
    }
    // zero-block skip: row pointers [p+1] and row lists [p*q] of S's nonzeros (ints)
    L.offI = o; if (skip) o = up4(o + (size_t)s.p + 1 + (size_t)s.p * s.q);
    L.total = o;
    return L;
}

// Nonzero pattern of S for the zero-block skip (KRON_FLAG_SKIP_ZERO_BLOCKS).  C_i = S (.) A_i,
// so C_i[a,c] = 0 for every rank wherever S[a,c] = 0 (page "kronecker-layer-benchmark",
// introduction: a zero S entry zeroes a whole block of W); those products are dropped and
// the others are accumulated in the same order as the dense loops, so the results equal
// the unflagged ones.
template <typename TI>
__device__ __forceinline__ bool s_nz(const TI *S, int e) { return to_f(S[e]) != 0.f; }

// Forward lists: rmap[a] = compact index of row a (-1 if S[a,:] is all zero), colptr /
// colidx = for each column c the rows a (ascending) with S[a,c] != 0.  Returns the number of
// nonzero rows.
template <typename TI>
__device__ int build_col_lists(const TI *__restrict__ S, const Shape &s, int *rmap, int *colptr,
                               int *colidx, int *nrows_smem) {
    const int P = s.p, Q = s.q;
    for (int a = threadIdx.x; a < P; a += blockDim.x) {
        int nz = 0;
        for (int c = 0; c < Q; ++c) nz |= s_nz(S, a * Q + c);
        rmap[a] = nz;
    }
    for (int c = threadIdx.x; c < Q; c += blockDim.x) {
        int n = 0;
        for (int a = 0; a < P; ++a) n += s_nz(S, a * Q + c);
        colptr[c + 1] = n;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int n = 0;
        for (int a = 0; a < P; ++a) rmap[a] = rmap[a] ? n++ : -1;
        *nrows_smem = n;
        colptr[0] = 0;
        for (int c = 0; c < Q; ++c) colptr[c + 1] += colptr[c];
    }
    __syncthreads();
    for (int c = threadIdx.x; c < Q; c += blockDim.x) {
        int t = colptr[c];
        for (int a = 0; a < P; ++a)
            if (s_nz(S, a * Q + c)) colidx[t++] = a;
    }
    __syncthreads();
    return *nrows_smem;
}

// Backward lists: rowptr / rowidx = for each row a the columns c (ascending) with S[a,c] != 0.
template <typename TI>
__device__ void build_row_lists(const TI *__restrict__ S, const Shape &s, int *rowptr, int *rowidx) {
    const int P = s.p, Q = s.q;
    for (int a = threadIdx.x; a < P; a += blockDim.x) {
        int n = 0;
        for (int c = 0; c < Q; ++c) n += s_nz(S, a * Q + c);
        rowptr[a + 1] = n;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        rowptr[0] = 0;
        for (int a = 0; a < P; ++a) rowptr[a + 1] += rowptr[a];
    }
    __syncthreads();
    for (int a = threadIdx.x; a < P; a += blockDim.x) {
        int t = rowptr[a];
        for (int c = 0; c < Q; ++c)
            if (s_nz(S, a * Q + c)) rowidx[t++] = c;
    }
    __syncthreads();
}

// x rows of the tile, keeping only the blocks a with rmap[a] >= 0: shared row
// (n * nra + rmap[a]) of M1 values (stride ld).
template <typename TI>
__device__ __forceinline__ void load_rows_compact(const TI *__restrict__ g, int64_t n0, int64_t N,
                                                  int rows, const Shape &s, const int *rmap,
                                                  int nra, float *sm, int ld) {
    const int width = s.p * s.m1, w4 = width >> 2;
    for (int e = threadIdx.x; e < rows * w4; e += blockDim.x) {
        const int n = e / w4, c4 = (e - n * w4) << 2;
        const int a = c4 / s.m1, j = c4 - a * s.m1;
        const int ca = rmap[a];
        if (ca < 0) continue;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (n0 + n < N) v = load4(g + (n0 + n) * width + c4);
        float *d = sm + (size_t)(n * nra + ca) * ld + j;
        d[0] = v.x; d[1] = v.y; d[2] = v.z; d[3] = v.w;
    }
}

// Factor i into shared memory: Bs[j*ldb + k] = B_i[j,k], Cs[a*ldc + c] = S[a,c]*A_i[a,c].
template <typename TI>
__device__ __forceinline__ void load_factors(const TI *__restrict__ S,
                                             const TI *__restrict__ A,
                                             const TI *__restrict__ B, int i, const Shape &s,
                                             float *Bs, int ldb, float *Cs, int ldc) {
    const TI *Bi = B + (size_t)i * s.m1 * s.m2;
    for (int e = threadIdx.x; e < s.m1 * s.m2; e += blockDim.x) {
        const int j = e / s.m2, k = e - j * s.m2;
        Bs[j * ldb + k] = to_f(Bi[e]);
    }
    const TI *Ai = A + (size_t)i * s.p * s.q;
    for (int e = threadIdx.x; e < s.p * s.q; e += blockDim.x) {
        const int a = e / s.q, c = e - a * s.q;
        Cs[a * ldc + c] = to_f(S[e]) * to_f(Ai[e]);
    }
}

template <typename TI>
__global__ void __launch_bounds__(kThreads)
kron_fwd_simt_kernel(const TI *__restrict__ x, const TI *__restrict__ S,
                     const TI *__restrict__ A, const TI *__restrict__ B,
                     const TI *__restrict__ bias, TI *__restrict__ y, Shape s,
                     FwdLayout L) {
    extern __shared__ __align__(16) float smem[];
    float *Xs = smem + L.offX, *Bs = smem + L.offB, *Cs = smem + L.offC;
    float *Ts = smem + L.offT, *Ys = smem + L.offY;
    const int R = L.R;
    const int64_t n0 = (int64_t)blockIdx.x * R;
    const int P = s.p, Q = s.q, M1 = s.m1, M2 = s.m2;

    if (L.skip) {
        // zero-block skip: stage 1 only on rows a with a nonzero in S, stage 2 over each
        // column's nonzero rows (same accumulation order as the dense loops)
        __shared__ int nra_s;
        int *rmap = reinterpret_cast<int *>(smem + L.offI), *colptr = rmap + P, *colidx = colptr + Q + 1;
        const int nra = build_col_lists(S, s, rmap, colptr, colidx, &nra_s);
        load_rows_compact(x, n0, s.N, R, s, rmap, nra, Xs, L.ldx);
        for (int i = 0; i < s.r; ++i) {
            __syncthreads();
            load_factors(S, A, B, i, s, Bs, L.ldb, Cs, L.ldc);
            __syncthreads();
            if (nra > 0) {
                MM g1{Xs, 0, L.ldx, 0, 1, Bs, 0, 0, L.ldb, 1, Ts, 0, L.ldt, 1, R * nra, M2, 1, M1};
                smem_mm(g1, false);
            }
            __syncthreads();
            for (int e = threadIdx.x; e < R * Q * M2; e += blockDim.x) {
                const int n = e / (Q * M2), c = (e / M2) % Q, k = e % M2;
                float acc = 0.f;
                for (int t = colptr[c]; t < colptr[c + 1]; ++t) {
                    const int a = colidx[t];
                    acc = fmaf(Cs[a * L.ldc + c], Ts[(n * nra + rmap[a]) * L.ldt + k], acc);
                }
                Ys[e] = i > 0 ? Ys[e] + acc : acc;
            }
        }
    } else {
        load_rows(x, n0, s.N, R, P * M1, Xs, M1, L.ldx);
        for (int i = 0; i < s.r; ++i) {
            __syncthreads();  // previous stage 2 done with Bs/Cs/Ts
            load_factors(S, A, B, i, s, Bs, L.ldb, Cs, L.ldc);
            __syncthreads();
            // stage 1: T[(n,a),k] = sum_j X[(n,a),j] B_i[j,k]
            MM g1{Xs, 0, L.ldx, 0, 1, Bs, 0, 0, L.ldb, 1, Ts, 0, L.ldt, 1, R * P, M2, 1, M1};
            smem_mm(g1, false);
            __syncthreads();
            // stage 2, batched over rows n: Y[(n,c),k] += sum_a C_i[a,c] T[(n,a),k]
            MM g2{Cs, 0, 1, 0, L.ldc, Ts, P * L.ldt, 0, L.ldt, 1, Ys, Q * M2, M2, R, Q, M2, 1, P};
            smem_mm(g2, i > 0);
        }
    }
    __syncthreads();
    // y = Y + bias, coalesced float4 stores
    const int out = Q * M2, o4 = out >> 2;
    for (int e = threadIdx.x; e < R * o4; e += blockDim.x) {
        const int n = e / o4, c4 = (e - n * o4) << 2;
        if (n0 + n >= s.N) continue;
        float4 v = *reinterpret_cast<const float4 *>(Ys + n * out + c4);
        if (bias) {
            const float4 bv = load4(bias + c4);
            v.x += bv.x; v.y += bv.y; v.z += bv.z; v.w += bv.w;
        }
        store4(y + (n0 + n) * out + c4, v);
    }
}

template <typename TI>
__global__ void __launch_bounds__(kThreads)
kron_bwd_simt_kernel(const TI *__restrict__ x, const TI *__restrict__ S,
                     const TI *__restrict__ A, const TI *__restrict__ B,
                     const TI *__restrict__ G, TI *__restrict__ dX,
                     float *__restrict__ ws, int64_t rows_per_part, size_t ws_stride, Shape s,
                     BwdLayout L) {
    extern __shared__ __align__(16) float smem[];
    float *Xs = smem + L.offX, *Gs = smem + L.offG, *dXs = smem + L.offDX;
    float *Us = smem + L.offU, *Ts = smem + L.offT, *Bs = smem + L.offB, *Cs = smem + L.offC;
    const int R = L.R;
    const int P = s.p, Q = s.q, M1 = s.m1, M2 = s.m2;
    const size_t n_dc = (size_t)s.r * P * Q, n_db = (size_t)s.r * M1 * M2;
    float *part = ws + (size_t)blockIdx.x * ws_stride;
    float *dCs = L.acc_smem ? smem + L.offDC : part;
    float *dBs = L.acc_smem ? smem + L.offDB : part + n_dc;
    float *dbs = L.acc_smem ? smem + L.offDb : part + n_dc + n_db;
    const int64_t lo = (int64_t)blockIdx.x * rows_per_part;
    const int64_t hi = lo + rows_per_part < s.N ? lo + rows_per_part : s.N;

    for (size_t e = threadIdx.x; e < n_dc; e += blockDim.x) dCs[e] = 0.f;
    for (size_t e = threadIdx.x; e < n_db; e += blockDim.x) dBs[e] = 0.f;
    for (int e = threadIdx.x; e < Q * M2; e += blockDim.x) dbs[e] = 0.f;
    int *rowptr = reinterpret_cast<int *>(smem + L.offI), *rowidx = rowptr + P + 1;
    if (L.skip) build_row_lists(S, s, rowptr, rowidx);
    if (L.resident)   // every rank's factors, once (made visible by the first tile's barrier)
        for (int i = 0; i < s.r; ++i)
            load_factors(S, A, B, i, s, Bs + (size_t)i * M1 * L.ldb, L.ldb, Cs + (size_t)i * P * L.ldc, L.ldc);

    for (int64_t n0 = lo; n0 < hi; n0 += R) {
        __syncthreads();
        load_rows(x, n0, hi, R, P * M1, Xs, M1, L.ldx);
        load_rows(G, n0, hi, R, Q * M2, Gs, M2, L.ldg);
        __syncthreads();
        // dbias partial: rows beyond the range were loaded as zero
        for (int o = threadIdx.x; o < Q * M2; o += blockDim.x) {
            const int c = o / M2, k = o - c * M2;
            float acc = 0.f;
            for (int n = 0; n < R; ++n) acc += Gs[(n * Q + c) * L.ldg + k];
            dbs[o] += acc;
        }
        for (int i = 0; i < s.r; ++i) {
            __syncthreads();
            float *Bi = Bs, *Ci = Cs;
            if (L.resident) {
                Bi = Bs + (size_t)i * M1 * L.ldb;
                Ci = Cs + (size_t)i * P * L.ldc;
            } else {
                load_factors(S, A, B, i, s, Bs, L.ldb, Cs, L.ldc);
                __syncthreads();
            }
            // U[(n,a),k] = sum_c C_i[a,c] G[(n,c),k]          (batched over n)
            if (L.skip) {   // only the nonzero S[a,c], in the dense loop's order
                for (int e = threadIdx.x; e < R * P * M2; e += blockDim.x) {
                    const int n = e / (P * M2), a = (e / M2) % P, k = e % M2;
                    float acc = 0.f;
                    for (int t = rowptr[a]; t < rowptr[a + 1]; ++t) {
                        const int c = rowidx[t];
                        acc = fmaf(Ci[a * L.ldc + c], Gs[(n * Q + c) * L.ldg + k], acc);
                    }
                    Us[(n * P + a) * L.ldt + k] = acc;
                }
            }
            // T[(n,a),k] = sum_j X[(n,a),j] B_i[j,k]  (with U when U is a dense product)
            MM gt{Xs, 0, L.ldx, 0, 1, Bi, 0, 0, L.ldb, 1, Ts, 0, L.ldt, 1, R * P, M2, 1, M1};
            if (L.skip) {
                smem_mm(gt, false);
            } else {
                MM gu{Ci, 0, L.ldc, 0, 1, Gs, Q * L.ldg, 0, L.ldg, 1, Us, P * L.ldt, L.ldt,
                      R, P, M2, 1, Q};
                smem_mm2<4, 4, 4, 4>(gu, false, gt, false);
            }
            __syncthreads();
            // dX[(n,a),j] += sum_k U[(n,a),k] B_i[j,k]
            MM gx{Us, 0, L.ldt, 0, 1, Bi, 0, 0, 1, L.ldb, dXs, 0, L.ldx, 1, R * P, M1, 1, M2};
            // dB_i[j,k] += sum_(n,a) X[(n,a),j] U[(n,a),k]
            MM gb{Xs, 0, 1, 0, L.ldx, Us, 0, 0, L.ldt, 1, dBs + (size_t)i * M1 * M2, 0, M2,
                  1, M1, M2, 1, R * P};
            // dC_i[a,c] += sum_n sum_k T[(n,a),k] G[(n,c),k]
            MM gc{Ts, 0, L.ldt, P * L.ldt, 1, Gs, 0, Q * L.ldg, 1, L.ldg,
                  dCs + (size_t)i * P * Q, 0, Q, 1, P, Q, R, M2};
            // three independent products (dX reads U, dB reads X and U, dC reads T and G) in
            // one pass: dX on 2 x 4 grids, dB and dC, whose outputs are few, on 2 x 2 grids
            smem_mm3<2, 4, 2, 2, 2, 2>(gx, i > 0, gb, true, gc, true);
        }
        __syncthreads();
        if (dX) {
            const int w = P * M1, w4 = w >> 2;
            for (int e = threadIdx.x; e < R * w4; e += blockDim.x) {
                const int n = e / w4, c4 = (e - n * w4) << 2;
                if (n0 + n >= hi) continue;
                float v[4];
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    const int c = c4 + t, a = c / M1, j = c - a * M1;
                    v[t] = dXs[(n * P + a) * L.ldx + j];
                }
                store4(dX + (n0 + n) * w + c4, make_float4(v[0], v[1], v[2], v[3]));
            }
        }
    }
    if (!L.acc_smem) return;  // accumulated in place
    __syncthreads();
    for (size_t e = threadIdx.x; e < n_dc; e += blockDim.x) part[e] = dCs[e];
    for (size_t e = threadIdx.x; e < n_db; e += blockDim.x) part[n_dc + e] = dBs[e];
    for (size_t e = threadIdx.x; e < (size_t)Q * M2; e += blockDim.x)
        part[n_dc + n_db + e] = dbs[e];
}

// ---------------------------------------------------------------------------------------
// Forward for a compiled shape (P, Q, M1, M2, R rows per tile): the same two stages with
// compile-time strides, 4 x 8 outputs per thread and 128-bit shared-memory loads, so the
// inner loops are FFMAs plus few loads; every rank's factors stay in shared memory and each
// thread keeps its 4 x 8 block of Y in registers across the ranks (no Y tile in shared
// memory).  Persistent CTAs, two per SM.
//   stage 1, item (rb, kb): T[4rb+u][8kb+v] = sum_j X[4rb+u][j] B_i[j][8kb+v]
//   stage 2, item (n, cb, kb): Y_n[4cb+u][8kb+v] += sum_a C_i[a][4cb+u] T[n*P+a][8kb+v]
constexpr int kF32Threads = 256;

template <int P_, int Q_, int M1_, int M2_, int R_, int RT_>
struct F32Cfg {
    static constexpr int P = P_, Q = Q_, M1 = M1_, M2 = M2_, R = R_, RT = RT_;
    static constexpr int LDX = M1 + 1;    // A operand of stage 1: scalar loads down a column
    static constexpr int LDT = M2 + 4;    // 16-byte rows: STS.128 / LDS.128
    static constexpr int LDB = M2 + 4, LDC = Q + 4;
    static constexpr int OFF_X = 0;
    static constexpr int OFF_T = OFF_X + RT * P * LDX;
    static constexpr int OFF_B = (OFF_T + RT * P * LDT + 3) & ~3;
    static constexpr int OFF_C = OFF_B + R * M1 * LDB;
    static constexpr int TOTAL = OFF_C + R * P * LDC;   // floats
    static_assert((RT * P / 4) * (M2 / 8) == kF32Threads, "stage 1: one 4 x 8 block per thread");
    static_assert(RT * (Q / 4) * (M2 / 8) == kF32Threads, "stage 2: one 4 x 8 block per thread");
    static_assert(P % 4 == 0 && Q % 4 == 0 && M1 % 4 == 0 && M2 % 8 == 0, "vector widths");
    static_assert(TOTAL * 4 + 1024 <= 116736, "two CTAs per SM");
};

// TR = true computes dX = dY W^T with the same two stages (dX_n = sum_i C_i G_n B_i^T): the
// kernel's (P, Q, M1, M2) are the layer's (q, p, m2, m1), x is dY, y is dX, there is no bias,
// and the factors are read transposed while they are packed.
template <class Cfg, typename TI, bool TR = false>
__global__ void __launch_bounds__(kF32Threads, 2)
kron_fwd_f32_kernel(const TI *__restrict__ x, const TI *__restrict__ S, const TI *__restrict__ A,
                    const TI *__restrict__ B, const TI *__restrict__ bias, TI *__restrict__ y,
                    int64_t N) {
    constexpr int P = Cfg::P, Q = Cfg::Q, M1 = Cfg::M1, M2 = Cfg::M2, R = Cfg::R, RT = Cfg::RT;
    constexpr int LDX = Cfg::LDX, LDT = Cfg::LDT, LDB = Cfg::LDB, LDC = Cfg::LDC;
    constexpr int KB = M2 / 8, CB = Q / 4;
    extern __shared__ __align__(16) float smem[];
    float *Xs = smem + Cfg::OFF_X, *Ts = smem + Cfg::OFF_T, *Bs = smem + Cfg::OFF_B, *Cs = smem + Cfg::OFF_C;
    const int t = threadIdx.x;
    // every rank's factors, once: Bs[i][j][k] = B_i[j][k], Cs[i][a][c] = S[a][c] A_i[a][c]
    // (transposed: B_i[k][j] of the layer's m2' x m1' B_i, and C_i[c][a] of its q' x p' C_i)
    for (int e = t; e < R * M1 * M2; e += kF32Threads) {
        const int i = e / (M1 * M2), j = (e / M2) % M1, k = e % M2;
        Bs[(i * M1 + j) * LDB + k] = to_f(B[TR ? ((size_t)i * M2 + k) * M1 + j : (size_t)e]);
    }
    for (int e = t; e < R * P * Q; e += kF32Threads) {
        const int i = e / (P * Q), a = (e / Q) % P, c = e % Q;
        Cs[(i * P + a) * LDC + c] =
            TR ? to_f(S[c * P + a]) * to_f(A[((size_t)i * Q + c) * P + a])
               : to_f(S[a * Q + c]) * to_f(A[e]);
    }
    // this thread's items
    const int rb = t / KB, kb1 = t % KB;                          // stage 1
    const int n2 = t / (CB * KB), cb = (t / KB) % CB, kb2 = t % KB; // stage 2
    const int64_t tiles = (N + RT - 1) / RT;
    for (int64_t tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
        const int64_t n0 = tile * RT;
        __syncthreads();   // the previous tile is done with Xs (and the factors are in place)
        constexpr int W4 = P * M1 / 4;
        for (int e = t; e < RT * W4; e += kF32Threads) {
            const int n = e / W4, c4 = (e % W4) * 4, a = c4 / M1, j = c4 % M1;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (n0 + n < N) v = load4(x + (n0 + n) * (P * M1) + c4);
            float *d = Xs + (n * P + a) * LDX + j;
            d[0] = v.x; d[1] = v.y; d[2] = v.z; d[3] = v.w;
        }
        float yacc[4][8];
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int v = 0; v < 8; ++v) yacc[u][v] = 0.f;
        for (int i = 0; i < R; ++i) {
            __syncthreads();   // Xs written / the previous rank's stage 2 is done with Ts
            {
                const float *Bi = Bs + i * M1 * LDB + kb1 * 8;
                const float *Xr = Xs + (rb * 4) * LDX;
                float acc[4][8];
#pragma unroll
                for (int u = 0; u < 4; ++u)
#pragma unroll
                    for (int v = 0; v < 8; ++v) acc[u][v] = 0.f;
#pragma unroll 8
                for (int j = 0; j < M1; ++j) {
                    const float4 b0 = *reinterpret_cast<const float4 *>(Bi + j * LDB);
                    const float4 b1 = *reinterpret_cast<const float4 *>(Bi + j * LDB + 4);
                    const float bb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const float a = Xr[u * LDX + j];
#pragma unroll
                        for (int v = 0; v < 8; ++v) acc[u][v] = fmaf(a, bb[v], acc[u][v]);
                    }
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    float *d = Ts + (rb * 4 + u) * LDT + kb1 * 8;
                    *reinterpret_cast<float4 *>(d) = make_float4(acc[u][0], acc[u][1], acc[u][2], acc[u][3]);
                    *reinterpret_cast<float4 *>(d + 4) = make_float4(acc[u][4], acc[u][5], acc[u][6], acc[u][7]);
                }
            }
            __syncthreads();
            {
                const float *Ci = Cs + i * P * LDC + cb * 4;
                const float *Tn = Ts + (n2 * P) * LDT + kb2 * 8;
#pragma unroll 8
                for (int a = 0; a < P; ++a) {
                    const float4 c4 = *reinterpret_cast<const float4 *>(Ci + a * LDC);
                    const float4 t0 = *reinterpret_cast<const float4 *>(Tn + a * LDT);
                    const float4 t1 = *reinterpret_cast<const float4 *>(Tn + a * LDT + 4);
                    const float cc[4] = {c4.x, c4.y, c4.z, c4.w};
                    const float tt[8] = {t0.x, t0.y, t0.z, t0.w, t1.x, t1.y, t1.z, t1.w};
#pragma unroll
                    for (int u = 0; u < 4; ++u)
#pragma unroll
                        for (int v = 0; v < 8; ++v) yacc[u][v] = fmaf(cc[u], tt[v], yacc[u][v]);
                }
            }
        }
        // y[n][(4cb+u)*M2 + 8kb+v] = Y + bias
        if (n0 + n2 < N) {
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int o = (cb * 4 + u) * M2 + kb2 * 8;
                float v8[8];
#pragma unroll
                for (int v = 0; v < 8; ++v) v8[v] = yacc[u][v] + (bias ? to_f(bias[o + v]) : 0.f);
                TI *dst = y + (n0 + n2) * (Q * M2) + o;
                store4(dst, make_float4(v8[0], v8[1], v8[2], v8[3]));
                store4(dst + 4, make_float4(v8[4], v8[5], v8[6], v8[7]));
            }
        }
    }
}

// ---------------------------------------------------------------------------------------
// Parameter-gradient partials for a compiled shape (dX comes from kron_fwd_f32_kernel<TR>).
// Per tile of RT rows, every product reads both operands with 128-bit shared loads along a
// contiguous index, from arrays laid out for it:
//   T  [(n,a)][(i,k)] = sum_j  XT[j][(n,a)] Ball[j][(i,k)]    -> stored as TT[(n,k)][(i,a)]
//   U  [(n,a)][(i,k)] = sum_c  CT_i[c][a]   G[(n,c)][k]       (batch (n, i))
//   dB [j][(i,k)]    += sum_(n,a) X[(n,a)][j] U[(n,a)][(i,k)]
//   dC [(i,a)][c]    += sum_(n,k) TT[(n,k)][(i,a)] GT[(n,k)][c]
//   dbias[c*m2+k]    += sum_n G[(n,c)][k]
// dB and dC stay in registers for the CTA's whole row range, each thread summing one half of
// every tile's K range; the two halves are added in a fixed order at the end and written as
// the range's partials (the layout reduce.cu sums).  One CTA per SM of two 256-thread
// groups: group 0 takes the T blocks and then the dB blocks, group 1 the U and dC blocks.
constexpr int kPgF32Threads = 512;
constexpr int kPgF32Group = 256;

template <int P_, int Q_, int M1_, int M2_, int R_, int RT_>
struct PgF32Cfg {
    static constexpr int P = P_, Q = Q_, M1 = M1_, M2 = M2_, R = R_, RT = RT_;
    static constexpr int LX = M1 + 4, LXT = RT * P + 4, LG = M2 + 4, LGT = Q + 4;
    static constexpr int LTT = R * P + 4, LU = R * M2 + 4, LB = R * M2 + 4, LCT = P + 4;
    static constexpr int OFF_X = 0;
    static constexpr int OFF_XT = OFF_X + RT * P * LX;
    static constexpr int OFF_G = OFF_XT + M1 * LXT;
    static constexpr int OFF_GT = OFF_G + RT * Q * LG;
    static constexpr int OFF_TT = OFF_GT + RT * M2 * LGT;
    static constexpr int OFF_U = OFF_TT + RT * M2 * LTT;
    static constexpr int OFF_B = OFF_U + RT * P * LU;
    static constexpr int OFF_CT = OFF_B + M1 * LB;
    static constexpr int TOTAL = OFF_CT + R * Q * LCT;   // floats
    // work items per product, one 4 x 8 block each
    static constexpr int NT_T = (RT * P / 4) * (R * M2 / 8);
    static constexpr int NT_U = RT * R * (P / 4) * (M2 / 8);
    static constexpr int NT_DB = (M1 / 4) * (R * M2 / 8);
    static constexpr int NT_DC = (R * P / 4) * (Q / 8);
    static_assert(NT_T == kPgF32Group && NT_U == kPgF32Group, "T and U: one block per thread");
    static_assert(2 * NT_DB == kPgF32Group && 2 * NT_DC == kPgF32Group,
                  "dB and dC: one block per thread and K half");
    static_assert((Q * M2) % kPgF32Threads == 0, "dbias columns per thread");
    static_assert(M1 / 4 == 8 && (R * M2 / 8) % 4 == 0, "dB block order: 8 row blocks, column blocks by 4");
    static_assert(P % 4 == 0 && Q % 8 == 0 && M1 % 4 == 0 && M2 % 8 == 0 && (RT * P) % 8 == 0 &&
                  (RT * M2) % 2 == 0, "vector widths and K halves");
    static_assert(TOTAL * 4 <= 232448, "shared memory");
};

template <class Cfg, typename TI>
__global__ void __launch_bounds__(kPgF32Threads, 1)
kron_pgrad_f32_kernel(const TI *__restrict__ x, const TI *__restrict__ S, const TI *__restrict__ A,
                      const TI *__restrict__ B, const TI *__restrict__ G, float *__restrict__ ws,
                      int64_t rows_per_part, size_t ws_stride, int64_t N) {
    constexpr int P = Cfg::P, Q = Cfg::Q, M1 = Cfg::M1, M2 = Cfg::M2, R = Cfg::R, RT = Cfg::RT;
    constexpr int LX = Cfg::LX, LXT = Cfg::LXT, LG = Cfg::LG, LGT = Cfg::LGT;
    constexpr int LTT = Cfg::LTT, LU = Cfg::LU, LB = Cfg::LB, LCT = Cfg::LCT;
    constexpr int DBIAS = Q * M2 / kPgF32Threads;
    extern __shared__ __align__(16) float smem[];
    float *X = smem + Cfg::OFF_X, *XT = smem + Cfg::OFF_XT, *Gs = smem + Cfg::OFF_G;
    float *GT = smem + Cfg::OFF_GT, *TT = smem + Cfg::OFF_TT, *U = smem + Cfg::OFF_U;
    float *Ball = smem + Cfg::OFF_B, *CT = smem + Cfg::OFF_CT;
    const int t = threadIdx.x;
    // factors, once: Ball[j][(i,k)] = B_i[j][k]; CT[i][c][a] = S[a][c] A_i[a][c]
    for (int e = t; e < R * M1 * M2; e += kPgF32Threads) {
        const int i = e / (M1 * M2), j = (e / M2) % M1, k = e % M2;
        Ball[j * LB + i * M2 + k] = to_f(B[e]);
    }
    for (int e = t; e < R * P * Q; e += kPgF32Threads) {
        const int i = e / (P * Q), a = (e / Q) % P, c = e % Q;
        CT[(i * Q + c) * LCT + a] = to_f(S[a * Q + c]) * to_f(A[e]);
    }
    // this thread's blocks (tl: index within the group)
    const int grp = t / kPgF32Group, tl = t % kPgF32Group;
    const int t_rb = tl % (RT * P / 4), t_kb = tl / (RT * P / 4);        // T: 4 (n,a) x 8 (i,k)
    const int u_kb = tl % (M2 / 8), u_ab = (tl / (M2 / 8)) % (P / 4),      // U: 4 a x 8 k of (n,i)
              u_b = tl / ((M2 / 8) * (P / 4)), u_n = u_b / R, u_i = u_b % R;
    const int half = tl / Cfg::NT_DB;                                      // K half of dB and dC
    // dB blocks: a warp takes 4 column blocks x 8 row blocks, so its 128-bit loads of U touch
    // 128 contiguous bytes per instruction (one wavefront) instead of 16 spread blocks
    const int db_h = tl % Cfg::NT_DB;
    const int db_cb = (db_h % 4) + 4 * (db_h / 32), db_jb = (db_h / 4) % 8;
    const int dc_cb = tl % (Q / 8), dc_mb = (tl % Cfg::NT_DC) / (Q / 8);
    float acc2[4][8], dbias[DBIAS];   // acc2: dB (group 0) or dC (group 1) over the range
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 8; ++v) acc2[u][v] = 0.f;
#pragma unroll
    for (int e = 0; e < DBIAS; ++e) dbias[e] = 0.f;

    const int64_t lo = (int64_t)blockIdx.x * rows_per_part;
    const int64_t hi = lo + rows_per_part < N ? lo + rows_per_part : N;
    for (int64_t n0 = lo; n0 < hi; n0 += RT) {
        __syncthreads();   // the previous tile's dB/dC pass is done with X, G, TT, U
        // x rows -> X[(n,a)][j] and XT[j][(n,a)]; dY rows -> G[(n,c)][k] and GT[(n,k)][c]
        // (rows at or past the range end read as zero)
        for (int e = t; e < RT * P * M1 / 4; e += kPgF32Threads) {
            const int n = e / (P * M1 / 4), c4 = (e % (P * M1 / 4)) * 4, a = c4 / M1, j = c4 % M1;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (n0 + n < hi) v = load4(x + (n0 + n) * (P * M1) + c4);
            *reinterpret_cast<float4 *>(X + (n * P + a) * LX + j) = v;
            XT[(j + 0) * LXT + n * P + a] = v.x;
            XT[(j + 1) * LXT + n * P + a] = v.y;
            XT[(j + 2) * LXT + n * P + a] = v.z;
            XT[(j + 3) * LXT + n * P + a] = v.w;
        }
        for (int e = t; e < RT * Q * M2 / 4; e += kPgF32Threads) {
            const int n = e / (Q * M2 / 4), c4 = (e % (Q * M2 / 4)) * 4, c = c4 / M2, k = c4 % M2;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (n0 + n < hi) v = load4(G + (n0 + n) * (Q * M2) + c4);
            *reinterpret_cast<float4 *>(Gs + (n * Q + c) * LG + k) = v;
            GT[(n * M2 + k + 0) * LGT + c] = v.x;
            GT[(n * M2 + k + 1) * LGT + c] = v.y;
            GT[(n * M2 + k + 2) * LGT + c] = v.z;
            GT[(n * M2 + k + 3) * LGT + c] = v.w;
        }
        __syncthreads();
        if (grp == 0) {   // T block: rows (n,a) = 4 t_rb .. +3, columns (i,k) = 8 t_kb .. +7  -> TT
            float acc[4][8];
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int v = 0; v < 8; ++v) acc[u][v] = 0.f;
#pragma unroll 4
            for (int j = 0; j < M1; ++j) {
                const float4 a4 = *reinterpret_cast<const float4 *>(XT + j * LXT + t_rb * 4);
                const float4 b0 = *reinterpret_cast<const float4 *>(Ball + j * LB + t_kb * 8);
                const float4 b1 = *reinterpret_cast<const float4 *>(Ball + j * LB + t_kb * 8 + 4);
                const float aa[4] = {a4.x, a4.y, a4.z, a4.w};
                const float bb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
                for (int u = 0; u < 4; ++u)
#pragma unroll
                    for (int v = 0; v < 8; ++v) acc[u][v] = fmaf(aa[u], bb[v], acc[u][v]);
            }
            const int n = (t_rb * 4) / P, a0 = (t_rb * 4) % P;
#pragma unroll
            for (int v = 0; v < 8; ++v) {
                const int ik = t_kb * 8 + v, i = ik / M2, k = ik % M2;
                *reinterpret_cast<float4 *>(TT + (n * M2 + k) * LTT + i * P + a0) =
                    make_float4(acc[0][v], acc[1][v], acc[2][v], acc[3][v]);
            }
        }
        else {   // U block of (n, i): a = 4 u_ab .. +3, k = 8 u_kb .. +7
            float acc[4][8];
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int v = 0; v < 8; ++v) acc[u][v] = 0.f;
            const float *Ci = CT + u_i * Q * LCT + u_ab * 4;
            const float *Gn = Gs + u_n * Q * LG + u_kb * 8;
#pragma unroll 4
            for (int c = 0; c < Q; ++c) {
                const float4 a4 = *reinterpret_cast<const float4 *>(Ci + c * LCT);
                const float4 b0 = *reinterpret_cast<const float4 *>(Gn + c * LG);
                const float4 b1 = *reinterpret_cast<const float4 *>(Gn + c * LG + 4);
                const float aa[4] = {a4.x, a4.y, a4.z, a4.w};
                const float bb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
                for (int u = 0; u < 4; ++u)
#pragma unroll
                    for (int v = 0; v < 8; ++v) acc[u][v] = fmaf(aa[u], bb[v], acc[u][v]);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                float *d = U + (u_n * P + u_ab * 4 + u) * LU + u_i * M2 + u_kb * 8;
                *reinterpret_cast<float4 *>(d) = make_float4(acc[u][0], acc[u][1], acc[u][2], acc[u][3]);
                *reinterpret_cast<float4 *>(d + 4) = make_float4(acc[u][4], acc[u][5], acc[u][6], acc[u][7]);
            }
        }
        // dbias: this thread's columns, summed over the tile's rows
#pragma unroll
        for (int e = 0; e < DBIAS; ++e) {
            const int o = t + e * kPgF32Threads, c = o / M2, k = o % M2;
#pragma unroll
            for (int n = 0; n < RT; ++n) dbias[e] += Gs[(n * Q + c) * LG + k];
        }
        __syncthreads();
        if (grp == 0) {   // dB: j = 4 db_jb .. +3, (i,k) = 8 db_cb .. +7, K = (n,a) in this thread's half
            constexpr int KH = RT * P / 2;
            const float *Xk = X + (half * KH) * LX + db_jb * 4;
            const float *Uk = U + (half * KH) * LU + db_cb * 8;
#pragma unroll 4
            for (int kk = 0; kk < KH; ++kk) {
                const float4 a4 = *reinterpret_cast<const float4 *>(Xk + kk * LX);
                const float4 b0 = *reinterpret_cast<const float4 *>(Uk + kk * LU);
                const float4 b1 = *reinterpret_cast<const float4 *>(Uk + kk * LU + 4);
                const float aa[4] = {a4.x, a4.y, a4.z, a4.w};
                const float bb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
                for (int u = 0; u < 4; ++u)
#pragma unroll
                    for (int v = 0; v < 8; ++v) acc2[u][v] = fmaf(aa[u], bb[v], acc2[u][v]);
            }
        } else {   // dC: (i,a) = 4 dc_mb .. +3, c = 8 dc_cb .. +7, K = (n,k) in this thread's half
            constexpr int KH = RT * M2 / 2;
            const float *Tk = TT + (half * KH) * LTT + dc_mb * 4;
            const float *Gk = GT + (half * KH) * LGT + dc_cb * 8;
#pragma unroll 4
            for (int kk = 0; kk < KH; ++kk) {
                const float4 a4 = *reinterpret_cast<const float4 *>(Tk + kk * LTT);
                const float4 b0 = *reinterpret_cast<const float4 *>(Gk + kk * LGT);
                const float4 b1 = *reinterpret_cast<const float4 *>(Gk + kk * LGT + 4);
                const float aa[4] = {a4.x, a4.y, a4.z, a4.w};
                const float bb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
                for (int u = 0; u < 4; ++u)
#pragma unroll
                    for (int v = 0; v < 8; ++v) acc2[u][v] = fmaf(aa[u], bb[v], acc2[u][v]);
            }
        }
    }
    // the two K halves, added in a fixed order (half 0 + half 1), as this range's partials
    __syncthreads();
    float *scratch = smem;   // the tile arrays are free now
    constexpr int NDB = R * M1 * M2, NDC = R * P * Q;
    auto db_index = [&](int u, int v) {
        const int j = db_jb * 4 + u, ik = db_cb * 8 + v, i = ik / M2, k = ik % M2;
        return (i * M1 + j) * M2 + k;
    };
    auto dc_index = [&](int u, int v) {
        const int ia = dc_mb * 4 + u, i = ia / P, a = ia % P, c = dc_cb * 8 + v;
        return (i * P + a) * Q + c;
    };
    // scratch[dB | dC] holds half 1; the output index: dB after dC in the partial layout
    auto sidx = [&](int u, int v) { return grp == 0 ? db_index(u, v) : NDB + dc_index(u, v); };
    auto pidx = [&](int u, int v) { return grp == 0 ? NDC + db_index(u, v) : dc_index(u, v); };
    if (half == 1) {
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int v = 0; v < 8; ++v) scratch[sidx(u, v)] = acc2[u][v];
    }
    __syncthreads();
    float *part = ws + (size_t)blockIdx.x * ws_stride;
    if (half == 0) {
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int v = 0; v < 8; ++v) part[pidx(u, v)] = acc2[u][v] + scratch[sidx(u, v)];
    }
#pragma unroll
    for (int e = 0; e < DBIAS; ++e) part[NDC + NDB + t + e * kPgF32Threads] = dbias[e];
}

size_t fwd_bytes(const Shape &s, int R, bool skip) { return fwd_layout(s, R, skip).total * sizeof(float); }
size_t bwd_bytes(const Shape &s, int R, bool acc_smem, bool skip, bool resident = false) {
    return bwd_layout(s, R, acc_smem, skip, resident).total * sizeof(float);
}

// Backward tile choice: rows per tile R and where the accumulators live.  The row split
// (and with it the summation order of the partials) does not depend on `skip`: R is chosen
// for the larger (skip) layout whenever that fits.
BwdLayout bwd_choose(const Shape &s, bool skip) {
    for (int acc = 1; acc >= 0; --acc)
        for (int R : {4, 2, 1})
            for (int res = 1; res >= 0; --res)
                if (bwd_bytes(s, R, acc, true, res) <= kMaxSmem) return bwd_layout(s, R, acc, skip, res);
    for (int acc = 1; acc >= 0; --acc)
        for (int R : {4, 2, 1})
            if (bwd_bytes(s, R, acc, false) <= kMaxSmem) return bwd_layout(s, R, acc, false);
    BwdLayout none = bwd_layout(s, 1, false, false);
    none.R = 0;
    return none;
}

}  // namespace

int simt_forward_rows(const Shape &s) {
    for (int R : {8, 4, 2, 1})
        if (fwd_bytes(s, R, false) <= kMaxSmem) return R;
    return 0;
}

int simt_backward_rows(const Shape &s) { return bwd_choose(s, false).R; }

namespace {

template <class Cfg, typename TI, bool TR = false>
cudaError_t launch_fwd_f32(const void *x, const void *S, const void *A, const void *B,
                           const void *bias, void *y, const Shape &s, cudaStream_t st) {
    const size_t smem = (size_t)Cfg::TOTAL * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(kron_fwd_f32_kernel<Cfg, TI, TR>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t tiles = (s.N + Cfg::RT - 1) / Cfg::RT;
    const int64_t slots = (int64_t)tc::num_sms() * 2;   // persistent: two CTAs per SM
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(tiles < slots ? tiles : slots));
    cfg.blockDim = dim3(kF32Threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    return cudaLaunchKernelEx(&cfg, kron_fwd_f32_kernel<Cfg, TI, TR>, (const TI *)x, (const TI *)S,
                              (const TI *)A, (const TI *)B, (const TI *)bias, (TI *)y, s.N);
}

template <typename TI>
cudaError_t simt_forward_t(const void *x, const void *S, const void *A, const void *B,
                           const void *bias, void *y, const Shape &s, bool skip, cudaStream_t st) {
    // compiled shapes: the tutorial layer (p = q = m1 = m2 = 32, r = 4), 8 rows per tile
    if (!skip && s.p == 32 && s.q == 32 && s.m1 == 32 && s.m2 == 32 && s.r == 4)
        return launch_fwd_f32<F32Cfg<32, 32, 32, 32, 4, 8>, TI>(x, S, A, B, bias, y, s, st);
    int R = simt_forward_rows(s);
    // the skip lists need room too; rows of a tile are independent, so R may shrink
    while (skip && R > 1 && fwd_bytes(s, R, true) > kMaxSmem) R >>= 1;
    if (skip && fwd_bytes(s, R, true) > kMaxSmem) skip = false;
    const FwdLayout L = fwd_layout(s, R, skip);
    const size_t smem = L.total * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(kron_fwd_simt_kernel<TI>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t tiles = (s.N + R - 1) / R;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)tiles);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    return cudaLaunchKernelEx(&cfg, kron_fwd_simt_kernel<TI>, (const TI *)x, (const TI *)S,
                              (const TI *)A, (const TI *)B, (const TI *)bias, (TI *)y, s, L);
}

template <typename TI>
cudaError_t simt_backward_t(const void *x, const void *S, const void *A, const void *B,
                            const void *dY, void *dX, float *ws, int parts, const Shape &s,
                            bool skip, cudaStream_t st) {
    // compiled shape (the tutorial layer): dX by the forward kernel with transposed factors,
    // the parameter-gradient partials by their own kernel
    if (!skip && s.p == 32 && s.q == 32 && s.m1 == 32 && s.m2 == 32 && s.r == 4) {
        using PC = PgF32Cfg<32, 32, 32, 32, 4, 2>;
        cudaError_t e = cudaSuccess;
        if (dX) {
            const Shape ts{s.N, s.q, s.p, s.m2, s.m1, s.r};
            e = launch_fwd_f32<F32Cfg<32, 32, 32, 32, 4, 8>, TI, true>(dY, S, A, B, nullptr, dX, ts, st);
            if (e != cudaSuccess) return e;
        }
        const size_t smem = (size_t)PC::TOTAL * sizeof(float);
        e = cudaFuncSetAttribute(kron_pgrad_f32_kernel<PC, TI>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        const int64_t rows_per_part = (s.N + parts - 1) / parts;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)parts);
        cfg.blockDim = dim3(kPgF32Threads);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = st;
        return cudaLaunchKernelEx(&cfg, kron_pgrad_f32_kernel<PC, TI>, (const TI *)x, (const TI *)S,
                                  (const TI *)A, (const TI *)B, (const TI *)dY, ws, rows_per_part,
                                  partial_stride(s), s.N);
    }
    const BwdLayout L = bwd_choose(s, skip);
    const size_t smem = L.total * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(kron_bwd_simt_kernel<TI>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t rows_per_part = (s.N + parts - 1) / parts;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)parts);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    return cudaLaunchKernelEx(&cfg, kron_bwd_simt_kernel<TI>, (const TI *)x, (const TI *)S,
                              (const TI *)A, (const TI *)B, (const TI *)dY, (TI *)dX, ws,
                              rows_per_part, partial_stride(s), s, L);
}

}  // namespace

cudaError_t simt_forward(const void *x, const void *S, const void *A, const void *B,
                         const void *bias, void *y, const Shape &s, bool skip, cudaStream_t st) {
    return simt_forward_t<float>(x, S, A, B, bias, y, s, skip, st);
}

cudaError_t simt_backward(const void *x, const void *S, const void *A, const void *B,
                          const void *dY, void *dX, float *ws, int parts, const Shape &s,
                          bool skip, cudaStream_t st) {
    return simt_backward_t<float>(x, S, A, B, dY, dX, ws, parts, s, skip, st);
}

}  // namespace kron
