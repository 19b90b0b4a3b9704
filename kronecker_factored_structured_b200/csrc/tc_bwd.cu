// tc_bwd.cu -- backward of the Kronecker layer on the sm_100a tensor cores (tcgen05).
//
// Gradients of L = <G, y> (G = dY), W = sum_i kron(C_i, B_i), C_i = S (.) A_i (page
// "kronecker-layer-benchmark", section "1. Build W, then multiply"; the page leaves the
// backward to autograd).  Two kernels:
//
//   dX_n = sum_i C_i G_n B_i^T        the forward's vec trick with C_i^T and B_i^T: the
//                                     forward kernel in its transposed mode (tc_fwd.cu)
//   parameter gradients (this file), per tile of NT = 2 rows, all on the tensor cores:
//     T [(i,k),(n,a)] = sum_j  B_i[j,k] X_n[a,j]      A = B_all^T (TMEM), B = x tile
//     U [(i,a),(n,k)] = sum_c  C_i[a,c] G_n[c,k]      A = C_stack (TMEM), B = G tile MN-major
//     dC[(i,a),c]    += sum_(n,k) T[n,a,i,k] G_n[c,k]  A = T2 [(i,a)][(n,k)], B = G tile
//     dB[(i,k),j]    += sum_(n,a) U[n,a,i,k] X_n[a,j]  A = U2 [(i,k)][(n,a)], B = X^T [j][(n,a)]
//     dbias[c*m2+k]  += sum_n G_n[c,k]
//   dC and dB accumulate in TMEM over the CTA's fixed, contiguous range of rows and are
//   written to the workspace as that range's partials; after a grid barrier (cooperative
//   launch) the same kernel adds the partials in a fixed order and forms dA = dC (.) S and
//   dS = sum_i dC_i (.) A_i, plus l1 * sign(S) when the page's l1 penalty on S is fused
//   (bitwise reproducible, no separate reduction launch).
//
// The G tile serves as a K-major operand (dC) and as an MN-major one (U): TMA brings it in
// both shared-memory layouts for TF32 (whose MN-major layout is the 128-byte swizzle with
// 32-byte atoms), once for BF16 (one swizzled tile is valid both ways).  dB reads a K-major
// X^T that the dbias warps write from the x tile (an MN-major x operand costs ~40 clocks
// more per MMA).  The other permutes are the two epilogues, which move the T and U
// accumulators (TMEM -> registers) into the K-major layouts dC and dB read, one 128-byte
// row segment per warp store.
//
// Warp roles (736 threads, one CTA per SM, tiles of the CTA's row range in order):
//   warp 0       TMA producer: an SI-deep ring of input sets (x and G tiles)
//   warp 1       issuer A: T and U of tile t into TMEM (two accumulator slots); owns TMEM
//   warp 2       issuer B: dC and dB of tile t from T2/U2 (an SB-deep ring in shared memory)
//   warps 3-18   epilogue: every tile by all 16 warps, per TMEM lane quadrant one warp for
//                each of T -> T2 and U -> U2 and column block n = 0, 1 (the TMEM slots and
//                T2/U2 buffers rotate tile by tile)
//   warps 19-22  X^T copies of the x tiles (for dB) and dbias column sums of the G tiles
// Issuers run their loops as whole warps and let one elected lane issue each burst; every
// consumer takes the tiles in order, so no mbarrier phase can be mistaken for another.
#include "internal.h"
#include "tc_ptx.cuh"

#include <cuda_runtime.h>

namespace kron {
namespace tc {

namespace {

template <typename T> struct BE;
template <> struct BE<float> {
    static constexpr int bytes = 4;
    static constexpr uint32_t fmt = 2;
    static constexpr bool tf32 = true;
};
template <> struct BE<__nv_bfloat16> {
    static constexpr int bytes = 2;
    static constexpr uint32_t fmt = 1;
    static constexpr bool tf32 = false;
};

constexpr int imin(int a, int b) { return a < b ? a : b; }
constexpr int kPgThreads = 736;
constexpr int kPgPrefetch = 1;  // tiles in flight to L2 ahead of the input ring (measured: 1 beats 3, 6, 12)

template <typename T>
__device__ __forceinline__ float bld(const void *p, size_t i) {
    if constexpr (BE<T>::tf32) return static_cast<const float *>(p)[i];
    else return __bfloat162float(static_cast<const __nv_bfloat16 *>(p)[i]);
}


template <int P_, int Q_, int M1_, int M2_, int R_, typename T_>
struct PgCfg {
    using T = T_;
    static constexpr int P = P_, Q = Q_, M1 = M1_, M2 = M2_, R = R_;
    static constexpr int E = BE<T>::bytes;
    static constexpr bool TWO = BE<T>::tf32;       // TF32: dY in two layouts
    static constexpr int NT = 2;                   // rows per tile
    static constexpr int XR = NT * P, GR = NT * Q; // tile rows: (n,a) and (n,c)
    static constexpr int XRB = M1 * E, GRB = M2 * E;  // tile row bytes = their swizzle width
    static constexpr int X_BYTES = XR * XRB, G_BYTES = GR * GRB;
    // one input set: x (K-major), G (K-major) [, G MN-major] by TMA, then X^T [j][(n,a)]
    // (K-major, 128-byte rows per K-chunk) written by the dbias warps for dB
    static constexpr int XT_BYTES = M1 * NT * P * E;
    static constexpr int OFF_XK = 0, OFF_GK = X_BYTES;
    static constexpr int OFF_GM = TWO ? X_BYTES + G_BYTES : OFF_GK;
    static constexpr int TMA_BYTES = X_BYTES + G_BYTES * (TWO ? 2 : 1);
    static constexpr int OFF_XT = TMA_BYTES;
    static constexpr int IN_BYTES = TMA_BYTES + XT_BYTES;
    // intermediates: T2 [(i,a)][(n,k)] and U2 [(i,k)][(n,a)], 128 rows, K-major, SW128
    static constexpr int T2K = NT * M2, U2K = NT * P;          // K extents (elements)
    static constexpr int T2_BYTES = 128 * T2K * E, U2_BYTES = 128 * U2K * E;
    static constexpr int IB = T2_BYTES + U2_BYTES;
    static constexpr int BAR_BYTES = 512;
    static constexpr int SMEM_MAX = 232448;
    static constexpr int FREE = SMEM_MAX - 1024 - BAR_BYTES;
    // the input ring holds a set from its load until dC/dB of that tile are done (the
    // longest lifetime in the pipeline), so it gets every byte the intermediates leave
    static constexpr int SB = FREE - 4 * IB >= 8 * IN_BYTES ? 4 : 2;
    static constexpr int SI = imin(12, (FREE - SB * IB) / IN_BYTES);
    static constexpr int OFF_IN = 0;
    static constexpr int OFF_I = SI * IN_BYTES;
    static constexpr int OFF_BAR = OFF_I + SB * IB;
    static constexpr int SMEM = OFF_BAR + BAR_BYTES + 1024;
    // TMEM columns
    static constexpr int TM_BT = 0;                          // B_all^T: lanes (i,k), K = j
    static constexpr int TM_C = TM_BT + M1 * E / 4;          // C_stack: lanes (i,a), K = c
    static constexpr int TM_DT = TM_C + Q * E / 4;           // T: 2 slots of XR columns
    static constexpr int TM_DU = TM_DT + 2 * XR;             // U: 2 slots of NT*M2 columns
    static constexpr int TM_DC = TM_DU + 2 * NT * M2;        // dC: lanes (i,a), Q columns
    static constexpr int TM_DB = TM_DC + Q;                  // dB: lanes (i,k), M1 columns
    static constexpr int TM_USED = TM_DB + M1;
    static constexpr int TM_COLS = 512;
    static constexpr uint32_t ID_T = idesc_f32acc(128, XR, BE<T>::fmt);
    static constexpr uint32_t ID_U = idesc_f32acc(128, NT * M2, BE<T>::fmt) | kBMajorMN;
    static constexpr uint32_t ID_DC = idesc_f32acc(128, Q, BE<T>::fmt);
    static constexpr uint32_t ID_DB = idesc_f32acc(128, M1, BE<T>::fmt);
    // MN-major layouts of the input tiles: TF32 128-byte rows with 32-byte atoms (4-row
    // groups), BF16 the tile's own swizzle (8-row groups); both put 1 KB per 32-byte K step
    static constexpr uint32_t MN_LAYOUT = TWO ? kLayoutSw128Atom32 : layout_type(XRB);
    static constexpr uint32_t MN_SBO = TWO ? 4 * 128 : 8 * XRB;

    static_assert(R * P == 128 && R * M2 == 128, "T2/U2 rows and the U/T accumulators: M = 128");
    static_assert(XR % 32 == 0 && XR <= 256 && (NT * M2) % 32 == 0 && NT * M2 <= 256, "N of T and U");
    static_assert(XRB == GRB && (XRB == 128 || (!TWO && XRB == 64)),
                  "tile rows of 128 bytes (TF32) or 64/128 bytes (BF16)");
    static_assert(Q % 32 == 0 && M1 % 32 == 0 && Q <= 256 && M1 <= 256, "N of dC and dB");
    static_assert((T2K * E) % 128 == 0 && (U2K * E) % 128 == 0, "T2/U2 rows: whole 128-byte chunks");
    static_assert(P == 32 && M2 == 32, "epilogue: one 32-column TMEM load per (n, block)");
    static_assert(SI >= 2 && SB >= 2, "rings");
    static_assert(TMA_BYTES % 1024 == 0 && XT_BYTES % 1024 == 0 && (NT * P * E) % 128 == 0,
                  "X^T region: whole 128-byte K-chunks, 1024-aligned");
    static_assert(M1 == 32, "X^T transpose: lanes take the 32 rows j");
    static_assert(3 * SI + 4 + 2 * SB + 2 + 3 <= BAR_BYTES / 8, "barrier region");
    static_assert(TM_USED <= TM_COLS, "TMEM budget");
    static_assert(SMEM <= SMEM_MAX, "shared memory budget");
};

struct PgArgs {
    const void *S, *A, *B;
    float *ws;
    size_t ws_stride;
    int num_tiles;
    int tiles_per_part;
    int *device_error;
    unsigned *arrived;     // grid barrier counter (zeroed by the host before the launch)
    float *dS, *dA, *dB, *dbias;
    double l1;             // weight of the penalty l1 * sum|S| whose gradient joins dS
};

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned *p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Fixed-order reduction of every range's partials, run by the whole grid once all of them
// are written.  The partial columns are visited as virtual columns: dC ordered (position
// (a,c), rank i) so that the r ranks of a position are adjacent, then dB, then dbias.  CTA
// g owns a run of virtual columns (a multiple of r long); within a pass of CW columns,
// GS groups of threads each sum the ranges g' = ps, ps + GS, ... of one column in double
// with four accumulators, and the GS group sums are added in a fixed order.  Only `parts`
// decides the order, so the results are bitwise reproducible.  The epilogue forms
// dA_i = dC_i (.) S and dS = sum_i dC_i (.) A_i (C_i = S (.) A_i, product rule), adds
// l1 * sign(S) to dS when the l1 penalty is fused, and writes dB and dbias.
template <class Cfg>
__device__ void reduce_ranges(const PgArgs &args, int parts, double *red, double *vals) {
    using T = typename Cfg::T;
    constexpr int P = Cfg::P, Q = Cfg::Q, M1 = Cfg::M1, M2 = Cfg::M2, R = Cfg::R;
    constexpr int NDC = R * P * Q, NDB = R * M1 * M2, NB = Q * M2;
    constexpr int NCOL = NDC + NDB + NB;
    constexpr int CW = (64 / R) * R;                 // columns per pass (whole rank groups)
    constexpr int GS = kPgThreads / CW;              // thread groups splitting the ranges
    static_assert(64 % R == 0 || R <= 64, "rank groups within one pass");
    const int per = ((NCOL + (int)gridDim.x * R - 1) / ((int)gridDim.x * R)) * R;
    const int v0 = (int)blockIdx.x * per, v1 = imin(v0 + per, NCOL);
    const int cs = threadIdx.x % CW, ps = threadIdx.x / CW;
    for (int c0 = v0; c0 < v1; c0 += CW) {
        const int v = c0 + cs;
        if (ps < GS) {
            double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;
            if (v < v1) {
                const size_t col = v < NDC ? (size_t)(v % R) * P * Q + (size_t)(v / R) : (size_t)v;
                const float *src = args.ws + col;
                int g = ps;
                for (; g + 3 * GS < parts; g += 4 * GS) {
                    a0 += (double)__ldcg(src + (size_t)g * args.ws_stride);
                    a1 += (double)__ldcg(src + (size_t)(g + GS) * args.ws_stride);
                    a2 += (double)__ldcg(src + (size_t)(g + 2 * GS) * args.ws_stride);
                    a3 += (double)__ldcg(src + (size_t)(g + 3 * GS) * args.ws_stride);
                }
                for (; g < parts; g += GS) a0 += (double)__ldcg(src + (size_t)g * args.ws_stride);
            }
            red[ps * CW + cs] = (a0 + a1) + (a2 + a3);
        }
        __syncthreads();
        if (threadIdx.x < CW) {
            double tot = 0.0;
            for (int k = 0; k < GS; ++k) tot += red[k * CW + threadIdx.x];
            vals[threadIdx.x] = tot;
        }
        __syncthreads();
        if (threadIdx.x < CW && v < v1) {
            if (v < NDC) {
                if (v % R == 0) {   // the rank group of position (a,c) = v / R
                    const int pos = v / R;
                    const double sv = (double)bld<T>(args.S, pos);
                    double ds = 0.0;
                    for (int i = 0; i < R; ++i) {
                        const double dc = vals[threadIdx.x + i];
                        args.dA[(size_t)i * P * Q + pos] = (float)(dc * sv);
                        ds += dc * (double)bld<T>(args.A, (size_t)i * P * Q + pos);
                    }
                    if (args.l1 != 0.0) ds += args.l1 * sign_of((float)sv);
                    args.dS[pos] = (float)ds;
                }
            } else if (v < NDC + NDB) {
                args.dB[v - NDC] = (float)vals[threadIdx.x];
            } else if (args.dbias) {
                args.dbias[v - NDC - NDB] = (float)vals[threadIdx.x];
            }
        }
        __syncthreads();
    }
}

// Byte offset of element (row, kbyte) of a K-major swizzled operand region: K in chunks of
// sw bytes (chunk-major), rows in 8-row atoms of 8*sw bytes.
__device__ __forceinline__ uint32_t koff(int row, int kbyte, int rows, int sw) {
    const int chunk = kbyte / sw, inner = kbyte % sw;
    return swz((uint32_t)chunk * rows * sw + (uint32_t)(row >> 3) * 8 * sw +
                   (uint32_t)(row & 7) * sw + inner,
               sw);
}

// One accumulator value as an operand element of a K-major region (fp32 bits for TF32: the
// MMA reads the top 19 bits of each operand).
template <typename T>
__device__ __forceinline__ void st_elem(uint32_t addr, uint32_t v) {
    if constexpr (BE<T>::tf32) st_shared_u32(addr, v);
    else st_shared_u16(addr, __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(v))));
}

template <class Cfg>
__global__ void __launch_bounds__(kPgThreads, 1)
kron_pgrad_tc_kernel(const __grid_constant__ CUtensorMap tm_xk, const __grid_constant__ CUtensorMap tm_gk,
                     const __grid_constant__ CUtensorMap tm_xm, const __grid_constant__ CUtensorMap tm_gm,
                     PgArgs args) {
    using T = typename Cfg::T;
    constexpr int E = Cfg::E, P = Cfg::P, Q = Cfg::Q, M1 = Cfg::M1, M2 = Cfg::M2, R = Cfg::R;
    constexpr int NT = Cfg::NT, XR = Cfg::XR, GR = Cfg::GR, SI = Cfg::SI, SB = Cfg::SB;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    const uint32_t sb = smem_u32(smem);
    const uint32_t sIn = sb + Cfg::OFF_IN, sI = sb + Cfg::OFF_I;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::OFF_BAR);
    // barrier indices
    constexpr int IN_FULL = 0, IN_FREE = SI, D_FULL = 2 * SI, D_EMPTY = 2 * SI + 2,
                  I_FULL = 2 * SI + 4, I_EMPTY = I_FULL + SB, DONE = I_FULL + 2 * SB,
                  DRAIN = DONE + 1, XT_FULL = DRAIN + 1, NBARS = XT_FULL + SI;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + NBARS);
    const Abort ab{reinterpret_cast<volatile int *>(tmem_slot + 1), args.device_error};
    auto bar = [&](int i) { return smem_u32(bars + i); };
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

    const int t0 = blockIdx.x * args.tiles_per_part;
    const int t1 = imin(t0 + args.tiles_per_part, args.num_tiles);
    const int nt = t1 > t0 ? t1 - t0 : 0;
    // Input ring loads of tile u (the producer's step; a slot's first use needs no wait).
    // Every tile is first pulled into L2 kPgPrefetch tiles ahead of its ring load, so a ring
    // slot waits on L2 rather than HBM (a slot is held until dC/dB of its tile are done; the
    // load latency is part of that cycle).
    auto prefetch = [&](int u) {
        if (u < nt) {
            tma_prefetch_l2_2d(&tm_xk, 0, (t0 + u) * XR);
            tma_prefetch_l2_2d(&tm_gk, 0, (t0 + u) * GR);
        }
    };
    auto issue = [&](int u) {
        prefetch(u + kPgPrefetch);
        const int s = u % SI;
        const uint32_t dst = sIn + s * Cfg::IN_BYTES;
        const int tile = t0 + u;
        mbar_arrive_expect_tx(bar(IN_FULL + s), Cfg::TMA_BYTES);
        tma_load_2d(dst + Cfg::OFF_XK, &tm_xk, 0, tile * XR, bar(IN_FULL + s));
        tma_load_2d(dst + Cfg::OFF_GK, &tm_gk, 0, tile * GR, bar(IN_FULL + s));
        if (Cfg::TWO) tma_load_2d(dst + Cfg::OFF_GM, &tm_gm, 0, tile * GR, bar(IN_FULL + s));
    };
    const int pre = imin(SI, nt);   // ring sets filled before the set-up below

    // ---------------- set-up: barriers, first loads, TMEM, factors into TMEM ----------------
    if (threadIdx.x == 0) {
        for (int s = 0; s < SI; ++s) {
            mbar_init(bar(IN_FULL + s), 1);
            mbar_init(bar(IN_FREE + s), 1 + 1 + 4);  // issuer A, issuer B, dbias warps
            mbar_init(bar(XT_FULL + s), 4);          // dbias warps: X^T written
        }
        for (int d = 0; d < 2; ++d) {
            mbar_init(bar(D_FULL + d), 1);
            mbar_init(bar(D_EMPTY + d), 16);         // every epilogue warp
        }
        for (int b = 0; b < SB; ++b) {
            mbar_init(bar(I_FULL + b), 16);
            mbar_init(bar(I_EMPTY + b), 1);
        }
        mbar_init(bar(DONE), 1);
        mbar_init(bar(DRAIN), 1);
        *ab.flag = 0;
        mbar_init_fence();
        prefetch_tmap(&tm_xk);
        prefetch_tmap(&tm_gk);
        if (Cfg::TWO) prefetch_tmap(&tm_gm);
        // the first ring sets stream in while the factors are packed (warp 0 is the producer)
        for (int u = 0; u < kPgPrefetch; ++u) prefetch(u);
        for (int u = 0; u < pre; ++u) issue(u);
    }
    if (warp == 1) tmem_alloc(smem_u32(tmem_slot), Cfg::TM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // A operands in TMEM, one lane per row (two BF16 values per column):
    //   B_all^T: lane (i,k), column j -> B_i[j][k];   C_stack: lane (i,a), column c -> C_i[a][c]
    // BF16: the rows in the paired lane order of pair_lane_index (the epilogue stores K pairs)
    if (warp >= 3 && warp < 11) {   // team 0 loads the A operands
        const int qd = warp & 3, L = BE<T>::tf32 ? qd * 32 + lane : pair_lane_index(qd * 32 + lane);
        const uint32_t lane_addr = (uint32_t)(qd * 32) << 16;
        const bool is_c = warp >= 7;
        const int i = is_c ? L / P : L / M2, o = is_c ? L % P : L % M2;  // o = a or k
        const int K = is_c ? Q : M1;
        auto val = [&](int j) {
            return is_c ? bld<T>(args.S, (size_t)o * Q + j) * bld<T>(args.A, ((size_t)i * P + o) * Q + j)
                        : bld<T>(args.B, ((size_t)i * M1 + j) * M2 + o);
        };
        const uint32_t base = tmem + lane_addr + (is_c ? Cfg::TM_C : Cfg::TM_BT);
        for (int c0 = 0; c0 < K * E / 4; c0 += 8) {
            uint32_t w[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                if constexpr (BE<T>::tf32) w[u] = f32_to_tf32(val(c0 + u));
                else w[u] = pack_bf16x2(val(2 * (c0 + u)), val(2 * (c0 + u) + 1));
            }
            tmem_store8(base + c0, w);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            int issued = pre;
            for (int u = pre; u < nt; ++u) {
                if (!mbar_wait(bar(IN_FREE + u % SI), ((u / SI) & 1) ^ 1, ab)) break;
                issue(u);
                issued = u + 1;
            }
            for (int u = (issued > SI ? issued - SI : 0); u < issued; ++u)
                mbar_wait_drain(bar(IN_FULL + u % SI), (u / SI) & 1);
        }
    } else if (warp == 1) {
        // ---------------- issuer A: T and U of each tile ----------------
        for (int u = 0; u < nt; ++u) {
            const int s = u % SI, d = u & 1;
            if (!warp_wait(bar(IN_FULL + s), (u / SI) & 1, ab) ||
                !warp_wait(bar(D_EMPTY + d), ((u >> 1) & 1) ^ 1, ab))
                break;
            tc_fence_after();
            if (elect_one()) {
                const uint32_t in = sIn + s * Cfg::IN_BYTES;
                const uint64_t xd = sdesc_kmajor(in + Cfg::OFF_XK, Cfg::XRB);
                const uint64_t gd = sdesc_mn(in + Cfg::OFF_GM, Cfg::MN_LAYOUT, Q * Cfg::GRB, Cfg::MN_SBO);
#pragma unroll
                for (int kk = 0; kk < M1 * E / 32; ++kk)   // T[(i,k)][(n,a)], K = j
                    mma_ts<BE<T>::tf32>(tmem + Cfg::TM_DT + d * XR, tmem + Cfg::TM_BT + kk * 8,
                                        desc_add(xd, kk * 32), Cfg::ID_T, kk > 0);
#pragma unroll
                for (int kk = 0; kk < Q * E / 32; ++kk)    // U[(i,a)][(n,k)], K = c, G MN-major
                    mma_ts<BE<T>::tf32>(tmem + Cfg::TM_DU + d * NT * M2, tmem + Cfg::TM_C + kk * 8,
                                        desc_add(gd, kk * 1024), Cfg::ID_U, kk > 0);
                mma_commit(bar(D_FULL + d));
                mma_commit(bar(IN_FREE + s));
            }
            __syncwarp();
        }
        if (elect_one()) mma_commit(bar(DRAIN));
        __syncwarp();
        if (lane == 0) mbar_wait_drain(bar(DRAIN), 0);
        __syncwarp();
    } else if (warp == 2) {
        // ---------------- issuer B: dC and dB of each tile ----------------
        for (int u = 0; u < nt; ++u) {
            const int s = u % SI, b = u % SB;
            if (!warp_wait(bar(I_FULL + b), (u / SB) & 1, ab) ||
                !warp_wait(bar(IN_FULL + s), (u / SI) & 1, ab) ||
                !warp_wait(bar(XT_FULL + s), (u / SI) & 1, ab))
                break;
            tc_fence_after();
            if (elect_one()) {
                const uint32_t in = sIn + s * Cfg::IN_BYTES;
                const uint32_t t2 = sI + b * Cfg::IB, u2 = t2 + Cfg::T2_BYTES;
                const uint64_t t2d = sdesc_kmajor(t2, 128), u2d = sdesc_kmajor(u2, 128);
                const uint64_t gkd = sdesc_kmajor(in + Cfg::OFF_GK, Cfg::GRB);
                const uint64_t xtd = sdesc_kmajor(in + Cfg::OFF_XT, 128);
#pragma unroll
                for (int kk = 0; kk < Cfg::T2K * E / 32; ++kk) {   // dC, K = (n,k)
                    const int kb = kk * 32, n = kb / Cfg::GRB, ing = kb % Cfg::GRB;
                    mma_ss<BE<T>::tf32>(tmem + Cfg::TM_DC, desc_add(t2d, (kb / 128) * 128 * 128 + kb % 128),
                                        desc_add(gkd, n * Q * Cfg::GRB + ing), Cfg::ID_DC,
                                        (u > 0 || kk > 0) ? 1u : 0u);
                }
#pragma unroll
                for (int kk = 0; kk < Cfg::U2K * E / 32; ++kk) {   // dB, K = (n,a), B = X^T
                    const int kb = kk * 32;
                    mma_ss<BE<T>::tf32>(tmem + Cfg::TM_DB, desc_add(u2d, (kb / 128) * 128 * 128 + kb % 128),
                                        desc_add(xtd, (kb / 128) * M1 * 128 + kb % 128), Cfg::ID_DB,
                                        (u > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(bar(I_EMPTY + b));
                mma_commit(bar(IN_FREE + s));
            }
            __syncwarp();
        }
        // every dC/dB MMA is complete before the epilogue reads the sums (and before TMEM goes)
        if (elect_one()) mma_commit(bar(DONE));
        __syncwarp();
        if (lane == 0) mbar_wait_drain(bar(DONE), 0);
        __syncwarp();
    } else if (warp < 19) {
        // ---------------- epilogue: T -> T2 and U -> U2, all 16 warps on every tile ----------------
        // per TMEM lane quadrant one warp for each of T and U and column block n = 0, 1
        const int role = (warp - 3) >> 2, team = role >> 1;   // team 0: the n = 0 warps
        const bool is_u = role & 1;
        const int nb = role >> 1;                              // this warp's column block n
        const int qd = warp & 3, L = qd * 32 + lane;
        const uint32_t lane_addr = (uint32_t)(qd * 32) << 16;
        // T lane (i,k), columns (n,a) -> T2 row (i,a), K (n,k);
        // U lane (i,a), columns (n,k) -> U2 row (i,k), K (n,a)
        const int i = L / 32, o = L % 32;   // o = k (T) or a (U); p = m2 = 32
        bool ok = true;
        for (int u = 0; u < nt; ++u) {
            const int d = u & 1, b = u % SB;
            if (!mbar_wait(bar(D_FULL + d), (u >> 1) & 1, ab) ||
                !mbar_wait(bar(I_EMPTY + b), ((u / SB) & 1) ^ 1, ab)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t src = tmem + lane_addr + (is_u ? Cfg::TM_DU + d * NT * M2 : Cfg::TM_DT + d * XR);
            const uint32_t dst = sI + b * Cfg::IB + (is_u ? Cfg::T2_BYTES : 0);
#pragma unroll
            for (int n = nb; n < nb + 1; ++n) {   // column block (n, w), w = a (T) or k (U)
                // rows i*32 + w of the 128B-swizzled K-major region, K byte kb: the 16-byte
                // chunk index (kb >> 4) & 7 is XORed with the row's low three bits, which are
                // w & 7 (i*32 is a multiple of 8), so only that XOR varies with w at run time
                if constexpr (BE<T>::tf32) {
                    uint32_t r[32];
                    tmem_load32(src + n * 32, r);
                    const int kb = (n * 32 + o) * E;
                    const uint32_t base = dst + (uint32_t)(kb >> 7) * 128 * 128 + (uint32_t)i * 4096 +
                                          (uint32_t)(kb & 15);
                    const uint32_t c16 = (uint32_t)(kb >> 4) & 7u;
#pragma unroll
                    for (int w = 0; w < 32; ++w)
                        st_elem<T>(base + (uint32_t)(w >> 3) * 1024 + (uint32_t)(w & 7) * 128 +
                                       ((c16 ^ (uint32_t)(w & 7)) << 4),
                                   r[w]);
                } else {
                    // BF16: two 16x256b loads (lane halves h) give thread t the K pair
                    // o = 16h + 2(t/4), o + 1 of rows w = 8rp + 2(t%4) + {0, 1}; one 4-byte
                    // store per pair and row (the four rows of a store fall on distinct
                    // swizzled chunks: no bank conflict)
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        uint32_t q[16];
                        tmem_load16x256_x4(src - lane_addr + ((uint32_t)(qd * 32 + 16 * h) << 16) + n * 32, q);
                        const int kb = (n * 32 + 16 * h + 2 * (lane >> 2)) * E;
                        const uint32_t base = dst + (uint32_t)(kb >> 7) * 128 * 128 + (uint32_t)i * 4096 +
                                              (uint32_t)(kb & 15);
                        const uint32_t c16 = (uint32_t)(kb >> 4) & 7u;
#pragma unroll
                        for (int rp = 0; rp < 4; ++rp)
#pragma unroll
                            for (int dl = 0; dl < 2; ++dl) {
                                const int w = rp * 8 + (lane & 3) * 2 + dl;
                                st_shared_u32(base + (uint32_t)(w >> 3) * 1024 + (uint32_t)(w & 7) * 128 +
                                                  ((c16 ^ (uint32_t)(w & 7)) << 4),
                                              pack_bf16x2(__uint_as_float(q[4 * rp + dl]),
                                                          __uint_as_float(q[4 * rp + 2 + dl])));
                            }
                    }
                }
            }
            tc_fence_before();
            mbar_arrive_warp(bar(D_EMPTY + d));
            fence_proxy_async();
            mbar_arrive_warp(bar(I_FULL + b));
        }
        // this range's partial dC (team 0's T warps) or dB (team 0's U warps), after the last MMAs
        float *part = args.ws + (size_t)blockIdx.x * args.ws_stride;
        const bool ok_all = named_bar_and(1, 512, ok);
        if (team == 0 && ok_all && nt > 0 && mbar_wait(bar(DONE), 0, ab)) {
            tc_fence_after();
            if (!is_u) {   // dC: lane (i,a), columns c -> dC_i[a][c]
                for (int c0 = 0; c0 < Q; c0 += 32) {
                    uint32_t r[32];
                    tmem_load32(tmem + lane_addr + Cfg::TM_DC + c0, r);
                    float4 *dstp = reinterpret_cast<float4 *>(part + (size_t)i * P * Q + (size_t)o * Q + c0);
#pragma unroll
                    for (int q4 = 0; q4 < 8; ++q4)
                        dstp[q4] = make_float4(__uint_as_float(r[4 * q4]), __uint_as_float(r[4 * q4 + 1]),
                                               __uint_as_float(r[4 * q4 + 2]), __uint_as_float(r[4 * q4 + 3]));
                }
            } else {       // dB: lane (i,k), columns j -> dB_i[j][k]
                for (int j0 = 0; j0 < M1; j0 += 32) {
                    uint32_t r[32];
                    tmem_load32(tmem + lane_addr + Cfg::TM_DB + j0, r);
#pragma unroll
                    for (int t = 0; t < 32; ++t)
                        part[(size_t)R * P * Q + (size_t)i * M1 * M2 + (size_t)(j0 + t) * M2 + o] =
                            __uint_as_float(r[t]);
                }
            }
        } else if (team == 0 && nt == 0) {
            const size_t n0 = is_u ? (size_t)R * P * Q : 0, n1 = is_u ? (size_t)R * (P * Q + M1 * M2) : (size_t)R * P * Q;
            for (size_t e = n0 + (size_t)(threadIdx.x - (is_u ? 224 : 96)); e < n1; e += 128) part[e] = 0.f;
        }
    } else {
        // ---------------- dbias: column sums of the G tiles (zero rows past N come from TMA) ----------------
        const int tid = threadIdx.x - 608;
        constexpr int PER = Q * M2 / 128;
        float acc[PER];
#pragma unroll
        for (int e = 0; e < PER; ++e) acc[e] = 0.f;
        for (int u = 0; u < nt; ++u) {
            const int s = u % SI;
            if (!mbar_wait(bar(IN_FULL + s), (u / SI) & 1, ab)) break;
            // X^T [j][(n,a)] for dB (K-major): lane j reads element j of VPC consecutive x-tile
            // rows (one 128-byte row segment per warp load) and writes them as one 16-byte
            // chunk of row j (8 consecutive rows j of a warp hit 8 distinct chunk slots)
            {
                constexpr int VPC = 16 / E;
                const uint32_t xk = sIn + s * Cfg::IN_BYTES + Cfg::OFF_XK;
                const uint32_t xt = sIn + s * Cfg::IN_BYTES + Cfg::OFF_XT;
#pragma unroll
                for (int it = tid; it < M1 * XR / VPC; it += 128) {
                    const int j = it % M1, kap0 = (it / M1) * VPC;
                    uint32_t w[4];
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        if constexpr (BE<T>::tf32) {
                            asm volatile("ld.shared.b32 %0, [%1];" : "=r"(w[h])
                                         : "r"(xk + koff(kap0 + h, j * E, XR, Cfg::XRB)) : "memory");
                        } else {
                            unsigned short lo, hi;
                            asm volatile("ld.shared.b16 %0, [%1];" : "=h"(lo)
                                         : "r"(xk + koff(kap0 + 2 * h, j * E, XR, Cfg::XRB)) : "memory");
                            asm volatile("ld.shared.b16 %0, [%1];" : "=h"(hi)
                                         : "r"(xk + koff(kap0 + 2 * h + 1, j * E, XR, Cfg::XRB)) : "memory");
                            w[h] = (uint32_t)lo | ((uint32_t)hi << 16);
                        }
                    }
                    st_shared_v4(xt + koff(j, kap0 * E, M1, 128), w[0], w[1], w[2], w[3]);
                }
                fence_proxy_async();
                mbar_arrive_warp(bar(XT_FULL + s));
            }
            const uint32_t g = sIn + s * Cfg::IN_BYTES + Cfg::OFF_GK;
#pragma unroll
            for (int e = 0; e < PER; ++e) {
                const int idx = tid + 128 * e, c = idx / M2, k = idx % M2;
#pragma unroll
                for (int n = 0; n < NT; ++n) {
                    const uint32_t a = g + koff(n * Q + c, k * E, GR, Cfg::GRB);
                    if constexpr (BE<T>::tf32) {
                        float v;
                        asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a) : "memory");
                        acc[e] += v;
                    } else {
                        unsigned short h;
                        asm volatile("ld.shared.b16 %0, [%1];" : "=h"(h) : "r"(a) : "memory");
                        acc[e] += __bfloat162float(__ushort_as_bfloat16(h));
                    }
                }
            }
            mbar_arrive_warp(bar(IN_FREE + s));
        }
        float *part = args.ws + (size_t)blockIdx.x * args.ws_stride + (size_t)R * (P * Q + M1 * M2);
#pragma unroll
        for (int e = 0; e < PER; ++e) part[tid + 128 * e] = acc[e];
    }

    // ---------------- teardown of the tensor-core state ----------------
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, Cfg::TM_COLS);
    }

    // ---------------- grid barrier, then the fixed-order reduction ----------------
    // Every CTA arrives (also after an abort, so none waits forever); the launch is
    // cooperative, so all CTAs are resident.  The wait is bounded like every other.
    volatile int *grid_ok = reinterpret_cast<volatile int *>(tmem_slot + 2);
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        atomicAdd(args.arrived, 1u);
        const uint64_t w0 = globaltimer();
        int okb = 1;
        while (ld_acquire_gpu(args.arrived) < gridDim.x) {
            if (globaltimer() - w0 > kWaitTimeoutNs) {
                okb = 0;
                if (args.device_error) atomicOr(args.device_error, 2);
                break;
            }
            __nanosleep(128);
        }
        *grid_ok = okb && !*ab.flag;
    }
    __syncthreads();
    if (*grid_ok) {
        double *red = reinterpret_cast<double *>(smem);            // input ring: idle now
        double *vals = red + kPgThreads + 64;
        reduce_ranges<Cfg>(args, (int)gridDim.x, red, vals);
    }
}

template <class Cfg>
cudaError_t launch_pgrad(const void *x, const void *S, const void *A, const void *B, const void *dY,
                         float *ws, int parts, const Shape &s, float *dS, float *dA, float *dB,
                         float *dbias, double l1, cudaStream_t st) {
    using T = typename Cfg::T;
    const bool bf16 = !BE<T>::tf32;
    CUtensorMap txk, tgk, txm, tgm;
    launch_step() = "tensor map of x";
    cudaError_t e = make_tmap_2d(&txk, x, bf16, (uint64_t)s.N * Cfg::P, Cfg::M1, Cfg::M1, Cfg::XR,
                                 Cfg::XRB, false);
    if (e != cudaSuccess) return e;
    launch_step() = "tensor map of dY";
    e = make_tmap_2d(&tgk, dY, bf16, (uint64_t)s.N * Cfg::Q, Cfg::M2, Cfg::M2, Cfg::GR, Cfg::GRB, false);
    if (e != cudaSuccess) return e;
    txm = txk;   // unused: dB reads the X^T copy the kernel writes
    tgm = tgk;
    if (Cfg::TWO) {
        launch_step() = "MN-major tensor map of dY";
        e = make_tmap_2d(&tgm, dY, bf16, (uint64_t)s.N * Cfg::Q, Cfg::M2, Cfg::M2, Cfg::GR, 128, true);
        if (e != cudaSuccess) return e;
    }
    launch_step() = "shared-memory attribute";
    e = cudaFuncSetAttribute(kron_pgrad_tc_kernel<Cfg>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Cfg::SMEM);
    if (e != cudaSuccess) return e;
    PgArgs a;
    a.S = S; a.A = A; a.B = B; a.ws = ws;
    a.ws_stride = partial_stride(s);
    a.num_tiles = (int)((s.N + Cfg::NT - 1) / Cfg::NT);
    a.tiles_per_part = (a.num_tiles + parts - 1) / parts;
    a.device_error = device_error_ptr();
    a.arrived = reinterpret_cast<unsigned *>(ws + (size_t)parts * a.ws_stride);
    a.dS = dS; a.dA = dA; a.dB = dB; a.dbias = dbias;
    a.l1 = l1;
    launch_step() = "grid barrier reset";
    e = cudaMemsetAsync(a.arrived, 0, sizeof(unsigned), st);
    if (e != cudaSuccess) return e;
    launch_step() = "kernel launch (cooperative)";
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)parts);
    cfg.blockDim = dim3(kPgThreads);
    cfg.dynamicSmemBytes = Cfg::SMEM;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kron_pgrad_tc_kernel<Cfg>, txk, tgk, txm, tgm, a);
}

using PgFn = cudaError_t (*)(const void *, const void *, const void *, const void *, const void *,
                             float *, int, const Shape &, float *, float *, float *, float *,
                             double, cudaStream_t);
struct PgEntry {
    int p, q, m1, m2, r;
    bool bf16;
    PgFn fn;
};
const PgEntry kPgTable[] = {
    {32, 32, 32, 32, 4, false, &launch_pgrad<PgCfg<32, 32, 32, 32, 4, float>>},
    {32, 32, 32, 32, 4, true, &launch_pgrad<PgCfg<32, 32, 32, 32, 4, __nv_bfloat16>>},
};

PgFn find_pg(const Shape &s, bool bf16) {
    for (const auto &f : kPgTable)
        if (f.p == s.p && f.q == s.q && f.m1 == s.m1 && f.m2 == s.m2 && f.r == s.r && f.bf16 == bf16)
            return f.fn;
    return nullptr;
}

}  // namespace

// ---- entry points of the tuned parameter-gradient kernel ----
bool tuned_pgrad_supported(const Shape &s, bool bf16) { return find_pg(s, bf16) != nullptr; }

cudaError_t tuned_pgrad(const void *x, const void *S, const void *A, const void *B,
                        const void *dY, float *ws, int parts, const Shape &s, float *dS,
                        float *dA, float *dB, float *dbias, bool bf16, double l1,
                        cudaStream_t st) {
    PgFn fn = find_pg(s, bf16);
    if (!fn) return cudaErrorNotSupported;
    return fn(x, S, A, B, dY, ws, parts, s, dS, dA, dB, dbias, l1, st);
}

}  // namespace tc
}  // namespace kron
