// tc_bwd.cu -- backward of the Kronecker layer on the sm_100a tensor cores (tcgen05).
//
// Gradients of L = <G, y> (G = dY), W = sum_i kron(C_i, B_i), C_i = S (.) A_i (page
// "kronecker-layer-benchmark", section "1. Build W, then multiply"; the page leaves the
// backward to autograd).  Per tile of NT = r rows (shapes with p = m2 = 128/r), every
// contraction on the tensor cores with K-major operands and a TMEM accumulator:
//
//   U  = C_i G_n     as Ua[(i,a),(n,k)] = sum_c C[(i,a),c] G^T[(n,k),c]
//                    and Ub[(n,k),(i,a)] = sum_c G^T[(n,k),c] C[(i,a),c]
//   T  = X_n B_i     as T[(n,a),(i,k)]  = sum_j X[(n,a),j] Bt[(i,k),j]
//   dX[(n,a),j]   = sum_(i,k) U[n,a,i,k] B_i[j,k]           A = U1 [(n,a)][(i,k)]
//   dC[(i,a),c]  += sum_(n,k) T[n,a,i,k] G[(n,c),k]          A = T2 [(i,a)][(n,k)]
//   dB[(i,k),j]  += sum_(n,a) U[n,a,i,k] X[(n,a),j]          A = U2 [(i,k)][(n,a)], B = X^T
//   dbias[c*m2+k] += sum_n G[(n,c),k]
//
// U is computed in both orientations so that each TMEM lane holds a contiguous row of
// the operand the next contraction reads; every TMEM -> shared-memory epilogue is then
// a sequence of 16-byte stores into a K-major swizzled layout (the permute the page's
// loop-free version does in HBM).  dC and dB accumulate in TMEM over the CTA's fixed,
// contiguous range of rows and are written to the workspace as that range's partial
// sums; reduce.cu adds the partials in a fixed order (bitwise reproducible).
//
// Shared memory: factors C, Bt, Bdx; tiles G, X, G^T; two intermediate buffers:
//   A: U1 (read by dX), then U2 (read by dB)       -- "A chain"
//   B: T2 (read by dC), then X^T (read by dB)      -- "B chain"
// Warp roles (448 threads, one CTA per SM):
//   warp 0       TMA producer (G and X tiles)
//   warp 1       TMEM allocator + MMA issuer (the whole warp runs the issue loop, one
//                elected lane issues each burst)
//   warps 2-5    B chain: T2 epilogue, X^T; also G^T, dbias and the dX epilogue
//   warps 6-13   A chain: U1 and U2 epilogues, 2 warps per TMEM lane quadrant
#include "internal.h"
#include "tc_ptx.cuh"

#include <cuda_runtime.h>

namespace kron {
namespace tc {

int *device_error_ptr();
cudaError_t make_tmap_2d(CUtensorMap *map, const void *base, bool bf16, uint64_t rows,
                         uint64_t cols, uint32_t box_cols, uint32_t box_rows, int sw);

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

template <int P_, int Q_, int M1_, int M2_, int R_, typename T_>
struct BwdCfg {
    using T = T_;
    static constexpr int P = P_, Q = Q_, M1 = M1_, M2 = M2_, R = R_;
    static constexpr int E = BE<T>::bytes;
    static constexpr int NT = R;                   // rows per tile
    static constexpr int SWC = imin(128, Q * E);   // K = c       (Ua, Ub)
    static constexpr int SWJ = imin(128, M1 * E);  // K = j       (T)
    static constexpr int SW128 = 128;              // K = (i,k), (n,k), (n,a): 128 * E bytes
    static constexpr int SWG = M2 * E;             // G tile rows (k) and dC's B chunks
    // region sizes (bytes)
    static constexpr int F_C = 128 * Q * E;        // C    [(i,a)][c]
    static constexpr int F_BT = 128 * M1 * E;      // Bt   [(i,k)][j]
    static constexpr int F_BD = M1 * 128 * E;      // Bdx  [j][(i,k)]
    static constexpr int TILE_G = 128 * M2 * E;    // G    [(n,c)][k]   (NT*Q rows)
    static constexpr int TILE_X = 128 * M1 * E;    // X    [(n,a)][j]   (NT*P = 128 rows)
    static constexpr int TILE_GT = 128 * Q * E;    // G^T  [(n,k)][c]
    static constexpr int BUF = 128 * 128 * E;      // U1 | U2 (A), T2 | X^T (B)
    static constexpr int OFF_C = 0;
    static constexpr int OFF_BT = OFF_C + F_C;
    static constexpr int OFF_BD = OFF_BT + F_BT;
    static constexpr int OFF_G = OFF_BD + F_BD;
    static constexpr int OFF_X = OFF_G + NT * Q * M2 * E;
    static constexpr int OFF_GT = OFF_X + TILE_X;
    static constexpr int OFF_A = OFF_GT + TILE_GT;
    static constexpr int OFF_B = OFF_A + BUF;
    static constexpr int OFF_BAR = OFF_B + BUF;
    static constexpr int SMEM = OFF_BAR + 256 + 1024;
    // TMEM columns
    static constexpr int TM_UA = 0;              // Ua : lanes (i,a), 128 columns (n,k)
    static constexpr int TM_UB = 128;            // Ub : lanes (n,k), 128 columns (i,a)
    static constexpr int TM_T = 256;             // T  : lanes (n,a), 128 columns (i,k)
    static constexpr int TM_DX = 384;            // dX : lanes (n,a), M1 columns (j)
    static constexpr int TM_DC = TM_DX + M1;     // dC : lanes (i,a), Q columns (c)
    static constexpr int TM_DB = TM_DC + Q;      // dB : lanes (i,k), M1 columns (j)
    static constexpr int TM_USED = TM_DB + M1;
    static constexpr int TM_COLS = 512;
    static constexpr uint32_t ID_128 = idesc_f32acc(128, 128, BE<T>::fmt);
    static constexpr uint32_t ID_M1 = idesc_f32acc(128, M1, BE<T>::fmt);
    static constexpr uint32_t ID_Q = idesc_f32acc(128, Q, BE<T>::fmt);

    static_assert(R * P == 128 && R * M2 == 128, "needs p = m2 = 128 / r");
    static_assert(M2 % 32 == 0 && P % 32 == 0, "a 32-column TMEM chunk maps to one operand row");
    static_assert(NT * Q <= 256 && (NT * Q) % 8 == 0, "G tile rows (TMA box) at most 256");
    static_assert(M2 * E <= 128 && P * E <= 128 && M1 * E <= 128,
                  "a block of m2 (p, m1) values must fit one 128-byte swizzle row");
    static_assert(SWG == 32 || SWG == 64 || SWG == 128, "G tile swizzle");
    static_assert(M1 % 32 == 0 && Q % 32 == 0 && M1 <= 64 && Q <= 64, "m1, q in {32, 64}");
    static_assert((M1 * E) % 32 == 0 && (M1 * E <= 128 || M1 * E % 128 == 0), "m1 bytes");
    static_assert((Q * E) % 32 == 0 && (Q * E <= 128 || Q * E % 128 == 0), "q bytes");
    static_assert(TM_USED <= TM_COLS, "TMEM budget");
    static_assert(SMEM <= 232448, "shared memory budget");
};

struct BwdTcArgs {
    const void *S, *A, *B;
    void *dX;
    float *ws;
    size_t ws_stride;
    int64_t N;
    int num_tiles;
    int tiles_per_part;
    int *device_error;
};

template <typename T>
__device__ __forceinline__ float bld(const void *p, size_t i) {
    if constexpr (BE<T>::tf32) return static_cast<const float *>(p)[i];
    else return __bfloat162float(static_cast<const __nv_bfloat16 *>(p)[i]);
}

// (row, kbyte) of a K-major swizzled operand region: K in chunks of sw bytes
// (chunk-major), rows in 8-row atoms of 8*sw bytes.
__device__ __forceinline__ uint32_t koff(int row, int kbyte, int rows, int sw) {
    const int chunk = kbyte / sw, inner = kbyte % sw;
    return swz((uint32_t)chunk * rows * sw + (uint32_t)(row >> 3) * 8 * sw +
                   (uint32_t)(row & 7) * sw + inner,
               sw);
}

template <typename T>
__device__ __forceinline__ void st16v(uint32_t addr, const float *v) {
    if constexpr (BE<T>::tf32) {
        st_shared_v4(addr, f32_to_tf32(v[0]), f32_to_tf32(v[1]), f32_to_tf32(v[2]),
                     f32_to_tf32(v[3]));
    } else {
        st_shared_v4(addr, pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                     pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
    }
}

// TMEM (32 columns of this thread's lane) -> one operand row of a 128B-swizzled K-major
// region: the 32 values go to K bytes [kbyte0, kbyte0 + 32*E) of row `row` (kbyte0
// 16-byte aligned, the run stays inside one 128-byte K-chunk).
template <typename T>
__device__ __forceinline__ void tmem_row_to_smem(uint32_t taddr, uint32_t region, int rows,
                                                 int row, int kbyte0) {
    constexpr int VPC = 16 / BE<T>::bytes;
    uint32_t r[32];
    tmem_load32(taddr, r);
    const uint32_t base = sw128_row(region, rows, kbyte0 >> 7, row);
    const int slot0 = (kbyte0 & 127) >> 4, x = row & 7;
#pragma unroll
    for (int g = 0; g < 32 / VPC; ++g) {
        const uint32_t addr = base + (uint32_t)(((slot0 + g) ^ x) << 4);
        if constexpr (BE<T>::tf32) {
            // fp32 bits as they are: the TF32 MMA reads the top 19 bits of each operand
            st_shared_v4(addr, r[4 * g], r[4 * g + 1], r[4 * g + 2], r[4 * g + 3]);
        } else {
            st_shared_v4(addr, pack_bf16x2(__uint_as_float(r[8 * g]), __uint_as_float(r[8 * g + 1])),
                         pack_bf16x2(__uint_as_float(r[8 * g + 2]), __uint_as_float(r[8 * g + 3])),
                         pack_bf16x2(__uint_as_float(r[8 * g + 4]), __uint_as_float(r[8 * g + 5])),
                         pack_bf16x2(__uint_as_float(r[8 * g + 6]), __uint_as_float(r[8 * g + 7])));
        }
    }
}

// Transpose of 8 source rows x 16 bytes (VPC elements) held as in[8][4] words into VPC
// output rows of 8 elements each: out row e = (in[0][e], ..., in[7][e]).  The
// elements are copied as they are (fp32 bits for TF32: the MMA reads the top 19 bits,
// as it does for the tiles TMA brings in).
template <typename T>
__device__ __forceinline__ void store_transposed(const uint32_t (&in)[8][4], int e,
                                                 uint32_t addr_lo, uint32_t addr_hi) {
    if constexpr (BE<T>::tf32) {
        st_shared_v4(addr_lo, in[0][e], in[1][e], in[2][e], in[3][e]);
        st_shared_v4(addr_hi, in[4][e], in[5][e], in[6][e], in[7][e]);
    } else {
        const uint32_t sel = (e & 1) ? 0x7632u : 0x5410u;
        const int w = e >> 1;
        st_shared_v4(addr_lo, __byte_perm(in[0][w], in[1][w], sel), __byte_perm(in[2][w], in[3][w], sel),
                     __byte_perm(in[4][w], in[5][w], sel), __byte_perm(in[6][w], in[7][w], sel));
    }
}

template <class Cfg>
__global__ void __launch_bounds__(448, 1)
kron_bwd_tc_kernel(const __grid_constant__ CUtensorMap tmap_g,
                   const __grid_constant__ CUtensorMap tmap_x, BwdTcArgs args) {
    using T = typename Cfg::T;
    constexpr int E = Cfg::E, P = Cfg::P, Q = Cfg::Q, M1 = Cfg::M1, M2 = Cfg::M2, R = Cfg::R;
    constexpr int NT = Cfg::NT;
    constexpr int VPC = 16 / E;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    const uint32_t sb = smem_u32(smem);
    const uint32_t sC = sb + Cfg::OFF_C, sBT = sb + Cfg::OFF_BT, sBD = sb + Cfg::OFF_BD;
    const uint32_t sG = sb + Cfg::OFF_G, sX = sb + Cfg::OFF_X, sGT = sb + Cfg::OFF_GT;
    const uint32_t sA = sb + Cfg::OFF_A, sBb = sb + Cfg::OFF_B;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::OFF_BAR);
    enum {
        G_FULL, X_FULL,   // TMA landed
        G_FREE,           // dC done with G and G^T/dbias read it (transposer arrives after X^T)
        X_FREE,           // T done with X and X^T written
        GT_FULL,          // G^T written
        UT_FULL,          // Ua, Ub, T accumulators ready; G^T consumed
        E1A_DONE,         // U1 written (buffer A)
        E1B_DONE,         // T2 written (buffer B)
        DX_FULL,          // dX accumulator ready; U1 consumed (buffer A free)
        DX_FREE,          // dX accumulator read out
        DC_DONE,          // dC MMAs done: T2 consumed (buffer B free), G consumed
        U2_DONE,          // U2 written; Ua, Ub, T accumulators fully read out
        XT_DONE,          // X^T written
        DB_DONE,          // dB MMAs done: buffers A and B free
        DRAIN,
        NBARS
    };
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + NBARS);
    const Abort ab{reinterpret_cast<volatile int *>(tmem_slot + 1), args.device_error};
    auto bar = [&](int i) { return smem_u32(bars + i); };
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

    // ---------------- set-up ----------------
    if (threadIdx.x == 0) {
        mbar_init(bar(G_FULL), 1);
        mbar_init(bar(X_FULL), 1);
        mbar_init(bar(G_FREE), 1 + 4);   // dC commit + B-chain warps
        mbar_init(bar(X_FREE), 1 + 4);
        mbar_init(bar(GT_FULL), 4);
        mbar_init(bar(UT_FULL), 1);
        mbar_init(bar(E1A_DONE), 8);     // A-chain warps
        mbar_init(bar(E1B_DONE), 4);
        mbar_init(bar(DX_FULL), 1);
        mbar_init(bar(DX_FREE), 4);
        mbar_init(bar(DC_DONE), 1);
        mbar_init(bar(U2_DONE), 8);
        mbar_init(bar(XT_DONE), 4);
        mbar_init(bar(DB_DONE), 1);
        mbar_init(bar(DRAIN), 1);
        *ab.flag = 0;
        mbar_init_fence();
        prefetch_tmap(&tmap_g);
        prefetch_tmap(&tmap_x);
    }
    if (warp == 1) tmem_alloc(smem_u32(tmem_slot), Cfg::TM_COLS);
    // factors: C[(i,a)][c] = S[a][c] A_i[a][c]; Bt[(i,k)][j] = B_i[j][k]; Bdx[j][(i,k)] = B_i[j][k]
    for (int e = threadIdx.x; e < 128 * (Q / VPC); e += blockDim.x) {
        const int row = e / (Q / VPC), c0 = (e % (Q / VPC)) * VPC;
        const int i = row / P, a = row % P;
        float v[8];
#pragma unroll
        for (int t = 0; t < VPC; ++t)
            v[t] = bld<T>(args.S, (size_t)a * Q + c0 + t) * bld<T>(args.A, ((size_t)i * P + a) * Q + c0 + t);
        st16v<T>(sC + koff(row, c0 * E, 128, Cfg::SWC), v);
    }
    for (int e = threadIdx.x; e < 128 * (M1 / VPC); e += blockDim.x) {
        const int row = e / (M1 / VPC), j0 = (e % (M1 / VPC)) * VPC;
        const int i = row / M2, k = row % M2;
        float v[8];
#pragma unroll
        for (int t = 0; t < VPC; ++t) v[t] = bld<T>(args.B, ((size_t)i * M1 + j0 + t) * M2 + k);
        st16v<T>(sBT + koff(row, j0 * E, 128, Cfg::SWJ), v);
    }
    for (int e = threadIdx.x; e < M1 * (128 / VPC); e += blockDim.x) {
        const int j = e / (128 / VPC), ik0 = (e % (128 / VPC)) * VPC;
        const int i = ik0 / M2, k0 = ik0 % M2;
        float v[8];
#pragma unroll
        for (int t = 0; t < VPC; ++t) v[t] = bld<T>(args.B, ((size_t)i * M1 + j) * M2 + k0 + t);
        st16v<T>(sBD + koff(j, ik0 * E, M1, Cfg::SW128), v);
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    const int t0 = blockIdx.x * args.tiles_per_part;
    const int t1 = imin(t0 + args.tiles_per_part, args.num_tiles);
    const int nt = t1 > t0 ? t1 - t0 : 0;

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            int issued = 0;
            for (int u = 0; u < nt; ++u) {
                const uint32_t ph = u & 1;
                const int tile = t0 + u;
                if (!mbar_wait(bar(G_FREE), ph ^ 1, ab)) break;
                mbar_arrive_expect_tx(bar(G_FULL), NT * Q * M2 * E);
                tma_load_2d(sG, &tmap_g, 0, tile * NT * Q, bar(G_FULL));
                if (!mbar_wait(bar(X_FREE), ph ^ 1, ab)) break;
                mbar_arrive_expect_tx(bar(X_FULL), Cfg::TILE_X);
                tma_load_2d(sX, &tmap_x, 0, tile * NT * P, bar(X_FULL));
                issued = u + 1;
            }
            if (issued > 0) {
                mbar_wait_drain(bar(G_FULL), (issued - 1) & 1);
                mbar_wait_drain(bar(X_FULL), (issued - 1) & 1);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer (whole warp; one elected lane issues) ----------------
        auto mma = [&](uint32_t d, uint32_t a, int swa, uint32_t b, int swb, uint32_t id, uint32_t acc) {
            mma_ss<BE<T>::tf32>(d, sdesc_kmajor(a, swa), sdesc_kmajor(b, swb), id, acc);
        };
        // Ua, Ub and T of the current tile
        auto issue_ut = [&]() {
            if (elect_one()) {
#pragma unroll
                for (int kb = 0; kb < Q * E; kb += 32) {
                    const int ch = kb / Cfg::SWC, in = kb % Cfg::SWC;
                    mma(tmem + Cfg::TM_UA, sC + ch * 128 * Cfg::SWC + in, Cfg::SWC,
                        sGT + ch * 128 * Cfg::SWC + in, Cfg::SWC, Cfg::ID_128, kb > 0);
                    mma(tmem + Cfg::TM_UB, sGT + ch * 128 * Cfg::SWC + in, Cfg::SWC,
                        sC + ch * 128 * Cfg::SWC + in, Cfg::SWC, Cfg::ID_128, kb > 0);
                }
#pragma unroll
                for (int kb = 0; kb < M1 * E; kb += 32) {
                    const int ch = kb / Cfg::SWJ, in = kb % Cfg::SWJ;
                    mma(tmem + Cfg::TM_T, sX + ch * 128 * Cfg::SWJ + in, Cfg::SWJ,
                        sBT + ch * 128 * Cfg::SWJ + in, Cfg::SWJ, Cfg::ID_128, kb > 0);
                }
                mma_commit(bar(UT_FULL));
                mma_commit(bar(X_FREE));
            }
            __syncwarp();
        };
        bool ok = true;
        if (nt > 0) {
            ok = warp_wait(bar(X_FULL), 0, ab) && warp_wait(bar(GT_FULL), 0, ab);
            if (ok) {
                tc_fence_after();
                issue_ut();
            }
        }
        for (int u = 0; u < nt && ok; ++u) {
            const uint32_t ph = u & 1;
            // dX(u) = U1 . Bdx^T  (K = (i,k)); dC(u) += T2 . G^T (K = (n,k))
            if (!warp_wait(bar(E1A_DONE), ph, ab) || !warp_wait(bar(DX_FREE), ph ^ 1, ab)) break;
            tc_fence_after();
            if (elect_one()) {
#pragma unroll
                for (int kb = 0; kb < 128 * E; kb += 32) {
                    const int ch = kb / 128, in = kb % 128;
                    mma(tmem + Cfg::TM_DX, sA + ch * 128 * 128 + in, 128, sBD + ch * M1 * 128 + in, 128,
                        Cfg::ID_M1, kb > 0);
                }
                mma_commit(bar(DX_FULL));
            }
            __syncwarp();
            if (!warp_wait(bar(E1B_DONE), ph, ab)) break;
            tc_fence_after();
            if (elect_one()) {
#pragma unroll
                for (int kb = 0; kb < 128 * E; kb += 32) {
                    const int ch = kb / 128, in = kb % 128;                // T2: 128-byte chunks
                    const int chg = kb / Cfg::SWG, ing = kb % Cfg::SWG;    // G: one chunk per n
                    mma(tmem + Cfg::TM_DC, sBb + ch * 128 * 128 + in, 128,
                        sG + chg * Q * Cfg::SWG + ing, Cfg::SWG, Cfg::ID_Q, (u > 0 || kb > 0) ? 1u : 0u);
                }
                mma_commit(bar(DC_DONE));
                mma_commit(bar(G_FREE));
            }
            __syncwarp();
            // dB(u) += U2 . X^T^T (K = (n,a)) once U2 and X^T are written
            if (!warp_wait(bar(U2_DONE), ph, ab) || !warp_wait(bar(XT_DONE), ph, ab)) break;
            tc_fence_after();
            if (elect_one()) {
#pragma unroll
                for (int kb = 0; kb < 128 * E; kb += 32) {
                    const int ch = kb / 128, in = kb % 128;
                    mma(tmem + Cfg::TM_DB, sA + ch * 128 * 128 + in, 128, sBb + ch * M1 * 128 + in, 128,
                        Cfg::ID_M1, (u > 0 || kb > 0) ? 1u : 0u);
                }
                mma_commit(bar(DB_DONE));
            }
            __syncwarp();
            // Ua, Ub, T of tile u+1 (their accumulators were read out before U2_DONE(u))
            if (u + 1 < nt) {
                if (!warp_wait(bar(X_FULL), ph ^ 1, ab) || !warp_wait(bar(GT_FULL), ph ^ 1, ab)) break;
                tc_fence_after();
                issue_ut();
            }
        }
        if (elect_one()) mma_commit(bar(DRAIN));
        __syncwarp();
        if (lane == 0) mbar_wait_drain(bar(DRAIN), 0);
        __syncwarp();
    } else if (warp < 6) {
        // ---------------- B chain (128 threads) ----------------
        const int tid = threadIdx.x - 64;
        const int quad = warp & 3;
        const int L = quad * 32 + lane;
        const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
        float dbias[Q * M2 / 128];
#pragma unroll
        for (int e = 0; e < Q * M2 / 128; ++e) dbias[e] = 0.f;
        for (int u = 0; u < nt; ++u) {
            const uint32_t ph = u & 1;
            const int64_t row0 = (int64_t)(t0 + u) * NT;
            // G^T(u) [(n,k)][c] from G(u) [(n,c)][k] (8-row register blocks), dbias partial.
            // G^T(u-1) was consumed by the U MMAs of tile u-1 (UT_FULL(u-1) preceded E1B(u-1)).
            if (!mbar_wait(bar(G_FULL), ph, ab)) break;
            for (int blk = tid; blk < NT * (Q / 8) * (M2 / VPC); blk += 128) {
                const int kb = blk % (M2 / VPC), cb = (blk / (M2 / VPC)) % (Q / 8), n = blk / ((M2 / VPC) * (Q / 8));
                uint32_t in[8][4];
#pragma unroll
                for (int t = 0; t < 8; ++t)
                    ld_shared_v4(sG + koff(n * Q + cb * 8 + t, kb * 16, NT * Q, Cfg::SWG), in[t]);
#pragma unroll
                for (int e = 0; e < VPC; ++e) {
                    const int row = n * M2 + kb * VPC + e;
                    const uint32_t lo = sGT + koff(row, cb * 8 * E, 128, Cfg::SWC);
                    store_transposed<T>(in, e, lo, lo ^ 16u);
                }
            }
#pragma unroll
            for (int e = 0; e < Q * M2 / 128; ++e) {
                const int o = tid + 128 * e, c = o / M2, k = o % M2;
                float sacc = 0.f;
                for (int n = 0; n < NT; ++n) {
                    if (row0 + n < args.N) {
                        const uint32_t a = sG + koff(n * Q + c, k * E, NT * Q, Cfg::SWG);
                        if constexpr (BE<T>::tf32) {
                            float v;
                            asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a) : "memory");
                            sacc += v;
                        } else {
                            unsigned short h;
                            asm volatile("ld.shared.b16 %0, [%1];" : "=h"(h) : "r"(a) : "memory");
                            sacc += __bfloat162float(*reinterpret_cast<__nv_bfloat16 *>(&h));
                        }
                    }
                }
                dbias[e] += sacc;
            }
            fence_proxy_async();
            mbar_arrive_warp(bar(GT_FULL));
            // T2(u) [(i,a)][(n,k)] <- T accumulator (lanes (n,a), columns (i,k)) into buffer B,
            // once dB(u-1) has consumed X^T(u-1)
            if (!mbar_wait(bar(UT_FULL), ph, ab) || !mbar_wait(bar(DB_DONE), ph ^ 1, ab)) break;
            tc_fence_after();
            {
                const int n = L / P, a = L % P;
#pragma unroll
                for (int c0 = 0; c0 < 128; c0 += 32) {   // columns (i,k): i = c0 / M2
                    const int i = c0 / M2, k0 = c0 % M2;
                    tmem_row_to_smem<T>(tmem + lane_addr + Cfg::TM_T + c0, sBb, 128, i * P + a,
                                        (n * M2 + k0) * E);
                }
            }
            tc_fence_before();
            fence_proxy_async();
            mbar_arrive_warp(bar(E1B_DONE));
            // dX(u): lanes (n,a), columns j -> dx[row0 + n][a*m1 + j] (16-byte stores)
            if (!mbar_wait(bar(DX_FULL), ph, ab)) break;
            tc_fence_after();
            {
                const int n = L / P, a = L % P;
                const int64_t row = row0 + n;
#pragma unroll
                for (int j0 = 0; j0 < M1; j0 += 32) {
                    uint32_t r[32];
                    tmem_load32(tmem + lane_addr + Cfg::TM_DX + j0, r);
                    if (j0 + 32 >= M1) {
                        tc_fence_before();
                        mbar_arrive_warp(bar(DX_FREE));
                    }
                    if (args.dX && row < args.N) {
                        if constexpr (BE<T>::tf32) {
                            float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(args.dX) +
                                                                     (size_t)row * (P * M1) + (size_t)a * M1 + j0);
#pragma unroll
                            for (int q4 = 0; q4 < 8; ++q4)
                                dst[q4] = make_float4(__uint_as_float(r[4 * q4]), __uint_as_float(r[4 * q4 + 1]),
                                                      __uint_as_float(r[4 * q4 + 2]), __uint_as_float(r[4 * q4 + 3]));
                        } else {
                            uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(args.dX) +
                                                                   (size_t)row * (P * M1) + (size_t)a * M1 + j0);
#pragma unroll
                            for (int q8 = 0; q8 < 4; ++q8)
                                dst[q8] = make_uint4(
                                    pack_bf16x2(__uint_as_float(r[8 * q8]), __uint_as_float(r[8 * q8 + 1])),
                                    pack_bf16x2(__uint_as_float(r[8 * q8 + 2]), __uint_as_float(r[8 * q8 + 3])),
                                    pack_bf16x2(__uint_as_float(r[8 * q8 + 4]), __uint_as_float(r[8 * q8 + 5])),
                                    pack_bf16x2(__uint_as_float(r[8 * q8 + 6]), __uint_as_float(r[8 * q8 + 7])));
                        }
                    }
                }
            }
            // X^T(u) [j][(n,a)] into buffer B once dC(u) has consumed T2(u)
            if (!mbar_wait(bar(DC_DONE), ph, ab)) break;
            for (int blk = tid; blk < NT * (P / 8) * (M1 / VPC); blk += 128) {
                const int jb = blk % (M1 / VPC), ab8 = (blk / (M1 / VPC)) % (P / 8), n = blk / ((M1 / VPC) * (P / 8));
                uint32_t in[8][4];
#pragma unroll
                for (int t = 0; t < 8; ++t)
                    ld_shared_v4(sX + koff(n * P + ab8 * 8 + t, jb * 16, 128, Cfg::SWJ), in[t]);
#pragma unroll
                for (int e = 0; e < VPC; ++e) {
                    const int j = jb * VPC + e;
                    const uint32_t lo = sBb + koff(j, (n * P + ab8 * 8) * E, M1, 128);
                    store_transposed<T>(in, e, lo, lo ^ 16u);
                }
            }
            fence_proxy_async();
            mbar_arrive_warp(bar(XT_DONE));
            mbar_arrive_warp(bar(X_FREE));
            mbar_arrive_warp(bar(G_FREE));
        }
        const size_t off = (size_t)R * P * Q + (size_t)R * M1 * M2;
        float *part = args.ws + (size_t)blockIdx.x * args.ws_stride;
#pragma unroll
        for (int e = 0; e < Q * M2 / 128; ++e) part[off + tid + 128 * e] = dbias[e];
    } else {
        // ---------------- A chain (256 threads) ----------------
        const int half = (warp - 6) / 4;
        const int quad = warp & 3;
        const int L = quad * 32 + lane;
        const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
        for (int u = 0; u < nt; ++u) {
            const uint32_t ph = u & 1;
            // U1(u) [(n,a)][(i,k)] <- Ua (lanes (i,a), columns (n,k)) into buffer A, once
            // dB(u-1) has consumed U2(u-1)
            if (!mbar_wait(bar(UT_FULL), ph, ab) || !mbar_wait(bar(DB_DONE), ph ^ 1, ab)) break;
            tc_fence_after();
            {
                const int i = L / P, a = L % P;
#pragma unroll
                for (int c0 = half * 64; c0 < half * 64 + 64; c0 += 32) {   // columns (n,k)
                    const int n = c0 / M2, k0 = c0 % M2;
                    tmem_row_to_smem<T>(tmem + lane_addr + Cfg::TM_UA + c0, sA, 128, n * P + a,
                                        (i * M2 + k0) * E);
                }
            }
            tc_fence_before();
            fence_proxy_async();
            mbar_arrive_warp(bar(E1A_DONE));
            // U2(u) [(i,k)][(n,a)] <- Ub (lanes (n,k), columns (i,a)) into buffer A, once
            // dX(u) has consumed U1(u)
            if (!mbar_wait(bar(DX_FULL), ph, ab)) break;
            tc_fence_after();
            {
                const int n = L / M2, k = L % M2;
#pragma unroll
                for (int c0 = half * 64; c0 < half * 64 + 64; c0 += 32) {   // columns (i,a)
                    const int i = c0 / P, a0 = c0 % P;
                    tmem_row_to_smem<T>(tmem + lane_addr + Cfg::TM_UB + c0, sA, 128, i * M2 + k,
                                        (n * P + a0) * E);
                }
            }
            tc_fence_before();
            fence_proxy_async();
            mbar_arrive_warp(bar(U2_DONE));
        }
        // dC and dB partials of this row range, after the last dB MMAs
        float *part = args.ws + (size_t)blockIdx.x * args.ws_stride;
        if (nt > 0 && mbar_wait(bar(DB_DONE), (nt - 1) & 1, ab)) {
            tc_fence_after();
            if (half == 0) {   // dC: lanes (i,a), columns c -> dC_i[a][c] (16-byte stores)
                const int i = L / P, a = L % P;
                for (int c0 = 0; c0 < Q; c0 += 32) {
                    uint32_t r[32];
                    tmem_load32(tmem + lane_addr + Cfg::TM_DC + c0, r);
                    float4 *dst = reinterpret_cast<float4 *>(part + (size_t)i * P * Q + (size_t)a * Q + c0);
#pragma unroll
                    for (int q4 = 0; q4 < 8; ++q4)
                        dst[q4] = make_float4(__uint_as_float(r[4 * q4]), __uint_as_float(r[4 * q4 + 1]),
                                              __uint_as_float(r[4 * q4 + 2]), __uint_as_float(r[4 * q4 + 3]));
                }
            } else {           // dB: lanes (i,k), columns j -> dB_i[j][k]
                const int i = L / M2, k = L % M2;
                for (int j0 = 0; j0 < M1; j0 += 32) {
                    uint32_t r[32];
                    tmem_load32(tmem + lane_addr + Cfg::TM_DB + j0, r);
#pragma unroll
                    for (int t = 0; t < 32; ++t)
                        part[(size_t)R * P * Q + (size_t)i * M1 * M2 + (size_t)(j0 + t) * M2 + k] =
                            __uint_as_float(r[t]);
                }
            }
        } else if (nt == 0) {
            for (int e = threadIdx.x - 192; e < R * P * Q + R * M1 * M2; e += 256) part[e] = 0.f;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, Cfg::TM_COLS);
    }
}

template <class Cfg>
cudaError_t launch_bwd(const void *x, const void *S, const void *A, const void *B, const void *dY,
                       void *dX, float *ws, int parts, const Shape &s, cudaStream_t st) {
    using T = typename Cfg::T;
    const bool bf16 = !BE<T>::tf32;
    CUtensorMap tg, tx;
    launch_step() = "tensor map of dY";
    cudaError_t e = make_tmap_2d(&tg, dY, bf16, (uint64_t)s.N * Cfg::Q, Cfg::M2, Cfg::M2,
                                 Cfg::NT * Cfg::Q, Cfg::M2 * Cfg::E);
    if (e != cudaSuccess) return e;
    launch_step() = "tensor map of x";
    e = make_tmap_2d(&tx, x, bf16, (uint64_t)s.N * Cfg::P, Cfg::M1, Cfg::SWJ / Cfg::E,
                     Cfg::NT * Cfg::P, Cfg::SWJ);
    if (e != cudaSuccess) return e;
    launch_step() = "shared-memory attribute";
    e = cudaFuncSetAttribute(kron_bwd_tc_kernel<Cfg>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Cfg::SMEM);
    if (e != cudaSuccess) return e;
    launch_step() = "kernel launch";
    BwdTcArgs a;
    a.S = S; a.A = A; a.B = B; a.dX = dX; a.ws = ws;
    a.ws_stride = partial_stride(s);
    a.N = s.N;
    a.num_tiles = (int)((s.N + Cfg::NT - 1) / Cfg::NT);
    a.tiles_per_part = (a.num_tiles + parts - 1) / parts;
    a.device_error = device_error_ptr();
    {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)parts);
        cfg.blockDim = dim3(448);
        cfg.dynamicSmemBytes = Cfg::SMEM;
        cfg.stream = st;
        return cudaLaunchKernelEx(&cfg, kron_bwd_tc_kernel<Cfg>, tg, tx, a);
    }
}

using BwdFn = cudaError_t (*)(const void *, const void *, const void *, const void *,
                              const void *, void *, float *, int, const Shape &, cudaStream_t);
struct BwdEntry {
    int p, q, m1, m2, r;
    bool bf16;
    BwdFn fn;
};
const BwdEntry kBwdTable[] = {
    {32, 32, 32, 32, 4, false, &launch_bwd<BwdCfg<32, 32, 32, 32, 4, float>>},
    {32, 32, 32, 32, 4, true, &launch_bwd<BwdCfg<32, 32, 32, 32, 4, __nv_bfloat16>>},
};

BwdFn find_bwd(const Shape &s, bool bf16) {
    for (const auto &f : kBwdTable)
        if (f.p == s.p && f.q == s.q && f.m1 == s.m1 && f.m2 == s.m2 && f.r == s.r && f.bf16 == bf16)
            return f.fn;
    return nullptr;
}

}  // namespace
}  // namespace tc

bool tc_backward_supported(const Shape &s, bool bf16) { return tc::find_bwd(s, bf16) != nullptr; }

int tc_backward_tile_rows(const Shape &s) { return s.r; }

cudaError_t tc_backward(const void *x, const void *S, const void *A, const void *B,
                        const void *dY, void *dX, float *ws, int parts, const Shape &s,
                        bool bf16, cudaStream_t st) {
    tc::BwdFn fn = tc::find_bwd(s, bf16);
    if (!fn) return cudaErrorNotSupported;
    return fn(x, S, A, B, dY, dX, ws, parts, s, st);
}

}  // namespace kron
