// tc_fwd.cu -- forward of the Kronecker layer on the sm_100a tensor cores (tcgen05).
//
// Vec trick (page "kronecker-layer-benchmark", section "3. The vec trick without the
// loop"): per tile of NT = 128/m2 rows of x,
//   stage 1   T[(i,k),(n,a)] = sum_j B_i[j,k] X_n[a,j]        one MMA chain, M = r*m2,
//                                                             N = NT*p, K = m1
//   stage 2   Y[(n,k),c]     = sum_(i,a) T[n,a,i,k] C_i[a,c]   M = NT*m2 = 128, N = q,
//                                                             K = r*p
//   y[n, c*m2 + k] = Y[(n,k),c] + bias[c*m2 + k]
// Stage 1 is computed transposed, so each accumulator lane (i,k) holds a whole row of
// stage 2's A operand: the epilogue moves it TMEM -> registers -> shared memory with
// 16-byte stores straight into the K-major swizzled layout stage 2 reads.  That is the
// page's permute of Z, done on chip; T never reaches HBM.  Stage 1's A operand, B_all^T,
// stays in TMEM for the whole kernel.
//
// Warp roles (736 threads, one CTA per SM, persistent over tiles):
//   warp 0       TMA producer: x tiles into an S-stage ring (128B-swizzled)
//   warp 1       stage-1 MMA issuer (also owns the TMEM allocation)
//   warp 2       stage-2 MMA issuer
//   warps 3-18   epilogue 1: stage-1 accumulator -> T in shared memory; every tile is
//                handled by all 16 warps, four per TMEM lane quadrant, 32 columns each
//   warps 19-22  epilogue 2: stage-2 accumulator + bias -> y in HBM (coalesced rows)
// Both issuers run their loops as whole warps (waits and descriptors warp-uniform) and
// let one elected lane issue each burst of MMAs: a loop run by a single lane issues
// several times slower.  Each issuer waits once per tile; while one waits, the other's
// MMAs keep the tensor pipe busy.  Both accumulators are triple-buffered in TMEM; T
// rotates over TB shared-memory buffers (as many as fit beside a deep x ring), which
// sets how far epilogue 1 can run ahead of stage 2.  Every consumer takes the tiles in
// order, which keeps each mbarrier's phases in order (no test of a phase two ahead).
#include "internal.h"
#include "tc_ptx.cuh"

#include <cuda_runtime.h>

namespace kron {
namespace tc {

template <typename T> struct Elt;
template <> struct Elt<float> {
    static constexpr int bytes = 4;
    static constexpr uint32_t fmt = 2;  // TF32
    static constexpr bool tf32 = true;
};
template <> struct Elt<__nv_bfloat16> {
    static constexpr int bytes = 2;
    static constexpr uint32_t fmt = 1;  // BF16
    static constexpr bool tf32 = false;
};

constexpr int cmin(int a, int b) { return a < b ? a : b; }

constexpr int kFwdThreads = 736;

template <int P_, int Q_, int M1_, int M2_, int R_, typename T_>
struct FwdCfg {
    using T = T_;
    static constexpr int P = P_, Q = Q_, M1 = M1_, M2 = M2_, R = R_;
    static constexpr int E = Elt<T>::bytes;
    static constexpr int NT = 128 / M2;        // rows of x per tile
    static constexpr int N1 = NT * P;          // stage-1 N: (n,a)
    static constexpr int SW1 = cmin(128, M1 * E);
    static constexpr int KC1 = M1 * E / SW1;   // K-chunks of SW1 bytes along j
    static constexpr int K2B = R * P * E;      // stage-2 K in bytes: (i,a)
    static constexpr int SW2 = cmin(128, K2B);
    // shared memory (bytes, each region 1024-aligned)
    static constexpr int B2_BYTES = Q * K2B;             // C'      [c][(i,a)]
    static constexpr int X_BYTES = N1 * M1 * E;          // x tile  [(n,a)][j]
    static constexpr int T_BYTES = 128 * K2B;            // T       [(n,k)][(i,a)]
    static constexpr int BAR_BYTES = 512;
    static constexpr int SMEM_MAX = 232448;
    static constexpr int FIXED = 1024 + BAR_BYTES + B2_BYTES;
    // TS2 (TF32, r = 128/m2 = 4 rows per tile, p = m2 = 32): stage 2 reads T from TMEM.  The
    // stage-1 accumulator block of rank i and row n (lanes i*32.., columns n*32..) belongs,
    // as stage 2's A operand, at lanes n*32.., columns i*32..: the four diagonal blocks are
    // in place and the twelve others swap in pairs through a shared-memory scratch (two
    // buffers of 16 warps x 4 KB), so no T buffer is needed.
    static constexpr bool TS2 = Elt<T>::tf32 && R == NT && P == 32 && M2 == 32;
    static constexpr int SWP_BYTES = TS2 ? 2 * 16 * 4096 : 0;
    // T buffers (SS path): as many as leave room for at least 6 x stages (at most 4)
    static constexpr int TB = TS2 ? 0
                            : (SMEM_MAX - FIXED - 4 * T_BYTES) / X_BYTES >= 6 ? 4
                            : (SMEM_MAX - FIXED - 3 * T_BYTES) / X_BYTES >= 6 ? 3 : 2;
    static constexpr int STAGES =
        cmin(8, (SMEM_MAX - FIXED - SWP_BYTES - TB * T_BYTES) / X_BYTES);
    static constexpr int OFF_B2 = 0;
    static constexpr int OFF_T = OFF_B2 + B2_BYTES;
    static constexpr int OFF_X = OFF_T + TB * T_BYTES + SWP_BYTES;
    static constexpr int OFF_BAR = OFF_X + STAGES * X_BYTES;
    static constexpr int SMEM = OFF_BAR + BAR_BYTES + 1024;  // barriers + alignment slack
    // TMEM columns: D1[3] (N1 each), D2[3] (Q each), stage 1's A operand B_all^T
    // [(i,k)][j] (M1 values per lane, two per column for BF16)
    static constexpr int D1_SLOTS = 3, D2_SLOTS = 3;
    static constexpr int TM_D1 = 0, TM_D2 = D1_SLOTS * N1, TM_A1 = TM_D2 + D2_SLOTS * Q;
    static constexpr int A1_COLS = M1 * E / 4;
    static constexpr int TM_COLS_USED = TM_A1 + A1_COLS;
    static constexpr int TM_COLS = TM_COLS_USED <= 32 ? 32 : TM_COLS_USED <= 64 ? 64
                                 : TM_COLS_USED <= 128 ? 128 : TM_COLS_USED <= 256 ? 256 : 512;
    static constexpr uint32_t IDESC1 = idesc_f32acc(128, N1, Elt<T>::fmt);
    static constexpr uint32_t IDESC2 = idesc_f32acc(128, Q, Elt<T>::fmt);

    static_assert(R * M2 == 128, "stage-1 M = r*m2 must be 128");
    static_assert(128 % M2 == 0, "m2 must divide 128");
    static_assert(N1 == 128, "stage-1 N = (128/m2)*p: 128 (four 32-column epilogue chunks)");
    static_assert(Q % 32 == 0 && Q <= 256, "q must be a multiple of 32, at most 256");
    static_assert(M1 * E % 32 == 0 && (M1 * E <= 128 || M1 * E % 128 == 0), "m1 bytes");
    static_assert(A1_COLS % 8 == 0, "stage-1 A operand: whole 8-column groups");
    static_assert(K2B % 32 == 0 && (K2B <= 128 || K2B % 128 == 0), "r*p bytes");
    static_assert(P % 32 == 0 && (32 * E) <= SW2 && SW2 == 128,
                  "a 32-column TMEM chunk maps to one 128B-swizzled row of T");
    static_assert(STAGES >= 3, "x ring");
    static_assert(2 * STAGES + 2 * D1_SLOTS + 2 * (TS2 ? D1_SLOTS : TB) + 2 * D2_SLOTS + 2 + 2 <=
                      BAR_BYTES / 8,
                  "barrier region");
    static_assert(TM_COLS_USED <= 512, "TMEM budget");
    static_assert(SMEM <= SMEM_MAX, "shared memory budget");
};

struct FwdArgs {
    const void *S, *A, *B, *bias;
    void *y;
    int64_t N;
    int num_tiles;
    int *device_error;
};

// Byte offset of element (row, kbyte) of a K-major operand with `rows` rows, K split
// into chunks of `sw` bytes (chunk-major), 8-row atoms of 8*sw bytes, swizzled.
__device__ __forceinline__ uint32_t kmajor_off(int row, int kbyte, int rows, int sw) {
    const int chunk = kbyte / sw, inner = kbyte % sw;
    const uint32_t off = (uint32_t)chunk * rows * sw + (uint32_t)(row >> 3) * 8 * sw +
                         (uint32_t)(row & 7) * sw + inner;
    return swz(off, sw);
}

template <typename T>
__device__ __forceinline__ float ldf(const void *p, size_t i) {
    if constexpr (Elt<T>::tf32) return static_cast<const float *>(p)[i];
    else return __bfloat162float(static_cast<const __nv_bfloat16 *>(p)[i]);
}

// Write 16 bytes worth of operand values (4 tf32 / 8 bf16) from floats.
template <typename T>
__device__ __forceinline__ void st16(uint32_t addr, const float *v) {
    if constexpr (Elt<T>::tf32) {
        st_shared_v4(addr, f32_to_tf32(v[0]), f32_to_tf32(v[1]), f32_to_tf32(v[2]),
                     f32_to_tf32(v[3]));
    } else {
        st_shared_v4(addr, pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                     pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
    }
}

// TR = false: the layer's forward, y = x W + bias.
// TR = true:  dX = dY W^T, the same vec trick with C_i^T and B_i^T (dX_n = sum_i C_i G_n B_i^T):
//             the kernel's (p, q, m1, m2) are the layer's (q, p, m2, m1), x is dY, y is dX,
//             and the factors are read transposed while they are packed.
template <class Cfg, bool TR>
__global__ void __launch_bounds__(kFwdThreads, 1)
kron_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmap_x, FwdArgs args) {
    using T = typename Cfg::T;
    constexpr int E = Cfg::E, P = Cfg::P, Q = Cfg::Q, M1 = Cfg::M1, M2 = Cfg::M2, R = Cfg::R;
    // (TS2 has no T buffers: TB stands at 1 in the SS-path code, which TS2 never runs)
    constexpr int NT = Cfg::NT, N1 = Cfg::N1, S = Cfg::STAGES, TB = Cfg::TB > 0 ? Cfg::TB : 1;
    constexpr int D1S = Cfg::D1_SLOTS, D2S = Cfg::D2_SLOTS;
    constexpr int VPC = 16 / E;  // values per 16-byte chunk

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t sB2 = sbase + Cfg::OFF_B2, sX = sbase + Cfg::OFF_X, sT = sbase + Cfg::OFF_T;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::OFF_BAR);
    // barrier indices
    constexpr bool TS2 = Cfg::TS2;
    constexpr int NTB = TS2 ? D1S : TB;   // TS2: B_TFULL + d1 = "A operand of slot d1 ready"
    constexpr int B_XFULL = 0, B_XEMPTY = S, B_D1FULL = 2 * S, B_D1EMPTY = 2 * S + D1S,
                  B_TFULL = 2 * S + 2 * D1S, B_TEMPTY = B_TFULL + NTB, B_D2FULL = B_TFULL + 2 * NTB,
                  B_D2EMPTY = B_D2FULL + D2S, B_DRAIN = B_D2FULL + 2 * D2S, NBARS = B_DRAIN + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + NBARS);
    const Abort abort_flag{reinterpret_cast<volatile int *>(tmem_slot + 1), args.device_error};
    auto bar = [&](int i) { return smem_u32(bars + i); };

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int my_tiles = (args.num_tiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;
    // x ring load of the CTA's t-th tile (the producer's step; a stage's first use needs no wait)
    auto issue = [&](int t) {
        const int s = t % S;
        const int tile = blockIdx.x + t * gridDim.x;
        mbar_arrive_expect_tx(bar(B_XFULL + s), Cfg::X_BYTES);
#pragma unroll
        for (int kc = 0; kc < Cfg::KC1; ++kc)
            tma_load_2d(sX + s * Cfg::X_BYTES + kc * N1 * Cfg::SW1, &tmap_x, kc * (Cfg::SW1 / E),
                        tile * N1, bar(B_XFULL + s));
    };
    const int pre = my_tiles < S ? my_tiles : S;   // stages filled before the set-up below

    // ---------------- set-up: barriers, first loads, TMEM, packed factors ----------------
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(bar(B_XFULL + s), 1);
            mbar_init(bar(B_XEMPTY + s), 1);
        }
        for (int b = 0; b < D1S; ++b) {
            mbar_init(bar(B_D1FULL + b), 1);
            // SS path: the epilogue-1 warps free a slot once it is in registers; TS2: the
            // stage-2 MMAs that read it free it
            mbar_init(bar(B_D1EMPTY + b), TS2 ? 1 : 16);
        }
        for (int b = 0; b < NTB; ++b) {
            mbar_init(bar(B_TFULL + b), 16);
            mbar_init(bar(B_TEMPTY + b), 1);
        }
        for (int b = 0; b < D2S; ++b) {
            mbar_init(bar(B_D2FULL + b), 1);
            mbar_init(bar(B_D2EMPTY + b), 4);   // epilogue-2 warps
        }
        mbar_init(bar(B_DRAIN + 0), 1);
        mbar_init(bar(B_DRAIN + 1), 1);
        *abort_flag.flag = 0;
        mbar_init_fence();
        prefetch_tmap(&tmap_x);
        // the first x tiles stream in while the factors are packed (warp 0 is the producer)
        for (int t = 0; t < pre; ++t) issue(t);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), Cfg::TM_COLS);
    }
    // stage-2 B operand: C'[c][(i,a)] = S[a][c] * A_i[a][c]
    // (thread order: consecutive c for the forward, whose S and A rows run along c;
    // consecutive (i,a) chunks for the transposed factors, whose rows run along a)
    for (int e = threadIdx.x; e < Q * (R * P / VPC); e += blockDim.x) {
        const int c = TR ? e / (R * P / VPC) : e % Q;
        const int ia0 = (TR ? e % (R * P / VPC) : e / Q) * VPC;
        float v[8];
#pragma unroll
        for (int t = 0; t < VPC; ++t) {
            const int ia = ia0 + t, i = ia / P, a = ia % P;
            // C'_i[a][c] = S[a][c] A_i[a][c]; transposed: the layer's C_i[c][a] (S is q' x p')
            const size_t sa = TR ? (size_t)c * P + a : (size_t)a * Q + c;
            const size_t aa = TR ? ((size_t)i * Q + c) * P + a : ((size_t)i * P + a) * Q + c;
            v[t] = ldf<T>(args.S, sa) * ldf<T>(args.A, aa);
        }
        st16<T>(sB2 + kmajor_off(c, ia0 * E, Q, Cfg::SW2), v);
    }
    fence_proxy_async();  // generic-proxy writes of the factors -> visible to the MMA
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // stage-1 A operand in TMEM: lane (i,k) holds B_all^T[(i,k)][j] = B_i[j][k] along j
    if (warp >= 4 && warp < 8) {
        const int L = (warp & 3) * 32 + lane, i = L / M2, k = L % M2;
        const uint32_t ta = tmem + ((uint32_t)((warp & 3) * 32) << 16) + Cfg::TM_A1;
#pragma unroll
        for (int c0 = 0; c0 < Cfg::A1_COLS; c0 += 8) {
            uint32_t w[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                // B'_i[j][k]; transposed: the layer's B_i[k][j] (B_i is m2' x m1')
                auto bidx = [&](int j) {
                    return TR ? ((size_t)i * M2 + k) * M1 + j : ((size_t)i * M1 + j) * M2 + k;
                };
                if constexpr (Elt<T>::tf32) {
                    w[u] = f32_to_tf32(ldf<T>(args.B, bidx(c0 + u)));
                } else {
                    const int j = 2 * (c0 + u);
                    w[u] = pack_bf16x2(ldf<T>(args.B, bidx(j)), ldf<T>(args.B, bidx(j + 1)));
                }
            }
            tmem_store8(ta + c0, w);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            int issued = pre;
            for (int t = pre; t < my_tiles; ++t) {
                if (!mbar_wait(bar(B_XEMPTY + t % S), ((t / S) & 1) ^ 1, abort_flag)) break;
                issue(t);
                issued = t + 1;
            }
            // drain: loads still in flight complete before the CTA may exit
            for (int t = (issued > S ? issued - S : 0); t < issued; ++t)
                mbar_wait_drain(bar(B_XFULL + t % S), (t / S) & 1);
        }
    } else if (warp == 1) {
        // ---------------- stage-1 issuer: D1[(i,k)][(n,a)] = B_all^T (TMEM) . x tile ----------------
        for (int t = 0; t < my_tiles; ++t) {
            const int s = t % S, d1 = t % D1S;
            if (!warp_wait(bar(B_XFULL + s), (t / S) & 1, abort_flag) ||
                !warp_wait(bar(B_D1EMPTY + d1), ((t / D1S) & 1) ^ 1, abort_flag))
                break;
            tc_fence_after();
            if (elect_one()) {
                const uint32_t d = tmem + Cfg::TM_D1 + d1 * N1;
                const uint64_t bd0 = sdesc_kmajor(sX + s * Cfg::X_BYTES, Cfg::SW1);
#pragma unroll
                for (int kk = 0; kk < M1 * E / 32; ++kk) {
                    const int kb = kk * 32, ch = kb / Cfg::SW1, in = kb % Cfg::SW1;
                    mma_ts<Elt<T>::tf32>(d, tmem + Cfg::TM_A1 + kk * 8,
                                         desc_add(bd0, ch * N1 * Cfg::SW1 + in), Cfg::IDESC1, kk > 0);
                }
                mma_commit(bar(B_XEMPTY + s));
                mma_commit(bar(B_D1FULL + d1));
            }
            __syncwarp();
        }
        // every MMA of this issuer has completed before TMEM can be released
        if (elect_one()) mma_commit(bar(B_DRAIN + 0));
        __syncwarp();
        if (lane == 0) mbar_wait_drain(bar(B_DRAIN + 0), 0);
        __syncwarp();
    } else if (warp == 2 && TS2) {
        // ---------------- stage-2 issuer, TS2: D2[(n,k)][c] = A2 (TMEM) . C' ----------------
        const uint64_t bd0 = sdesc_kmajor(sB2, Cfg::SW2);
        for (int t = 0; t < my_tiles; ++t) {
            const int d1 = t % D1S, d2 = t % D2S;
            if (!warp_wait(bar(B_D2EMPTY + d2), ((t / D2S) & 1) ^ 1, abort_flag) ||
                !warp_wait(bar(B_TFULL + d1), (t / D1S) & 1, abort_flag))
                break;
            tc_fence_after();
            if (elect_one()) {
                const uint32_t d = tmem + Cfg::TM_D2 + d2 * Q;
#pragma unroll
                for (int kk = 0; kk < Cfg::K2B / 32; ++kk) {
                    const int kb = kk * 32, ch = kb / Cfg::SW2, in = kb % Cfg::SW2;
                    mma_ts<true>(d, tmem + Cfg::TM_D1 + d1 * N1 + kk * 8,
                                 desc_add(bd0, ch * Q * Cfg::SW2 + in), Cfg::IDESC2, kk > 0);
                }
                mma_commit(bar(B_D1EMPTY + d1));
                mma_commit(bar(B_D2FULL + d2));
            }
            __syncwarp();
        }
        if (elect_one()) mma_commit(bar(B_DRAIN + 1));
        __syncwarp();
        if (lane == 0) mbar_wait_drain(bar(B_DRAIN + 1), 0);
        __syncwarp();
    } else if (warp == 2) {
        // ---------------- stage-2 issuer: D2[(n,k)][c] = T . C' ----------------
        const uint64_t bd0 = sdesc_kmajor(sB2, Cfg::SW2);
        for (int t = 0; t < my_tiles; ++t) {
            const int b = t % TB, d2 = t % D2S;
            if (!warp_wait(bar(B_D2EMPTY + d2), ((t / D2S) & 1) ^ 1, abort_flag) ||
                !warp_wait(bar(B_TFULL + b), (t / TB) & 1, abort_flag))
                break;
            tc_fence_after();
            if (elect_one()) {
                const uint32_t d = tmem + Cfg::TM_D2 + d2 * Q;
                const uint64_t ad0 = sdesc_kmajor(sT + b * Cfg::T_BYTES, Cfg::SW2);
#pragma unroll
                for (int kk = 0; kk < Cfg::K2B / 32; ++kk) {
                    const int kb = kk * 32, ch = kb / Cfg::SW2, in = kb % Cfg::SW2;
                    mma_ss<Elt<T>::tf32>(d, desc_add(ad0, ch * 128 * Cfg::SW2 + in),
                                         desc_add(bd0, ch * Q * Cfg::SW2 + in), Cfg::IDESC2, kk > 0);
                }
                mma_commit(bar(B_TEMPTY + b));
                mma_commit(bar(B_D2FULL + d2));
            }
            __syncwarp();
        }
        if (elect_one()) mma_commit(bar(B_DRAIN + 1));
        __syncwarp();
        if (lane == 0) mbar_wait_drain(bar(B_DRAIN + 1), 0);
        __syncwarp();
    } else if (warp < 19 && TS2) {
        // ---------------- epilogue 1, TS2: swap the off-diagonal blocks in TMEM ----------------
        // warp (quadrant i, part n) holds block (i, n): lanes (i,k), columns (n, a).  It belongs
        // at lanes (n,k), columns (i, a), where warp (n, i) holds block (n, i), which belongs
        // here: the two warps exchange their blocks through the scratch and each stores the
        // other's into its own place.  Diagonal warps (i == n) have nothing to move.
        const int quad = warp & 3, part = (warp - 3) >> 2;
        const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
        const bool diag = quad == part;
        const int lo = quad < part ? quad : part, hi = quad < part ? part : quad;
        const int pair_bar = 1 + (lo == 0 ? hi - 1 : lo == 1 ? hi + 1 : 5);   // ids 1..6
        const uint32_t sswp = sT;   // the scratch sits where the T buffers would be
        const uint32_t mine = (uint32_t)(quad * 4 + part) * 4096 + (uint32_t)lane * 128;
        const uint32_t theirs = (uint32_t)(part * 4 + quad) * 4096 + (uint32_t)lane * 128;
        for (int t = 0; t < my_tiles; ++t) {
            const int d1 = t % D1S;
            const uint32_t buf = sswp + (uint32_t)(t & 1) * 16 * 4096;
            const bool ok = mbar_wait(bar(B_D1FULL + d1), (t / D1S) & 1, abort_flag);
            if (diag) {
                if (!ok) break;
                tc_fence_after();
                tc_fence_before();
                mbar_arrive_warp(bar(B_TFULL + d1));
                continue;
            }
            const uint32_t col = tmem + lane_addr + Cfg::TM_D1 + d1 * N1 + part * 32;
            if (ok) {
                tc_fence_after();
                uint32_t r[32];
                tmem_load32(col, r);
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    st_shared_v4(buf + mine + (uint32_t)((j ^ (lane & 7)) << 4), r[4 * j],
                                 r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]);
            }
            // both warps of the pair have written (or both leave: one verdict for the pair)
            if (!named_bar_and(pair_bar, 64, ok)) break;
            uint32_t v[32];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                uint32_t q4[4];
                ld_shared_v4(buf + theirs + (uint32_t)((j ^ (lane & 7)) << 4), q4);
                v[4 * j] = q4[0]; v[4 * j + 1] = q4[1]; v[4 * j + 2] = q4[2]; v[4 * j + 3] = q4[3];
            }
            tmem_store32(col, v);
            tc_fence_before();
            mbar_arrive_warp(bar(B_TFULL + d1));
        }
    } else if (warp < 19) {
        // ---------------- epilogue 1: D1 (lanes (i,k), columns (n,a)) -> T smem ----------------
        const int quad = warp & 3, part = (warp - 3) >> 2;
        const int L = quad * 32 + lane;  // (i,k)
        const int i = L / M2, k = L % M2;
        const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
        const int c0 = part * 32;        // this warp's 32 columns (n, a0 .. a0+31)
        const int n = c0 / P, a0 = c0 % P, row = n * M2 + k;
        const int kbyte0 = (i * P + a0) * E;
        const uint32_t roff = (uint32_t)(kbyte0 / Cfg::SW2) * 128 * Cfg::SW2 +
                              (uint32_t)(row >> 3) * 8 * Cfg::SW2 + (uint32_t)(row & 7) * Cfg::SW2;
        const int slot0 = (kbyte0 % Cfg::SW2) >> 4, xr = (row & 7) & (Cfg::SW2 / 16 - 1);
        for (int t = 0; t < my_tiles; ++t) {
            const int b = t % TB, d1 = t % D1S;
            if (!mbar_wait(bar(B_D1FULL + d1), (t / D1S) & 1, abort_flag)) break;
            tc_fence_after();
            uint32_t r[32];
            tmem_load32(tmem + lane_addr + Cfg::TM_D1 + d1 * N1 + c0, r);
            tc_fence_before();
            mbar_arrive_warp(bar(B_D1EMPTY + d1));
            // 32 columns (n, a0..a0+31) -> row (n,k) of T, K bytes (i*p + a0)*E onward
            if (!mbar_wait(bar(B_TEMPTY + b), ((t / TB) & 1) ^ 1, abort_flag)) break;
            const uint32_t base = sT + b * Cfg::T_BYTES + roff;
#pragma unroll
            for (int g = 0; g < 32 / VPC; ++g) {
                const uint32_t addr = base + (uint32_t)(((slot0 + g) ^ xr) << 4);
                if constexpr (Elt<T>::tf32) {
                    // fp32 bits as they are: the TF32 MMA reads the top 19 bits of each
                    // operand (as it does for the x tile, which TMA copies unchanged)
                    st_shared_v4(addr, r[4 * g], r[4 * g + 1], r[4 * g + 2], r[4 * g + 3]);
                } else {
                    st_shared_v4(addr, pack_bf16x2(__uint_as_float(r[8 * g]), __uint_as_float(r[8 * g + 1])),
                                 pack_bf16x2(__uint_as_float(r[8 * g + 2]), __uint_as_float(r[8 * g + 3])),
                                 pack_bf16x2(__uint_as_float(r[8 * g + 4]), __uint_as_float(r[8 * g + 5])),
                                 pack_bf16x2(__uint_as_float(r[8 * g + 6]), __uint_as_float(r[8 * g + 7])));
                }
            }
            fence_proxy_async();
            mbar_arrive_warp(bar(B_TFULL + b));
        }
    } else {
        // ---------------- epilogue 2: D2 (lanes (n,k), columns c) + bias -> y ----------------
        const int quad = warp & 3;
        const int L = quad * 32 + lane;  // (n,k)
        const int n = L / M2, k = L % M2;
        const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
        float bias[Q];  // this lane's bias values, kept in registers
#pragma unroll
        for (int c = 0; c < Q; ++c) bias[c] = args.bias ? ldf<T>(args.bias, (size_t)c * M2 + k) : 0.f;
        for (int t = 0; t < my_tiles; ++t) {
            const int d2 = t % D2S;
            if (!mbar_wait(bar(B_D2FULL + d2), (t / D2S) & 1, abort_flag)) break;
            tc_fence_after();
            const int64_t row = (int64_t)(blockIdx.x + t * gridDim.x) * NT + n;
#pragma unroll
            for (int c0 = 0; c0 < Q; c0 += 32) {
                uint32_t r[32];
                tmem_load32(tmem + lane_addr + Cfg::TM_D2 + d2 * Q + c0, r);
                if (c0 + 32 >= Q) {
                    tc_fence_before();
                    mbar_arrive_warp(bar(B_D2EMPTY + d2));
                }
                if (row < args.N) {
#pragma unroll
                    for (int u = 0; u < 32; ++u) {
                        const float v = __uint_as_float(r[u]) + bias[c0 + u];
                        const size_t o = (size_t)row * (Q * M2) + (size_t)(c0 + u) * M2 + k;
                        if constexpr (Elt<T>::tf32) static_cast<float *>(args.y)[o] = v;
                        else static_cast<__nv_bfloat16 *>(args.y)[o] = __float2bfloat16_rn(v);
                    }
                }
            }
        }
    }

    // ---------------- teardown ----------------
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, Cfg::TM_COLS);
    }
}

// ---------------------------------------------------------------- host side
template <class Cfg, bool TR>
cudaError_t launch_fwd(const void *x, const void *S, const void *A, const void *B,
                       const void *bias, void *y, const Shape &s, cudaStream_t st) {
    using T = typename Cfg::T;
    const bool bf16 = !Elt<T>::tf32;
    CUtensorMap tm;
    launch_step() = "tensor map of x";
    cudaError_t e = make_tmap_2d(&tm, x, bf16, (uint64_t)s.N * Cfg::P, Cfg::M1,
                                 Cfg::SW1 / Cfg::E, Cfg::N1, Cfg::SW1, false);
    if (e != cudaSuccess) return e;
    launch_step() = "shared-memory attribute";
    e = cudaFuncSetAttribute(kron_fwd_tc_kernel<Cfg, TR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Cfg::SMEM);
    if (e != cudaSuccess) return e;
    launch_step() = "kernel launch";
    FwdArgs a{S, A, B, bias, y, s.N, (int)((s.N + Cfg::NT - 1) / Cfg::NT), device_error_ptr()};
    const int grid = a.num_tiles < num_sms() ? a.num_tiles : num_sms();
    {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)grid);
        cfg.blockDim = dim3(kFwdThreads);
        cfg.dynamicSmemBytes = Cfg::SMEM;
        cfg.stream = st;
        return cudaLaunchKernelEx(&cfg, kron_fwd_tc_kernel<Cfg, TR>, tm, a);
    }
}

using FwdFn = cudaError_t (*)(const void *, const void *, const void *, const void *,
                              const void *, void *, const Shape &, cudaStream_t);

struct FwdEntry {
    int p, q, m1, m2, r;  // the kernel's shape (for TR, the layer's q, p, m2, m1)
    bool bf16, tr;
    FwdFn fn;
};

// Shapes with a compiled tensor-core forward (tr = false) and dX kernel (tr = true).
const FwdEntry kFwdTable[] = {
    {32, 32, 32, 32, 4, false, false, &launch_fwd<FwdCfg<32, 32, 32, 32, 4, float>, false>},
    {32, 32, 32, 32, 4, true, false, &launch_fwd<FwdCfg<32, 32, 32, 32, 4, __nv_bfloat16>, false>},
    {32, 32, 32, 32, 4, false, true, &launch_fwd<FwdCfg<32, 32, 32, 32, 4, float>, true>},
    {32, 32, 32, 32, 4, true, true, &launch_fwd<FwdCfg<32, 32, 32, 32, 4, __nv_bfloat16>, true>},
};

FwdFn find_fwd(const Shape &s, bool bf16, bool tr) {
    for (const auto &f : kFwdTable)
        if (f.p == s.p && f.q == s.q && f.m1 == s.m1 && f.m2 == s.m2 && f.r == s.r &&
            f.bf16 == bf16 && f.tr == tr)
            return f.fn;
    return nullptr;
}

// ---- entry points of the tuned kernels (tc_dispatch.cu chooses between kernel families) ----
bool tuned_fwd_supported(const Shape &ks, bool bf16, bool tr) {
    return find_fwd(ks, bf16, tr) != nullptr;
}

cudaError_t tuned_fwd(const void *x, const void *S, const void *A, const void *B,
                      const void *bias, void *y, const Shape &ks, bool bf16, bool tr,
                      cudaStream_t st) {
    FwdFn fn = find_fwd(ks, bf16, tr);
    if (!fn) return cudaErrorNotSupported;
    return fn(x, S, A, B, tr ? nullptr : bias, y, ks, st);
}

}  // namespace tc
}  // namespace kron
