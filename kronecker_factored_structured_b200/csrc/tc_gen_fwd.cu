// tc_gen_fwd.cu -- generic forward (and dX) of the Kronecker layer on the sm_100a tensor
// cores, for shapes other than the tutorial layer's (page "kronecker-layer-benchmark",
// section "3. The vec trick without the loop"; rectangular factors as on the page "LLM
// Compression via Kronecker Product Decomposition", section "Factor Dimensions for GPT-2").
//
// Per tile of NT = 128/m2 rows of x the vec trick runs as MB1 = ceil(r / (128/m2)) chunks,
// one per block of 128/m2 ranks:
//   stage 1 (chunk b)  T_b[(i,k),(n,a)] = sum_j B_i[j,k] X_n[a,j]     M = 128 lanes (i,k) of
//                                                                    block b, N = NT*p, K = m1
//   stage 2            Y[(n,k),c] += sum_(i in b, a) T_b[n,a,i,k] C_i[a,c]
//                                                                    M = 128, N = q, K = (i,a)
//   y[n, c*m2 + k] = Y[(n,k),c] + bias[c*m2 + k]
// Stage 1's A operand (B_all^T, one 128-lane block per chunk) stays in TMEM; the epilogue
// moves each stage-1 accumulator TMEM -> registers -> shared memory into the K-major layout
// stage 2 reads (the page's permute of Z, on chip), and stage 2 accumulates the chunks of
// a tile into one TMEM accumulator.  Within a chunk the K index of stage 2 runs over
// (a-group, i, a-in-group) with groups of 16 bytes of a values, so that one MMA K step
// covers few rows a of S: with KRON_FLAG_SKIP_ZERO_BLOCKS a K step is not issued when S is
// zero in all of the step's rows a (the m1 x m2 blocks of W at zero entries of S are zero:
// page "kronecker-layer-benchmark", introduction), and the epilogue does not store the T
// values such a step would have read.  Every MMA keeps the one shape N = q (measured: MMAs
// of mixed N, issued over runs of non-zero 16-column blocks only, ran slower than the dense
// stage).  The first K step of every tile is always issued, which also clears the
// accumulator (the T values it reads where C' is zero may be stale, and meet zeros).  A
// per-16-column-block mask (bit cb of a K step's word) is kept for that reason only as the
// test of a K step's word against zero.
//
// TR = true computes dX = dY W^T with the same kernel: dX_n = sum_i C_i G_n B_i^T is the
// vec trick with C_i^T and B_i^T, so the kernel's (p, q, m1, m2) are the layer's
// (q, p, m2, m1) and the factors are read transposed while they are packed.
//
// Warp roles (736 threads, one CTA per SM, persistent over tiles), as in tc_fwd.cu:
//   warp 0       TMA producer: x tiles into an S-stage ring
//   warp 1       stage-1 MMA issuer (owns the TMEM allocation)
//   warp 2       stage-2 MMA issuer
//   warps 3..     epilogue 1: stage-1 accumulator -> T chunk in shared memory (E1W warps)
//   ..22          epilogue 2: stage-2 accumulator + bias -> y (E2W = 20 - E1W warps)
// The twenty epilogue warps are split by the shape.  Epilogue 2 stores y with one scalar
// store per value and sets the pace of most shapes (a per-role trace: it is busy ~90% of
// each tile's time), so it gets two warps per TMEM lane quadrant, each over half of the q
// columns, unless epilogue 1 needs all four of its warps per quadrant (a D1 slot of four
// or eight 32-column groups); epilogue 1 takes the other 12 or 16 warps.
#include "internal.h"
#include "tc_gen_common.cuh"

#include <cuda_runtime.h>

#include <type_traits>

namespace kron {
namespace tc {
namespace gen {

constexpr int kGFwdThreads = 736;

template <int P_, int Q_, int M1_, int M2_, int R_, typename T_>
struct GFwdCfg {
    using T = T_;
    static constexpr int P = P_, Q = Q_, M1 = M1_, M2 = M2_, R = R_;
    static constexpr int E = GE<T>::bytes;
    static constexpr int KSTEP = 32 / E;         // K values per MMA (32 bytes)
    static constexpr int VPC = 16 / E;           // values per 16-byte store
    static constexpr int AG = VPC;               // a values per K group
    static constexpr int IPB = 128 / M2;         // ranks per stage-1 block (chunk)
    static constexpr int IPBE = gmin(IPB, R);    // ranks laid out in a chunk's K range
    static constexpr int MB1 = cdiv(R, IPB);     // chunks per tile
    static constexpr int NT = 128 / M2;          // rows per tile (stage-2 M = 128)
    static constexpr int N1 = NT * P, N1P = up(N1, 16), N1S = up(N1P, 32);
    static constexpr int SW1 = gmin(128, M1 * E), KC1 = M1 * E / SW1;
    static constexpr int K1STEPS = M1 * E / 32;
    static constexpr int K2 = IPBE * P, K2P = up(K2, KSTEP), KS2 = K2P / KSTEP;
    static constexpr int KC2 = cdiv(K2P * E, 128);
    static constexpr int QP = up(Q, 16), QS = up(QP, 32), NCB = QP / 16;
    // shared memory (byte offsets from a 1024-aligned base)
    static constexpr int CP_BLK = KC2 * QP * 128;          // C'_b [kc][c][128 B]
    static constexpr int CP_BYTES = up(MB1 * CP_BLK, 1024);
    static constexpr int X_TMA = N1P * M1 * E;             // bytes one tile's TMA brings
    static constexpr int X_BYTES = up(X_TMA, 1024);
    static constexpr int TC_BYTES = KC2 * 128 * 128;       // one T chunk [kc][(n,k)][128 B]
    static constexpr int MASK_BYTES = up(MB1 * KS2 * 4, 16);
    static constexpr int BAR_BYTES = 512;
    static constexpr int SMEM_MAX = 232448;
    static constexpr int FIXED = 1024 + BAR_BYTES + CP_BYTES + MASK_BYTES;
    static constexpr int TBC = (SMEM_MAX - FIXED - 3 * TC_BYTES) / X_BYTES >= 4 ? 3 : 2;
    static constexpr int STAGES = gmin(8, (SMEM_MAX - FIXED - TBC * TC_BYTES) / X_BYTES);
    static constexpr int OFF_CP = 0;
    static constexpr int OFF_T = CP_BYTES;
    static constexpr int OFF_X = OFF_T + TBC * TC_BYTES;
    static constexpr int OFF_MASK = OFF_X + STAGES * X_BYTES;
    static constexpr int OFF_BAR = OFF_MASK + MASK_BYTES;
    static constexpr int SMEM = OFF_BAR + BAR_BYTES + 1024;
    // TMEM columns: B_all^T blocks, then the D1 and D2 accumulator slots
    static constexpr int A1C = M1 * E / 4;
    static constexpr int TM_A1 = 0, A1T = up(MB1 * A1C, 32);
    static constexpr bool fits(int d1, int d2) { return A1T + d1 * N1S + d2 * QS <= 512; }
    static constexpr int D1S = fits(3, 3) ? 3 : 2;
    static constexpr int D2S = fits(D1S, 3) ? 3 : 2;
    static constexpr int TM_D1 = A1T, TM_D2 = TM_D1 + D1S * N1S;
    static constexpr int TM_COLS = tmem_cols_pow2(TM_D2 + D2S * QS);
    static constexpr uint32_t IDESC1 = idesc_f32acc(128, N1P, GE<T>::fmt);
    // epilogue warps: H warps per quadrant for epilogue 2
    static constexpr int NG1 = N1S / 32;                   // 32-column groups of a D1 slot
#ifdef KRON_GFWD_H
    static constexpr int H = KRON_GFWD_H;
#else
    static constexpr int H = NG1 % 4 == 0 ? 1 : 2;   // measured: 4 warps per quadrant were slower
#endif
    static constexpr int E2W = 4 * H, E1W = 20 - E2W, NW1 = E1W / 4;
    static constexpr int GPW = cdiv(NG1, NW1);            // D1 column groups of one warp
    static constexpr int CW2 = QS / H;                     // D2 columns of one warp
    static constexpr int LW2 = gmin(CW2, 32);              // columns per TMEM load
    // one epilogue-2 warp per quadrant over a whole number of 32-column loads: the column
    // loop is unrolled (measured: stress forward 157 -> 152 us)
    static constexpr bool E2_UNROLL = H == 1 && Q % 32 == 0;

    static_assert(128 % M2 == 0 && M2 % 16 == 0, "m2 divides 128 (stage-2 M = 128)");
    static_assert(N1P <= 256, "stage-1 N = (128/m2)*p at most 256");
    static_assert(M1 * E == 32 || M1 * E == 64 || (M1 * E) % 128 == 0, "m1 row bytes");
    static_assert(A1C % 8 == 0, "whole 8-column groups of the TMEM A operand");
    static_assert(P % VPC == 0, "rows a in whole 16-byte groups");
    static_assert(QP <= 256, "stage-2 N = q at most 256");
    static_assert(NCB <= 32, "c blocks of the skip mask");
    static_assert(STAGES >= 3, "x ring");
    static_assert(H == 1 || H == 2 || H == 4, "epilogue-2 warps per quadrant");
    static_assert(CW2 % 8 == 0 && CW2 % LW2 == 0, "epilogue-2 column shares");
    static_assert(GPW <= 2, "epilogue-1 groups per warp");
    static_assert(2 * STAGES + 2 * D1S + 2 * TBC + 2 * D2S + 2 + 2 <= BAR_BYTES / 8, "barriers");
    static_assert(fits(D1S, D2S), "TMEM budget");
    static_assert(SMEM <= SMEM_MAX, "shared memory budget");
};

struct GFwdArgs {
    const void *S, *A, *B, *bias;
    void *y;
    int64_t N;
    int num_tiles;
    int skip;
    int *device_error;
};

template <class Cfg, bool TR>
__global__ void __launch_bounds__(kGFwdThreads, 1)
kron_fwd_gen_kernel(const __grid_constant__ CUtensorMap tmap_x, GFwdArgs args) {
    using T = typename Cfg::T;
    constexpr int E = Cfg::E, P = Cfg::P, Q = Cfg::Q, M1 = Cfg::M1, M2 = Cfg::M2, R = Cfg::R;
    constexpr int NT = Cfg::NT, N1 = Cfg::N1, N1P = Cfg::N1P, N1S = Cfg::N1S;
    constexpr int S = Cfg::STAGES, TBC = Cfg::TBC, D1S = Cfg::D1S, D2S = Cfg::D2S;
    constexpr int MB1 = Cfg::MB1, IPB = Cfg::IPB, IPBE = Cfg::IPBE, AG = Cfg::AG;
    constexpr int VPC = Cfg::VPC, KS2 = Cfg::KS2, QP = Cfg::QP, QS = Cfg::QS;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t sCP = sbase + Cfg::OFF_CP, sT = sbase + Cfg::OFF_T, sX = sbase + Cfg::OFF_X;
    uint32_t *mask = reinterpret_cast<uint32_t *>(smem + Cfg::OFF_MASK);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::OFF_BAR);
    constexpr int B_XFULL = 0, B_XEMPTY = S, B_D1FULL = 2 * S, B_D1EMPTY = B_D1FULL + D1S,
                  B_TFULL = B_D1EMPTY + D1S, B_TEMPTY = B_TFULL + TBC, B_D2FULL = B_TEMPTY + TBC,
                  B_D2EMPTY = B_D2FULL + D2S, B_DRAIN = B_D2EMPTY + D2S, NBARS = B_DRAIN + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + NBARS);
    const Abort abort_flag{reinterpret_cast<volatile int *>(tmem_slot + 1), args.device_error};
    auto bar = [&](int i) { return smem_u32(bars + i); };

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int my_tiles = (args.num_tiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;
    auto issue = [&](int t) {
        const int s = t % S;
        const int tile = blockIdx.x + t * gridDim.x;
        mbar_arrive_expect_tx(bar(B_XFULL + s), Cfg::X_TMA);
#pragma unroll
        for (int kc = 0; kc < Cfg::KC1; ++kc)
            tma_load_2d(sX + s * Cfg::X_BYTES + kc * N1P * Cfg::SW1, &tmap_x, kc * (Cfg::SW1 / E),
                        tile * N1, bar(B_XFULL + s));
    };
    const int pre = my_tiles < S ? my_tiles : S;

    // ---------------- set-up ----------------
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(bar(B_XFULL + s), 1);
            mbar_init(bar(B_XEMPTY + s), 1);
        }
        for (int d = 0; d < D1S; ++d) {
            mbar_init(bar(B_D1FULL + d), 1);
            mbar_init(bar(B_D1EMPTY + d), Cfg::E1W);
        }
        for (int b = 0; b < TBC; ++b) {
            mbar_init(bar(B_TFULL + b), Cfg::E1W);
            mbar_init(bar(B_TEMPTY + b), 1);
        }
        for (int d = 0; d < D2S; ++d) {
            mbar_init(bar(B_D2FULL + d), 1);
            mbar_init(bar(B_D2EMPTY + d), Cfg::E2W);
        }
        mbar_init(bar(B_DRAIN + 0), 1);
        mbar_init(bar(B_DRAIN + 1), 1);
        *abort_flag.flag = 0;
        mbar_init_fence();
        prefetch_tmap(&tmap_x);
        for (int t = 0; t < pre; ++t) issue(t);
    }
    if (warp == 1) tmem_alloc(smem_u32(tmem_slot), Cfg::TM_COLS);
    // T chunks start at zero: K positions past the chunk's ranks are never written
    zero_smem(sT, TBC * Cfg::TC_BYTES);
    // stage-2 B operand C'_b[c][kpos] = S[a][c] A_i[a][c] for rank i = b*IPB + i_local, with
    // kpos = (a / AG) * (IPBE * AG) + i_local * AG + a % AG; zero past q, r and p.  One
    // thread builds one 16-byte chunk (VPC consecutive kpos of one c); consecutive threads
    // take the chunks whose factor reads are adjacent in memory: consecutive c (S and A
    // rows run along c), or for TR consecutive a-groups (the transposed factors run along a)
    {
        constexpr int NCH = Cfg::K2P / VPC;               // chunks per (b, c)
        constexpr int NGR = P / AG;                       // a-groups per rank
#pragma unroll 2
        for (int e = threadIdx.x; e < MB1 * QP * NCH; e += blockDim.x) {
            int b, c, kp0;
            if constexpr (!TR) {
                b = e / (NCH * QP);
                const int rem = e % (NCH * QP);
                kp0 = (rem / QP) * VPC;
                c = rem % QP;
            } else {
                b = e / (QP * NCH);
                const int rem = e % (QP * NCH);
                c = rem / NCH;
                const int ch = rem % NCH, il = ch / NGR, g = ch % NGR;
                // the chunks past IPBE * NGR are the zero padding of K (kpos >= K2)
                kp0 = ch < IPBE * NGR ? (g * IPBE + il) * AG : ch * VPC;
            }
            float v[8];
#pragma unroll
            for (int t = 0; t < VPC; ++t) {
                const int kp = kp0 + t;
                const int g = kp / (IPBE * AG), il = (kp % (IPBE * AG)) / AG;
                const int a = g * AG + kp % AG, i = b * IPB + il;
                float val = 0.f;
                if (c < Q && a < P && i < R && kp < Cfg::K2) {
                    const size_t sa = TR ? (size_t)c * P + a : (size_t)a * Q + c;
                    const size_t aa = TR ? ((size_t)i * Q + c) * P + a : ((size_t)i * P + a) * Q + c;
                    val = ld_elt<T>(args.S, sa) * ld_elt<T>(args.A, aa);
                }
                v[t] = val;
            }
            uint32_t w[4];
            if constexpr (GE<T>::tf32) {
#pragma unroll
                for (int t = 0; t < 4; ++t) w[t] = tf32_bits(v[t]);
            } else {
#pragma unroll
                for (int t = 0; t < 4; ++t) w[t] = pack_bf16x2(v[2 * t], v[2 * t + 1]);
            }
            st_shared_v4(sCP + b * Cfg::CP_BLK + kmaj(c, kp0 * E, QP, 128), w[0], w[1], w[2], w[3]);
        }
    }
    // zero-block mask: bit cb of mask[b*KS2 + ks] is set when S has a non-zero in the rows a
    // of K step ks of chunk b and the 16 columns c of block cb.  Every thread tests one
    // (chunk, K position, c block) at a time; the words start at zero.
    if (args.skip) {
        for (int e = threadIdx.x; e < MB1 * KS2; e += blockDim.x) mask[e] = 0;
        __syncthreads();
        for (int e = threadIdx.x; e < MB1 * Cfg::K2P * Cfg::NCB; e += blockDim.x) {
            const int b = e / (Cfg::K2P * Cfg::NCB), rem = e % (Cfg::K2P * Cfg::NCB);
            const int kp = rem / Cfg::NCB, cb = rem % Cfg::NCB;
            const int g = kp / (IPBE * AG), il = (kp % (IPBE * AG)) / AG;
            const int a = g * AG + kp % AG;
            if (kp >= Cfg::K2 || b * IPB + il >= R) continue;
            bool nz = false;
            for (int c = cb * 16; c < cb * 16 + 16 && c < Q; ++c)
                nz |= ld_elt<T>(args.S, TR ? (size_t)c * P + a : (size_t)a * Q + c) != 0.f;
            if (nz) atomicOr(&mask[b * KS2 + kp / Cfg::KSTEP], 1u << cb);
        }
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // stage-1 A operand in TMEM: block b, lane L = (i_local, k) holds B_i[j][k] along j.
    // Warps 3-18 (four per TMEM lane quadrant) share the (block, 8-column group) items.
    if (warp >= 3 && warp < 19) {
        const int L = (warp & 3) * 32 + lane, il = L / M2, k = L % M2;
        const uint32_t lane_addr = (uint32_t)((warp & 3) * 32) << 16;
        constexpr int NCG = Cfg::A1C / 8;
#pragma unroll 2
        for (int it = (warp - 3) >> 2; it < MB1 * NCG; it += 4) {
            const int b = it / NCG, c0 = (it % NCG) * 8;
            const int i = b * IPB + il;
            const uint32_t ta = tmem + lane_addr + Cfg::TM_A1 + b * Cfg::A1C;
            {
                uint32_t w[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    auto bv = [&](int j) {
                        if (i >= R) return 0.f;
                        return ld_elt<T>(args.B, TR ? ((size_t)i * M2 + k) * M1 + j
                                                    : ((size_t)i * M1 + j) * M2 + k);
                    };
                    if constexpr (GE<T>::tf32) w[u] = tf32_bits(bv(c0 + u));
                    else w[u] = pack_bf16x2(bv(2 * (c0 + u)), bv(2 * (c0 + u) + 1));
                }
                tmem_store8(ta + c0, w);
            }
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
            for (int t = (issued > S ? issued - S : 0); t < issued; ++t)
                mbar_wait_drain(bar(B_XFULL + t % S), (t / S) & 1);
        }
    } else if (warp == 1) {
        // ---------------- stage 1: D1 = B_all^T (TMEM, block b) . x tile ----------------
        bool ok = true;
        for (int t = 0; t < my_tiles && ok; ++t) {
            const int s = t % S;
            if (!warp_wait(bar(B_XFULL + s), (t / S) & 1, abort_flag)) break;
            const uint64_t bd0 = sdesc_kmajor(sX + s * Cfg::X_BYTES, Cfg::SW1);
            for (int b = 0; b < MB1; ++b) {
                const int u = t * MB1 + b, d1 = u % D1S;
                if (!warp_wait(bar(B_D1EMPTY + d1), ((u / D1S) & 1) ^ 1, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (elect_one()) {
                    const uint32_t d = tmem + Cfg::TM_D1 + d1 * N1S;
#pragma unroll
                    for (int kk = 0; kk < Cfg::K1STEPS; ++kk) {
                        const int kb = kk * 32, ch = kb / Cfg::SW1, in = kb % Cfg::SW1;
                        mma_ts<GE<T>::tf32>(d, tmem + Cfg::TM_A1 + b * Cfg::A1C + kk * 8,
                                            desc_add(bd0, ch * N1P * Cfg::SW1 + in), Cfg::IDESC1,
                                            kk > 0);
                    }
                    mma_commit(bar(B_D1FULL + d1));
                    if (b == MB1 - 1) mma_commit(bar(B_XEMPTY + s));
                }
                __syncwarp();
            }
        }
        if (elect_one()) mma_commit(bar(B_DRAIN + 0));
        __syncwarp();
        if (lane == 0) mbar_wait_drain(bar(B_DRAIN + 0), 0);
        __syncwarp();
    } else if (warp == 2) {
        // ---------------- stage 2: D2 += T_b . C'_b over the chunks of a tile ----------------
        // the skip mask words in registers: lane l holds words l and l + 32
        const uint32_t mw0 = args.skip && lane < MB1 * KS2 ? mask[lane] : 0u;
        const uint32_t mw1 = args.skip && lane + 32 < MB1 * KS2 ? mask[lane + 32] : 0u;
        bool ok = true;
        for (int t = 0; t < my_tiles && ok; ++t) {
            const int d2 = t % D2S;
            if (!warp_wait(bar(B_D2EMPTY + d2), ((t / D2S) & 1) ^ 1, abort_flag)) break;
            for (int b = 0; b < MB1; ++b) {
                const int u = t * MB1 + b, tb = u % TBC;
                if (!warp_wait(bar(B_TFULL + tb), (u / TBC) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                uint32_t msk[KS2];   // this chunk's mask words, warp-uniform
#pragma unroll
                for (int ks = 0; ks < KS2; ++ks) {
                    const int wdx = b * KS2 + ks;
                    msk[ks] = __shfl_sync(0xffffffffu, wdx < 32 ? mw0 : mw1, wdx & 31);
                }
                if (elect_one()) {
                    const uint32_t d = tmem + Cfg::TM_D2 + d2 * QS;
                    const uint64_t ad0 = sdesc_kmajor(sT + tb * Cfg::TC_BYTES, 128);
                    const uint64_t bd0 = sdesc_kmajor(sCP + b * Cfg::CP_BLK, 128);
#pragma unroll
                    for (int ks = 0; ks < KS2; ++ks) {
                        const int kb = ks * 32, ch = kb / 128, in = kb % 128;
                        const uint64_t ad = desc_add(ad0, ch * 128 * 128 + in);
                        const uint64_t bd = desc_add(bd0, ch * QP * 128 + in);
                        const bool first = b == 0 && ks == 0;
                        // with the skip flag, a K step whose slice of C' is zero over every
                        // column is not issued (all MMAs keep one shape)
                        if (!args.skip || first || msk[ks] != 0u)
                            mma_ss<GE<T>::tf32>(d, ad, bd, idesc_f32acc(128, QP, GE<T>::fmt),
                                                first ? 0u : 1u);
                    }
                    mma_commit(bar(B_TEMPTY + tb));
                    if (b == MB1 - 1) mma_commit(bar(B_D2FULL + d2));
                }
                __syncwarp();
            }
        }
        if (elect_one()) mma_commit(bar(B_DRAIN + 1));
        __syncwarp();
        if (lane == 0) mbar_wait_drain(bar(B_DRAIN + 1), 0);
        __syncwarp();
    } else if (warp < 3 + Cfg::E1W) {
        // ---------------- epilogue 1: D1 (lanes (i,k), columns (n,a)) -> T chunk ----------------
        constexpr int NW1 = Cfg::NW1;                 // warps per quadrant
        const int quad = warp & 3, wi = (warp - 3) >> 2;
        const int L = quad * 32 + lane, il = L / M2, k = L % M2;
        const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
        constexpr int NG = Cfg::NG1;                  // 32-column groups of a D1 slot
        constexpr int GPW = Cfg::GPW;                 // groups of one warp (at most 2)
        constexpr int SPG = 32 / VPC;                 // 16-byte stores per group
        // byte offsets (within a T chunk) of this lane's 16-byte stores, fixed for the kernel:
        // column c = (n, a) of lane (i_local, k) goes to row (n, k), K position
        // (a / AG) * (IPBE * AG) + i_local * AG + a % AG; 0xFFFFFFFF marks a column past N1
        uint32_t soff[GPW][SPG];
        uint8_t sks[GPW][SPG];                        // K step of each store
#pragma unroll
        for (int gi = 0; gi < GPW; ++gi) {
#pragma unroll
            for (int g = 0; g < SPG; ++g) {
                const int c = (wi + NW1 * gi) * 32 + g * VPC;
                const int n = c / P, a = c % P;
                const int kp = (a / AG) * (IPBE * AG) + il * AG + a % AG;
                soff[gi][g] = c < N1 ? kmaj(n * M2 + k, kp * E, 128, 128) : 0xFFFFFFFFu;
                sks[gi][g] = (uint8_t)(kp / Cfg::KSTEP);
            }
        }
        // with the skip flag, bit (b*GPW + gi)*SPG + g says whether store (gi, g) of chunk b
        // feeds a K step that stage 2 issues
        static_assert(MB1 * GPW * SPG <= 64, "live bits");
        uint64_t keep = ~0ull;
        if (args.skip) {
            keep = 0;
#pragma unroll
            for (int b = 0; b < MB1; ++b)
#pragma unroll
                for (int gi = 0; gi < GPW; ++gi)
#pragma unroll
                    for (int g = 0; g < SPG; ++g)
                        if (mask[b * KS2 + sks[gi][g]] != 0u)
                            keep |= 1ull << ((b * GPW + gi) * SPG + g);
        }
        bool ok = true;
        for (int t = 0; t < my_tiles && ok; ++t) {
            for (int b = 0; b < MB1; ++b) {
                const int u = t * MB1 + b, d1 = u % D1S, tb = u % TBC;
                if (!mbar_wait(bar(B_D1FULL + d1), (u / D1S) & 1, abort_flag) ||
                    !mbar_wait(bar(B_TEMPTY + tb), ((u / TBC) & 1) ^ 1, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const bool live = il < IPBE && b * IPB + il < R;
                const uint32_t tbase = sT + tb * Cfg::TC_BYTES;
                if (wi >= NG) {   // no columns for this warp
                    tc_fence_before();
                    mbar_arrive_warp(bar(B_D1EMPTY + d1));
                }
#pragma unroll
                for (int gi = 0; gi < GPW; ++gi) {
                    const int cg = wi + NW1 * gi;
                    if (cg < NG) {
                        uint32_t r[32];
                        tmem_load32(tmem + lane_addr + Cfg::TM_D1 + d1 * N1S + cg * 32, r);
                        if (cg + NW1 >= NG) {
                            tc_fence_before();
                            mbar_arrive_warp(bar(B_D1EMPTY + d1));
                        }
                        if (live) {
#pragma unroll
                            for (int g = 0; g < SPG; ++g) {
                                // with the skip flag, T values whose K step multiplies an
                                // all-zero slice of C' are never used: their store is dropped
                                if (soff[gi][g] != 0xFFFFFFFFu &&
                                    ((keep >> ((b * GPW + gi) * SPG + g)) & 1ull))
                                    st_op16<T>(tbase + soff[gi][g], &r[g * VPC]);
                            }
                        }
                    }
                }
                fence_proxy_async();
                mbar_arrive_warp(bar(B_TFULL + tb));
            }
        }
    } else {
        // ---------------- epilogue 2: D2 (lanes (n,k), columns c) + bias -> y ----------------
        // warp HF of its quadrant takes columns [HF * CW2, (HF + 1) * CW2).  The loop is
        // compiled per HF: with compile-time column bounds the tail tests and store offsets
        // fold away (a run-time bound measured about three times slower).
        constexpr int CW2 = Cfg::CW2, LW2 = Cfg::LW2;
        const int quad = warp & 3, hf = (warp - 3 - Cfg::E1W) >> 2;
        const int L = quad * 32 + lane, n = L / M2, k = L % M2;
        const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
        // bias values of this lane (c*m2 + k), read through the non-coherent path in batches
        // that precede the y stores of the batch (so no load waits on an earlier store)
        const unsigned short *bias16 = static_cast<const unsigned short *>(args.bias);
        const float *bias32 = static_cast<const float *>(args.bias);
        auto run = [&](auto hf_const) {
            constexpr int HF = decltype(hf_const)::value;
            for (int t = 0; t < my_tiles; ++t) {
                const int d2 = t % D2S;
                if (!mbar_wait(bar(B_D2FULL + d2), (t / D2S) & 1, abort_flag)) break;
                tc_fence_after();
                const int64_t row = (int64_t)(blockIdx.x + t * gridDim.x) * NT + n;
                const size_t obase = (size_t)row * (Q * M2) + k;
                // the column loop: unrolled over the q real columns with one warp per quadrant
                // (E2_UNROLL), else a loop over this warp's share, padding columns skipped
                constexpr int C_END = Cfg::E2_UNROLL ? Q : (HF + 1) * CW2;
#pragma unroll(Cfg::E2_UNROLL ? 8 : 1)
                for (int c0 = HF * CW2; c0 < C_END; c0 += LW2) {
                    uint32_t r[LW2];
                    tmem_load_n<LW2>(tmem + lane_addr + Cfg::TM_D2 + d2 * QS + c0, r);
                    if (c0 + LW2 >= C_END) {
                        tc_fence_before();
                        mbar_arrive_warp(bar(B_D2EMPTY + d2));
                    }
                    if (row < args.N) {
#pragma unroll
                        for (int u0 = 0; u0 < LW2; u0 += 8) {
                            float bv[8];
#pragma unroll
                            for (int u = 0; u < 8; ++u) {
                                const int c = c0 + u0 + u;
                                bv[u] = 0.f;
                                if (args.bias && c < Q) {
                                    if constexpr (GE<T>::tf32) bv[u] = __ldg(bias32 + (size_t)c * M2 + k);
                                    else bv[u] = __bfloat162float(__ushort_as_bfloat16(
                                             __ldg(bias16 + (size_t)c * M2 + k)));
                                }
                            }
#pragma unroll
                            for (int u = 0; u < 8; ++u) {
                                const int c = c0 + u0 + u;
                                if (c < Q) {
                                    const float v = __uint_as_float(r[u0 + u]) + bv[u];
                                    const size_t o = obase + (size_t)c * M2;
                                    if constexpr (GE<T>::tf32) static_cast<float *>(args.y)[o] = v;
                                    else static_cast<__nv_bfloat16 *>(args.y)[o] = __float2bfloat16_rn(v);
                                }
                            }
                        }
                    }
                }
            }
        };
        if (hf == 0) run(std::integral_constant<int, 0>{});
        if constexpr (Cfg::H >= 2) {
            if (hf == 1) run(std::integral_constant<int, 1>{});
        }
        if constexpr (Cfg::H == 4) {
            if (hf == 2) run(std::integral_constant<int, 2>{});
            if (hf == 3) run(std::integral_constant<int, 3>{});
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

template <class Cfg, bool TR>
cudaError_t launch_gfwd(const void *x, const void *S, const void *A, const void *B,
                        const void *bias, void *y, const Shape &s, bool skip, cudaStream_t st) {
    using T = typename Cfg::T;
    CUtensorMap tm;
    launch_step() = "tensor map of x";
    cudaError_t e = make_tmap_2d(&tm, x, !GE<T>::tf32, (uint64_t)s.N * Cfg::P, Cfg::M1,
                                 Cfg::SW1 / Cfg::E, Cfg::N1P, Cfg::SW1, false);
    if (e != cudaSuccess) return e;
    launch_step() = "shared-memory attribute";
    e = cudaFuncSetAttribute(kron_fwd_gen_kernel<Cfg, TR>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM);
    if (e != cudaSuccess) return e;
    launch_step() = "kernel launch";
    GFwdArgs a{S, A, B, TR ? nullptr : bias, y, s.N, (int)((s.N + Cfg::NT - 1) / Cfg::NT),
               skip ? 1 : 0, device_error_ptr()};
    const int grid = a.num_tiles < num_sms() ? a.num_tiles : num_sms();
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kGFwdThreads);
    cfg.dynamicSmemBytes = Cfg::SMEM;
    cfg.stream = st;
    return cudaLaunchKernelEx(&cfg, kron_fwd_gen_kernel<Cfg, TR>, tm, a);
}

using GFwdFn = cudaError_t (*)(const void *, const void *, const void *, const void *,
                               const void *, void *, const Shape &, bool, cudaStream_t);
struct GFwdEntry {
    int p, q, m1, m2, r;   // the kernel's shape (for dX the layer's q, p, m2, m1)
    bool bf16, tr;
    GFwdFn fn;
};

#define KRON_GFWD(P, Q, M1, M2, R, T, BF)                                              \
    {P, Q, M1, M2, R, BF, false, &launch_gfwd<GFwdCfg<P, Q, M1, M2, R, T>, false>},   \
    {P, Q, M1, M2, R, BF, true, &launch_gfwd<GFwdCfg<P, Q, M1, M2, R, T>, true>}

// Kernel shapes compiled for the generic path: the GPT-2 small FFN shapes (c_fc 768 -> 3072
// with C_i 24 x 48 and B_i 32 x 64, c_proj the transpose; each one is also the other's dX
// shape) at r = 1 and 4, the 4096^2 stress layer (m = 64, r = 8) in BF16, and the block-size
// sweep's 64 x 64 and 128 x 128 blocks in TF32.
const GFwdEntry kGFwdTable[] = {
    KRON_GFWD(24, 48, 32, 64, 1, __nv_bfloat16, true),
    KRON_GFWD(24, 48, 32, 64, 4, __nv_bfloat16, true),
    KRON_GFWD(48, 24, 64, 32, 1, __nv_bfloat16, true),
    KRON_GFWD(48, 24, 64, 32, 4, __nv_bfloat16, true),
    KRON_GFWD(64, 64, 64, 64, 8, __nv_bfloat16, true),
    KRON_GFWD(16, 16, 64, 64, 1, float, false),
    KRON_GFWD(16, 16, 64, 64, 2, float, false),
    KRON_GFWD(16, 16, 64, 64, 8, float, false),
    KRON_GFWD(8, 8, 128, 128, 1, float, false),
    KRON_GFWD(8, 8, 128, 128, 2, float, false),
};
#undef KRON_GFWD

GFwdFn find_gfwd(const Shape &ks, bool bf16, bool tr) {
    for (const auto &f : kGFwdTable)
        if (f.p == ks.p && f.q == ks.q && f.m1 == ks.m1 && f.m2 == ks.m2 && f.r == ks.r &&
            f.bf16 == bf16 && f.tr == tr)
            return f.fn;
    return nullptr;
}

}  // namespace gen

bool generic_fwd_supported(const Shape &ks, bool bf16, bool tr) {
    return gen::find_gfwd(ks, bf16, tr) != nullptr;
}

cudaError_t generic_fwd(const void *x, const void *S, const void *A, const void *B,
                        const void *bias, void *y, const Shape &ks, bool bf16, bool tr,
                        bool skip, cudaStream_t st) {
    gen::GFwdFn fn = gen::find_gfwd(ks, bf16, tr);
    if (!fn) return cudaErrorNotSupported;
    return fn(x, S, A, B, bias, y, ks, skip, st);
}

}  // namespace tc
}  // namespace kron
