// tc_gen_pgrad.cu -- generic parameter gradients of the Kronecker layer on the sm_100a
// tensor cores, for shapes other than the tutorial layer's.
//
// Gradients of L = <G, y> (G = dY; page "kronecker-layer-benchmark", section "1. Build W,
// then multiply" leaves the backward to autograd), per tile of NT rows, for the ranks of
// one rank group (a CTA handles one contiguous row range and one group of RG ranks):
//   T [(i,k),(n,a)] = sum_j  B_i[j,k] X_n[a,j]        A = B_all^T block (TMEM), B = x tile
//   U [(i,a),(n,k)] = sum_c  C_i[a,c] G_n[c,k]        A = C_stack block (TMEM), B = G tile
//                                                     read MN-major
//   dC[(i,a),c]    += sum_(n,k) T[n,a,i,k] G_n[c,k]   A = T2 [(i,a)][(n,k)] (shared), B = G
//   dB[(i,k),j]    += sum_(n,a) U[n,a,i,k] X_n[a,j]   A = U2 [(i,k)][(n,a)] (shared), B = x tile
//                                                     read MN-major
//   dbias[c*m2+k]  += sum_n G_n[c,k]                  (rank group 0)
// T and U are recomputed from x and dY (nothing is kept from the forward).  The epilogue
// warps move them TMEM -> registers -> shared memory into the K-major layouts dC and dB
// read (T lanes (i,k) become T2 rows (i,a), U lanes (i,a) become U2 rows (i,k)).  dC and
// dB accumulate in TMEM over the CTA's rows and are written to the workspace as that row
// range's partials; after a grid barrier (cooperative launch: every CTA resident) the whole
// grid adds the ranges in a fixed order and forms dA = dC (.) S and dS = sum_i dC_i (.) A_i
// (plus l1 * sign(S) when the l1 penalty on S is fused) -- no separate reduction launch.  Splitting the ranks over groups keeps the accumulators and
// the working slots of one CTA inside the 512 TMEM columns for the larger layers; the CTAs
// of the groups of one row range are adjacent in the grid, so they stream the same rows at
// about the same time and the second and later reads of a tile mostly hit L2.
//
// Warp roles (736 threads, one CTA per SM):
//   warp 0       TMA producer: an SI-deep ring of input sets (x tile, dY tile)
//   warp 1       issuer A: T and U of tile t (two TMEM slot sets); owns TMEM
//   warp 2       issuer B: dC and dB of tile t from T2 / U2 (an SB-deep ring in shared memory)
//   warps 3-18   epilogue: T -> T2 and U -> U2 (per TMEM lane quadrant four warps share the
//                32-column groups of every block), then the partials
//   warps 19-22  the dbias column sums of the dY tiles (rank group 0)
// BF16 only: a 128-byte-swizzled BF16 tile is a valid operand both K-major and MN-major, so
// the x and dY tiles serve as they are loaded (T and dB; dC and U) with no copy.
#include "internal.h"
#include "tc_gen_common.cuh"

#include <cuda_runtime.h>

namespace kron {
namespace tc {
namespace gen {

constexpr int kGPgThreads = 736;

template <int P_, int Q_, int M1_, int M2_, int R_, typename T_, int RG_, int NT_>
struct GPgCfg {
    using T = T_;
    static constexpr int P = P_, Q = Q_, M1 = M1_, M2 = M2_, R = R_, RG = RG_, NT = NT_;
    static constexpr int E = GE<T>::bytes;
    static constexpr int KSTEP = 32 / E, VPC = 16 / E;
    static constexpr int NG = cdiv(R, RG);          // rank groups
    static constexpr int IPT = 128 / M2, MBT = cdiv(RG, IPT);   // T blocks: lanes (i,k)
    static constexpr int IPU = 128 / P, MBU = cdiv(RG, IPU);    // U blocks: lanes (i,a)
    static constexpr int NTN = up(NT * P, 16), NTS = up(NTN, 32);   // T: N = (n,a)
    static constexpr int NUN = NT * M2, NUS = up(NUN, 32);          // U: N = (n,k)
    static constexpr int QK = up(Q, KSTEP);                         // U: K = c
    static constexpr int QN = up(Q, 16), QNS = up(QN, 32);          // dC: N = c
    static constexpr int KT2 = NT * M2;                             // dC: K = (n,k)
    static constexpr int KU2 = up(NT * P, KSTEP);                   // dB: K = (n,a)
    static constexpr int M1N = up(M1, 16), M1S = up(M1N, 32);       // dB: N = j
    // input tiles
    static constexpr int XRB = M1 * E, SWX = gmin(128, XRB), KCX = XRB / SWX;
    static constexpr int GRB = M2 * E;              // dY row bytes = its swizzle width
    static constexpr int GBR = NT * Q + gmax(QN, QK) - Q;   // dY box rows (n,c) + slack
    static constexpr int KCT = cdiv(KT2 * E, 128), KCU = cdiv(KU2 * E, 128);
    static constexpr int X_BYTES = up(KCX * NTN * SWX, 1024);
    static constexpr int G_BYTES = up(GBR * GRB, 1024);
    static constexpr int TMA_BYTES = KCX * NTN * SWX + GBR * GRB;
    static constexpr int OFF_XK = 0, OFF_GK = X_BYTES;
    static constexpr int IN_BYTES = OFF_GK + G_BYTES;
    static constexpr int T2_BLK = KCT * 128 * 128, U2_BLK = KCU * 128 * 128;
    static constexpr int IB = MBU * T2_BLK + MBT * U2_BLK;
    static constexpr int BAR_BYTES = 512;
    static constexpr int SMEM_MAX = 232448;
    static constexpr int FREE = SMEM_MAX - 1024 - BAR_BYTES;
    static constexpr int SB = FREE - 3 * IB >= 4 * IN_BYTES ? 3 : 2;
    static constexpr int SI = gmin(8, (FREE - SB * IB) / IN_BYTES);
    static constexpr int OFF_IN = 0, OFF_I = SI * IN_BYTES, OFF_BAR = OFF_I + SB * IB;
    static constexpr int SMEM = OFF_BAR + BAR_BYTES + 1024;
    // TMEM columns
    static constexpr int BTC = up(M1 * E / 4, 16), CSC = up(QK * E / 4, 16);
    static constexpr int TM_BT = 0, TM_CS = up(MBT * BTC, 32);
    static constexpr int TM_DT = up(TM_CS + MBU * CSC, 32);
    static constexpr int TM_DU = TM_DT + 2 * MBT * NTS;
    static constexpr int TM_DC = TM_DU + 2 * MBU * NUS;
    static constexpr int TM_DB = TM_DC + MBU * QNS;
    static constexpr int TM_USED = TM_DB + MBT * M1S;
    static constexpr int TM_COLS = 512;
    static constexpr uint32_t ID_T = idesc_f32acc(128, NTN, GE<T>::fmt);
    static constexpr uint32_t ID_U = idesc_f32acc(128, NUN, GE<T>::fmt) | kBMajorMN;
    static constexpr uint32_t ID_DC = idesc_f32acc(128, QN, GE<T>::fmt);
    static constexpr uint32_t ID_DB = idesc_f32acc(128, M1N, GE<T>::fmt);
    static constexpr uint32_t MN_LAYOUT = layout_type(GRB);
    static constexpr uint32_t MN_SBO = 8 * GRB;
    static constexpr uint32_t XMN_LAYOUT = layout_type(SWX);
    static constexpr uint32_t ID_DBX = ID_DB | kBMajorMN;

    static_assert(128 % M2 == 0 && M2 % 16 == 0, "m2 divides 128, multiple of 16");
    static_assert(P <= 128 && P % VPC == 0, "p at most 128, whole 16-byte groups");
    static_assert(GRB == 64 || GRB == 128, "dY rows of 64 or 128 bytes (TF32: m2 = 32)");
    static_assert(!GE<T>::tf32, "generic parameter gradients: BF16 operands");
    static_assert(XRB <= 128 && NTN >= KU2, "x tile as dB's MN-major operand: one block of j");
    static_assert(Q % 8 == 0, "dY tile rows of each n start on an 8-row atom");
    static_assert(XRB == 32 || XRB == 64 || XRB % 128 == 0, "x row bytes");
    static_assert(M1 % VPC == 0, "X^T copy");
    static_assert((M1 * E / 4) % 8 == 0 && (QK * E / 4) % 8 == 0, "whole 8-column groups in TMEM");
    static_assert(NTN <= 256 && NUN <= 256 && QN <= 256 && M1N <= 256 && GBR <= 256, "MMA N / box");
    static_assert(KT2 % KSTEP == 0, "dC K steps");
    static_assert((Q * M2) % 128 == 0, "dbias: whole values per thread");
    static_assert(SI >= 2 && SB >= 2, "rings");
    static_assert(3 * SI + 4 + 2 * SB + 2 <= BAR_BYTES / 8 - 2, "barrier region");
    static_assert(TM_USED <= TM_COLS, "TMEM budget");
    static_assert(SMEM <= SMEM_MAX, "shared memory budget");
};

struct GPgArgs {
    const void *S, *A, *B;
    float *ws;
    size_t ws_stride;
    int num_tiles;
    int tiles_per_part;
    int *device_error;
    unsigned *arrived;     // grid-barrier counter, zeroed by the host before the launch
    float *dS, *dA, *dB, *dbias;
    double l1;             // weight of the penalty l1 * sum|S| whose gradient joins dS
};

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned *p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Fixed-order sum of every row range's partials, by the whole grid once all are written.
// Virtual columns: dC ordered (position (a,c), rank i) so that the r ranks of a position
// are adjacent, then dB, then dbias.  CTA b owns a run of virtual columns (a multiple of r
// long); in passes of CW columns, GS groups of threads each add ranges g = ps, ps + GS, ...
// of one column in double (four accumulators) and the group sums are added in a fixed
// order.  Only `parts` fixes the order: bitwise reproducible.  The epilogue forms
// dA_i = dC_i (.) S and dS = sum_i dC_i (.) A_i (+ l1 * sign(S)), and writes dB and dbias.
template <class Cfg>
__device__ void reduce_parts(const GPgArgs &args, int parts, double *red, double *vals) {
    using T = typename Cfg::T;
    constexpr int P = Cfg::P, Q = Cfg::Q, M1 = Cfg::M1, M2 = Cfg::M2, R = Cfg::R;
    constexpr int NDC = R * P * Q, NDB = R * M1 * M2, NB = Q * M2, NCOL = NDC + NDB + NB;
    constexpr int CW = R <= 64 ? (64 / R) * R : R;
    constexpr int GS = kGPgThreads / CW;
    const int per = ((NCOL + (int)gridDim.x * R - 1) / ((int)gridDim.x * R)) * R;
    const int v0 = (int)blockIdx.x * per, v1 = gmin(v0 + per, NCOL);
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
                    const double sv = (double)ld_elt<T>(args.S, pos);
                    double ds = 0.0;
                    for (int i = 0; i < R; ++i) {
                        const double dc = vals[threadIdx.x + i];
                        args.dA[(size_t)i * P * Q + pos] = (float)(dc * sv);
                        ds += dc * (double)ld_elt<T>(args.A, (size_t)i * P * Q + pos);
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

template <class Cfg>
__global__ void __launch_bounds__(kGPgThreads, 1)
kron_pgrad_gen_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_g,
                      GPgArgs args) {
    using T = typename Cfg::T;
    constexpr int E = Cfg::E, P = Cfg::P, Q = Cfg::Q, M1 = Cfg::M1, M2 = Cfg::M2, R = Cfg::R;
    constexpr int NT = Cfg::NT, RG = Cfg::RG, NG = Cfg::NG, SI = Cfg::SI, SB = Cfg::SB;
    constexpr int MBT = Cfg::MBT, MBU = Cfg::MBU, IPT = Cfg::IPT, IPU = Cfg::IPU;
    constexpr int KSTEP = Cfg::KSTEP;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    const uint32_t sb = smem_u32(smem);
    const uint32_t sIn = sb + Cfg::OFF_IN, sI = sb + Cfg::OFF_I;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::OFF_BAR);
    constexpr int IN_FULL = 0, IN_FREE = SI, D_FULL = 2 * SI, D_EMPTY = D_FULL + 2,
                  I_FULL = D_EMPTY + 2, I_EMPTY = I_FULL + SB, DONE = I_EMPTY + SB,
                  DRAIN = DONE + 1, NBARS = DRAIN + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + NBARS);
    const Abort ab{reinterpret_cast<volatile int *>(tmem_slot + 1), args.device_error};
    auto bar = [&](int i) { return smem_u32(bars + i); };
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

    const int part = blockIdx.x / NG, grp = blockIdx.x % NG;
    const int i0 = grp * RG, rgv = gmin(RG, R - i0);    // this CTA's ranks [i0, i0 + rgv)
    const int t0 = part * args.tiles_per_part;
    const int t1 = gmin(t0 + args.tiles_per_part, args.num_tiles);
    const int nt = t1 > t0 ? t1 - t0 : 0;
    auto issue = [&](int u) {
        const int s = u % SI;
        const uint32_t dst = sIn + s * Cfg::IN_BYTES;
        const int tile = t0 + u;
        mbar_arrive_expect_tx(bar(IN_FULL + s), Cfg::TMA_BYTES);
#pragma unroll
        for (int kc = 0; kc < Cfg::KCX; ++kc)
            tma_load_2d(dst + Cfg::OFF_XK + kc * Cfg::NTN * Cfg::SWX, &tm_x, kc * (Cfg::SWX / E),
                        tile * NT * P, bar(IN_FULL + s));
        tma_load_2d(dst + Cfg::OFF_GK, &tm_g, 0, tile * NT * Q, bar(IN_FULL + s));
    };
    const int pre = gmin(SI, nt);

    // ---------------- set-up ----------------
    // everything starts at zero: the K positions past (n,a) of U2 and X^T are never written
    zero_smem(sb, Cfg::OFF_BAR);
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int s = 0; s < SI; ++s) {
            mbar_init(bar(IN_FULL + s), 1);
            mbar_init(bar(IN_FREE + s), 1 + 1 + 4);   // issuer A, issuer B, dbias warps
        }
        for (int d = 0; d < 2; ++d) {
            mbar_init(bar(D_FULL + d), 1);
            mbar_init(bar(D_EMPTY + d), 16);
        }
        for (int b = 0; b < SB; ++b) {
            mbar_init(bar(I_FULL + b), 16);
            mbar_init(bar(I_EMPTY + b), 1);
        }
        mbar_init(bar(DONE), 1);
        mbar_init(bar(DRAIN), 1);
        *ab.flag = 0;
        mbar_init_fence();
        prefetch_tmap(&tm_x);
        prefetch_tmap(&tm_g);
        for (int u = 0; u < pre; ++u) issue(u);
    }
    if (warp == 1) tmem_alloc(smem_u32(tmem_slot), Cfg::TM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // A operands in TMEM (zero for lanes past the group's ranks and for K past q):
    //   B_all^T block bt: lane (i,k) = (i0 + bt*IPT + L/m2, L%m2), column j -> B_i[j][k]
    //   C_stack block bu: lane (i,a) = (i0 + bu*IPU + L/p, L%p), column c -> S[a][c] A_i[a][c]
    // (lanes in the paired order of pair_lane_index: the epilogue stores K pairs).  Warps
    // 3-18 (four per TMEM lane quadrant) share the work: per quadrant two warps take the
    // (block, 8-column group) items of B_all^T and two those of C_stack, so that many
    // factor loads are in flight at once.
    if (warp >= 3 && warp < 19) {
        const int qd = warp & 3, L = pair_lane_index(qd * 32 + lane);
        const uint32_t lane_addr = (uint32_t)(qd * 32) << 16;
        const int sub = (warp - 3) >> 2;
        const bool is_c = sub >= 2;
        const int nblk = is_c ? MBU : MBT;
        const int ncg = (is_c ? Cfg::QK : M1) * E / 4 / 8;   // 8-column groups per block
#pragma unroll 2
        for (int it = sub & 1; it < nblk * ncg; it += 2) {
            const int blk = it / ncg, c0 = (it % ncg) * 8;
            int i, o;
            bool valid;
            if (is_c) {
                const int ir = blk * IPU + L / P;
                i = i0 + ir; o = L % P;
                valid = L < IPU * P && ir < rgv;
            } else {
                const int ir = blk * IPT + L / M2;
                i = i0 + ir; o = L % M2;
                valid = ir < rgv;
            }
            auto val = [&](int j) {
                if (!valid) return 0.f;
                if (is_c) {
                    if (j >= Q) return 0.f;
                    return ld_elt<T>(args.S, (size_t)o * Q + j) *
                           ld_elt<T>(args.A, ((size_t)i * P + o) * Q + j);
                }
                return ld_elt<T>(args.B, ((size_t)i * M1 + j) * M2 + o);
            };
            const uint32_t base = tmem + lane_addr + (is_c ? Cfg::TM_CS + blk * Cfg::CSC
                                                           : Cfg::TM_BT + blk * Cfg::BTC);
            uint32_t w[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                if constexpr (GE<T>::tf32) w[u] = tf32_bits(val(c0 + u));
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
                const uint64_t xd = sdesc_kmajor(in + Cfg::OFF_XK, Cfg::SWX);
                const uint64_t gd = sdesc_mn(in + Cfg::OFF_GK, Cfg::MN_LAYOUT, Q * Cfg::GRB,
                                             Cfg::MN_SBO);
                for (int bt = 0; bt < MBT; ++bt) {
#pragma unroll
                    for (int kk = 0; kk < M1 * E / 32; ++kk) {   // T, K = j
                        const int kb = kk * 32, ch = kb / Cfg::SWX, inb = kb % Cfg::SWX;
                        mma_ts<GE<T>::tf32>(tmem + Cfg::TM_DT + (d * MBT + bt) * Cfg::NTS,
                                            tmem + Cfg::TM_BT + bt * Cfg::BTC + kk * 8,
                                            desc_add(xd, ch * Cfg::NTN * Cfg::SWX + inb), Cfg::ID_T,
                                            kk > 0);
                    }
                }
                for (int bu = 0; bu < MBU; ++bu) {
#pragma unroll
                    for (int kk = 0; kk < Cfg::QK / KSTEP; ++kk)   // U, K = c, dY MN-major
                        mma_ts<GE<T>::tf32>(tmem + Cfg::TM_DU + (d * MBU + bu) * Cfg::NUS,
                                            tmem + Cfg::TM_CS + bu * Cfg::CSC + kk * 8,
                                            desc_add(gd, kk * KSTEP * Cfg::GRB),
                                            Cfg::ID_U, kk > 0);
                }
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
                !warp_wait(bar(IN_FULL + s), (u / SI) & 1, ab))
                break;
            tc_fence_after();
            if (elect_one()) {
                const uint32_t in = sIn + s * Cfg::IN_BYTES;
                const uint32_t ib = sI + b * Cfg::IB;
                const uint64_t gkd = sdesc_kmajor(in + Cfg::OFF_GK, Cfg::GRB);
                // the x tile as dB's B operand: N = j along its rows, K = (n,a) down them
                const uint64_t xmd = sdesc_mn(in + Cfg::OFF_XK, Cfg::XMN_LAYOUT, Cfg::NTN * Cfg::SWX,
                                              8 * Cfg::SWX);
                for (int bu = 0; bu < MBU; ++bu) {
                    const uint64_t t2d = sdesc_kmajor(ib + bu * Cfg::T2_BLK, 128);
#pragma unroll
                    for (int kk = 0; kk < Cfg::KT2 / KSTEP; ++kk) {   // dC, K = (n,k)
                        const int kb = kk * 32;
                        const int kp = kk * KSTEP, n = kp / M2, kin = (kp % M2) * E;
                        mma_ss<GE<T>::tf32>(tmem + Cfg::TM_DC + bu * Cfg::QNS,
                                            desc_add(t2d, (kb / 128) * 128 * 128 + kb % 128),
                                            desc_add(gkd, n * Q * Cfg::GRB + kin), Cfg::ID_DC,
                                            (u > 0 || kk > 0) ? 1u : 0u);
                    }
                }
                for (int bt = 0; bt < MBT; ++bt) {
                    const uint64_t u2d = sdesc_kmajor(ib + MBU * Cfg::T2_BLK + bt * Cfg::U2_BLK, 128);
#pragma unroll
                    for (int kk = 0; kk < Cfg::KU2 / KSTEP; ++kk) {   // dB, K = (n,a), x MN-major
                        const int kb = kk * 32;
                        mma_ss<GE<T>::tf32>(tmem + Cfg::TM_DB + bt * Cfg::M1S,
                                            desc_add(u2d, (kb / 128) * 128 * 128 + kb % 128),
                                            desc_add(xmd, kk * KSTEP * Cfg::SWX), Cfg::ID_DBX,
                                            (u > 0 || kk > 0) ? 1u : 0u);
                    }
                }
                mma_commit(bar(I_EMPTY + b));
                mma_commit(bar(IN_FREE + s));
            }
            __syncwarp();
        }
        if (elect_one()) mma_commit(bar(DONE));
        __syncwarp();
        if (lane == 0) mbar_wait_drain(bar(DONE), 0);
        __syncwarp();
    } else if (warp < 19) {
        // ---------------- epilogue: T -> T2, U -> U2; then the partials ----------------
        const int qd = warp & 3, wi = (warp - 3) >> 2;
        const int L = qd * 32 + lane;
        const uint32_t lane_addr = (uint32_t)(qd * 32) << 16;
        constexpr int TG = Cfg::NTS / 32, UG = Cfg::NUS / 32;    // 32-column groups per block
        constexpr int NTASK = MBT * TG + MBU * UG;
        bool ok = true;
        for (int u = 0; u < nt; ++u) {
            const int d = u & 1, b = u % SB;
            if (!mbar_wait(bar(D_FULL + d), (u >> 1) & 1, ab) ||
                !mbar_wait(bar(I_EMPTY + b), ((u / SB) & 1) ^ 1, ab)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t ib = sI + b * Cfg::IB;
#pragma unroll
            for (int task = 0; task < NTASK; ++task) {
                if ((task & 3) != wi) continue;
                const bool is_t = task < MBT * TG;
                const int blk = is_t ? task / TG : (task - MBT * TG) / UG;
                const int cg = is_t ? task % TG : (task - MBT * TG) % UG;
                const uint32_t src = tmem + (is_t ? Cfg::TM_DT + (d * MBT + blk) * Cfg::NTS
                                                  : Cfg::TM_DU + (d * MBU + blk) * Cfg::NUS) + cg * 32;
                const int CW = is_t ? P : M2;                     // columns per n: a (T), k (U)
                const int KW = is_t ? M2 : P;                     // K positions per n
                const uint32_t dstb = ib + (is_t ? 0u : (uint32_t)(MBU * Cfg::T2_BLK));
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    // this thread's K pair: M indices nat, nat + 1 of lanes g and g + 8 of
                    // the half; T: (i,k) -> T2 row (i%IPU, a), K (n,k); U: (i,a) -> U2 row
                    // (i%IPT, k), K (n,a)
                    uint32_t r[16];
                    tmem_load16x256_x4(src + ((uint32_t)(qd * 32 + 16 * h) << 16), r);
                    const int nat = qd * 32 + 16 * h + 2 * (lane >> 2);
                    const int ir = is_t ? blk * IPT + nat / M2 : blk * IPU + nat / P;
                    const int own = is_t ? nat % M2 : nat % P;
                    const bool valid = (is_t || nat < IPU * P) && ir < rgv;
                    const uint32_t dst = dstb + (is_t ? (ir / IPU) * Cfg::T2_BLK : (ir / IPT) * Cfg::U2_BLK);
                    const int rbase = is_t ? (ir % IPU) * P : (ir % IPT) * M2;   // a multiple of 8
                    if constexpr (NT == 1) {
                        // one row per tile: column c of the task is row rbase + c at the fixed K
                        // byte kb of this thread.  In the 128-byte swizzle the row's low three
                        // bits, w = 2(t%4) + dl, pick the 16-byte chunk kb/16 XOR w: two offsets
                        // per thread, and each 8-row group rp adds 1 KB.  Groups past the task's
                        // columns (c >= p or m2) are dropped at compile time.
                        const int kb = own * E;
                        const uint32_t base = dst + (uint32_t)(kb >> 7) * 128 * 128 +
                                              (uint32_t)((rbase >> 3) + cg * 4) * 1024 + (uint32_t)(kb & 15);
                        const uint32_t c16 = (uint32_t)(kb >> 4) & 7u;
                        uint32_t off[2];
#pragma unroll
                        for (int dl = 0; dl < 2; ++dl) {
                            const uint32_t w = (uint32_t)((lane & 3) * 2 + dl);
                            off[dl] = w * 128 + ((c16 ^ w) << 4);
                        }
                        if (valid) {
#pragma unroll
                            for (int rp = 0; rp < 4; ++rp) {
                                if (cg * 32 + rp * 8 >= CW) continue;
#pragma unroll
                                for (int dl = 0; dl < 2; ++dl)
                                    st_shared_u32(base + off[dl] + rp * 1024,
                                                  pack_bf16x2(__uint_as_float(r[4 * rp + dl]),
                                                              __uint_as_float(r[4 * rp + 2 + dl])));
                            }
                        }
                    } else {
#pragma unroll
                        for (int rp = 0; rp < 4; ++rp) {
#pragma unroll
                            for (int dl = 0; dl < 2; ++dl) {
                                const int c = cg * 32 + rp * 8 + (lane & 3) * 2 + dl;
                                if (valid && c < NT * CW) {
                                    const int n = c / CW, row = rbase + c % CW;
                                    st_shared_u32(dst + kmaj(row, (n * KW + own) * E, 128, 128),
                                                  pack_bf16x2(__uint_as_float(r[4 * rp + dl]),
                                                              __uint_as_float(r[4 * rp + 2 + dl])));
                                }
                            }
                        }
                    }
                }
            }
            tc_fence_before();
            mbar_arrive_warp(bar(D_EMPTY + d));
            fence_proxy_async();
            mbar_arrive_warp(bar(I_FULL + b));
        }
        // this range's partial dC_i[a][c] and dB_i[j][k] of the group's ranks
        float *pw = args.ws + (size_t)part * args.ws_stride;
        const bool ok_all = named_bar_and(1, 512, ok);
        const bool have = __all_sync(0xffffffffu, nt > 0 && ok_all && mbar_wait(bar(DONE), 0, ab));
        if (have) tc_fence_after();
        constexpr int CG = Cfg::QNS / 32, BG = Cfg::M1S / 32;
        for (int task = wi; task < MBU * CG + MBT * BG; task += 4) {
            uint32_t r[32];
            if (task < MBU * CG) {
                const int bu = task / CG, cg = task % CG;
                const int ir = bu * IPU + L / P, a = L % P;
                if (have) tmem_load32(tmem + lane_addr + Cfg::TM_DC + bu * Cfg::QNS + cg * 32, r);
                if (L < IPU * P && ir < rgv) {
                    float *dst = pw + ((size_t)(i0 + ir) * P + a) * Q;
#pragma unroll
                    for (int w = 0; w < 32; ++w)
                        if (cg * 32 + w < Q) dst[cg * 32 + w] = have ? __uint_as_float(r[w]) : 0.f;
                }
            } else {
                const int tk = task - MBU * CG, bt = tk / BG, cg = tk % BG;
                const int ir = bt * IPT + L / M2, k = L % M2;
                if (have) tmem_load32(tmem + lane_addr + Cfg::TM_DB + bt * Cfg::M1S + cg * 32, r);
                if (ir < rgv) {
                    float *dst = pw + (size_t)R * P * Q + (size_t)(i0 + ir) * M1 * M2 + k;
#pragma unroll
                    for (int w = 0; w < 32; ++w)
                        if (cg * 32 + w < M1) dst[(size_t)(cg * 32 + w) * M2] = have ? __uint_as_float(r[w]) : 0.f;
                }
            }
        }
    } else {
        // ---------------- dbias column sums of the dY tiles ----------------
        const int tid = threadIdx.x - 608;
        constexpr int PER = Q * M2 / 256;   // pairs (c, k..k+1) per thread
        static_assert((Q * M2) % 256 == 0 && M2 % 2 == 0, "dbias pairs");
        float acc[2 * PER];
#pragma unroll
        for (int e = 0; e < 2 * PER; ++e) acc[e] = 0.f;
        for (int u = 0; u < nt; ++u) {
            const int s = u % SI;
            if (!mbar_wait(bar(IN_FULL + s), (u / SI) & 1, ab)) break;
            const uint32_t in = sIn + s * Cfg::IN_BYTES;
            if (grp == 0) {
#pragma unroll
                for (int e = 0; e < PER; ++e) {
                    const int idx = 2 * (tid + 128 * e), c = idx / M2, k = idx % M2;
#pragma unroll
                    for (int n = 0; n < NT; ++n) {
                        uint32_t v;
                        asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v)
                                     : "r"(in + Cfg::OFF_GK + kmaj(n * Q + c, k * E, Cfg::GBR, Cfg::GRB))
                                     : "memory");
                        acc[2 * e] += __bfloat162float(__ushort_as_bfloat16((unsigned short)(v & 0xFFFFu)));
                        acc[2 * e + 1] += __bfloat162float(__ushort_as_bfloat16((unsigned short)(v >> 16)));
                    }
                }
            }
            mbar_arrive_warp(bar(IN_FREE + s));
        }
        if (grp == 0) {
            float *pw = args.ws + (size_t)part * args.ws_stride + (size_t)R * (P * Q + M1 * M2);
#pragma unroll
            for (int e = 0; e < PER; ++e) {
                pw[2 * (tid + 128 * e)] = acc[2 * e];
                pw[2 * (tid + 128 * e) + 1] = acc[2 * e + 1];
            }
        }
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
        double *vals = red + kGPgThreads + 64;
        reduce_parts<Cfg>(args, (int)(gridDim.x / NG), red, vals);
    }
}

template <class Cfg>
cudaError_t launch_gpgrad(const void *x, const void *S, const void *A, const void *B,
                          const void *dY, float *ws, int parts, const Shape &s, float *dS,
                          float *dA, float *dB, float *dbias, double l1, cudaStream_t st) {
    using T = typename Cfg::T;
    const bool bf16 = !GE<T>::tf32;
    CUtensorMap tx, tg;
    launch_step() = "tensor map of x";
    cudaError_t e = make_tmap_2d(&tx, x, bf16, (uint64_t)s.N * Cfg::P, Cfg::M1, Cfg::SWX / Cfg::E,
                                 Cfg::NTN, Cfg::SWX, false);
    if (e != cudaSuccess) return e;
    launch_step() = "tensor map of dY";
    e = make_tmap_2d(&tg, dY, bf16, (uint64_t)s.N * Cfg::Q, Cfg::M2, Cfg::M2, Cfg::GBR, Cfg::GRB,
                     false);
    if (e != cudaSuccess) return e;
    launch_step() = "shared-memory attribute";
    e = cudaFuncSetAttribute(kron_pgrad_gen_kernel<Cfg>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Cfg::SMEM);
    if (e != cudaSuccess) return e;
    GPgArgs a;
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
    cfg.gridDim = dim3((unsigned)(parts * Cfg::NG));
    cfg.blockDim = dim3(kGPgThreads);
    cfg.dynamicSmemBytes = Cfg::SMEM;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kron_pgrad_gen_kernel<Cfg>, tx, tg, a);
}

using GPgFn = cudaError_t (*)(const void *, const void *, const void *, const void *,
                              const void *, float *, int, const Shape &, float *, float *,
                              float *, float *, double, cudaStream_t);
struct GPgEntry {
    int p, q, m1, m2, r;
    bool bf16;
    int nt, groups;
    GPgFn fn;
};

#define KRON_GPG(P, Q, M1, M2, R, T, BF, RG, NT)                                   \
    {P, Q, M1, M2, R, BF, NT, GPgCfg<P, Q, M1, M2, R, T, RG, NT>::NG,               \
     &launch_gpgrad<GPgCfg<P, Q, M1, M2, R, T, RG, NT>>}

// Shapes compiled for the generic backward (rows per tile, ranks per group): the GPT-2
// small FFN shapes at r = 1 and 4 and the 4096^2 stress layer (m = 64, r = 8), BF16.
const GPgEntry kGPgTable[] = {
    KRON_GPG(24, 48, 32, 64, 1, __nv_bfloat16, true, 1, 1),
    KRON_GPG(24, 48, 32, 64, 4, __nv_bfloat16, true, 4, 1),
    KRON_GPG(48, 24, 64, 32, 1, __nv_bfloat16, true, 1, 1),
    KRON_GPG(48, 24, 64, 32, 4, __nv_bfloat16, true, 4, 1),
    KRON_GPG(64, 64, 64, 64, 8, __nv_bfloat16, true, 2, 1),
};
#undef KRON_GPG

const GPgEntry *find_gpg(const Shape &s, bool bf16) {
    for (const auto &f : kGPgTable)
        if (f.p == s.p && f.q == s.q && f.m1 == s.m1 && f.m2 == s.m2 && f.r == s.r && f.bf16 == bf16)
            return &f;
    return nullptr;
}

}  // namespace gen

bool generic_pgrad_supported(const Shape &s, bool bf16) { return gen::find_gpg(s, bf16) != nullptr; }

int generic_pgrad_tile_rows(const Shape &s, bool bf16) {
    const gen::GPgEntry *f = gen::find_gpg(s, bf16);
    return f ? f->nt : 0;
}

int generic_pgrad_max_parts(const Shape &s, bool bf16) {
    const gen::GPgEntry *f = gen::find_gpg(s, bf16);
    return f ? kRowParts / f->groups : 0;
}

cudaError_t generic_pgrad(const void *x, const void *S, const void *A, const void *B,
                          const void *dY, float *ws, int parts, const Shape &s, float *dS,
                          float *dA, float *dB, float *dbias, bool bf16, double l1,
                          cudaStream_t st) {
    const gen::GPgEntry *f = gen::find_gpg(s, bf16);
    if (!f) return cudaErrorNotSupported;
    return f->fn(x, S, A, B, dY, ws, parts, s, dS, dA, dB, dbias, l1, st);
}

}  // namespace tc
}  // namespace kron
