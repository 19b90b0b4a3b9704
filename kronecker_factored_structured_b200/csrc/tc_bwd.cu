// tc_bwd.cu -- backward of the Kronecker layer on the sm_100a tensor cores (tcgen05).
//
// Gradients of L = <G, y> (G = dY), W = sum_i kron(C_i, B_i), C_i = S (.) A_i (page
// "kronecker-layer-benchmark", section "1. Build W, then multiply"; the page leaves the
// backward to autograd).  Per tile of NT = 128/m1 rows, with only K-major operands:
//
//   T'[(i,j),(n,c)] = sum_k B_i[j,k] G[(n,c),k]          (G B_i^T, A = B' [(i,j)][k])
//   U [(n,k),(i,a)] = sum_c G[(n,c),k] C_i[a,c]          (C_i G,   A = G^T [(n,k)][c])
//   dX[(n,j),a]     = sum_(i,c) T'[n,c,i,j] C_i[a,c]     (A = T'1 [(n,j)][(i,c)])
//   dC[(i,c),a]    += sum_(n,j) T'[n,c,i,j] X[(n,a),j]   (A = T'2 [(i,c)][(n,j)])
//   dB[(i,k),j]    += sum_(n,a) U[n,a,i,k] X[(n,a),j]    (A = U2 [(i,k)][(n,a)], B = X^T)
//   dbias[c*m2+k]  += sum_n G[(n,c),k]
//
// T' and U exist only in TMEM and shared memory.  The TMEM -> shared-memory epilogues
// write them in the K-major swizzled layouts the next contraction reads (the permute
// the page's loop-free version does in HBM).  dC and dB accumulate in TMEM over the
// CTA's fixed, contiguous range of rows, then go to the workspace as this range's
// partial sums; reduce.cu adds the partials in a fixed order, so results are
// reproducible bit for bit.
//
// Shared memory holds two intermediate buffers: A (T'1, then U2) and B (T'2, then X^T).
// Warp roles (448 threads, one CTA per SM):
//   warp 0       TMA producer (G and X tiles, one buffer each)
//   warp 1       TMEM allocator + single-thread MMA issuer
//   warps 2-5    G^T and X^T transposes, dbias partial, dX epilogue (TMEM -> HBM)
//   warps 6-13   T' epilogue (T'1 and T'2) and U epilogue (U2), 2 warps per TMEM quadrant
// The issuer waits at few points per tile (each wait drains its queued MMAs).
#include "internal.h"
#include "tc_ptx.cuh"

#include <cuda_runtime.h>

namespace kron {
namespace tc {

int *device_error_ptr();
int num_sms();
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
constexpr int imax(int a, int b) { return a > b ? a : b; }

template <int P_, int Q_, int M1_, int M2_, int R_, typename T_>
struct BwdCfg {
    using T = T_;
    static constexpr int P = P_, Q = Q_, M1 = M1_, M2 = M2_, R = R_;
    static constexpr int E = BE<T>::bytes;
    static constexpr int NT = 128 / M1;            // rows per tile
    // swizzle widths of the K extents used below (bytes)
    static constexpr int SWK = imin(128, M2 * E);  // K = k   (T' MMA: B', G)
    static constexpr int SWC = imin(128, Q * E);   // K = c   (U MMA: G^T, C_stack)
    static constexpr int SWQ = imin(128, Q * E);   // K = (i,c) chunks (dX: T'1, Cdx)
    static constexpr int SWJ = imin(128, M1 * E);  // K = (n,j) chunks (dC: T'2, X)
    static constexpr int SWA = imin(128, P * E);   // K = (n,a) chunks (dB: U2, X^T)
    // region sizes (bytes)
    static constexpr int F_BP = 128 * M2 * E;          // B'      [(i,j)][k]
    static constexpr int F_CS = R * P * Q * E;         // C_stack [(i,a)][c]
    static constexpr int F_CDX = P * R * Q * E;        // Cdx     [a][(i,c)]
    static constexpr int TILE_G = NT * Q * M2 * E;     // G tile  [(n,c)][k]
    static constexpr int TILE_X = NT * P * M1 * E;     // X tile  [(n,a)][j]
    static constexpr int TILE_GT = TILE_G;             // G^T     [(n,k)][c]
    static constexpr int BUF_A = imax(128 * R * Q * E, R * M2 * NT * P * E);  // T'1 | U2
    static constexpr int BUF_B = imax(R * Q * NT * M1 * E, M1 * NT * P * E);  // T'2 | X^T
    static constexpr int OFF_BP = 0;
    static constexpr int OFF_CS = OFF_BP + F_BP;
    static constexpr int OFF_CDX = OFF_CS + F_CS;
    static constexpr int OFF_G = OFF_CDX + F_CDX;
    static constexpr int OFF_X = OFF_G + TILE_G;
    static constexpr int OFF_GT = OFF_X + TILE_X;
    static constexpr int OFF_A = OFF_GT + TILE_GT;
    static constexpr int OFF_B = OFF_A + BUF_A;
    static constexpr int OFF_BAR = OFF_B + BUF_B;
    static constexpr int SMEM = OFF_BAR + 256 + 1024;
    // TMEM columns
    static constexpr int TM_TP = 0;                    // T'  : lanes (i,j), NT*Q columns (n,c)
    static constexpr int TM_U = TM_TP + NT * Q;        // U   : lanes (n,k), R*P columns (i,a)
    static constexpr int TM_DX = TM_U + R * P;         // dX  : lanes (n,j), P columns (a)
    static constexpr int TM_DC = TM_DX + P;            // dC  : lanes (i,c), P columns (a)
    static constexpr int TM_DB = TM_DC + P;            // dB  : lanes (i,k), M1 columns (j)
    static constexpr int TM_USED = TM_DB + M1;
    static constexpr int TM_COLS = TM_USED <= 128 ? 128 : TM_USED <= 256 ? 256 : 512;
    static constexpr uint32_t ID_TP = idesc_f32acc(128, NT * Q, BE<T>::fmt);
    static constexpr uint32_t ID_U = idesc_f32acc(128, R * P, BE<T>::fmt);
    static constexpr uint32_t ID_DX = idesc_f32acc(128, P, BE<T>::fmt);
    static constexpr uint32_t ID_DC = idesc_f32acc(128, P, BE<T>::fmt);
    static constexpr uint32_t ID_DB = idesc_f32acc(128, M1, BE<T>::fmt);

    static_assert(R * M1 == 128 && M1 == M2 && Q == M1, "needs r*m1 = 128 and m1 = m2 = q");
    static_assert(NT * M1 == 128 && NT * M2 == 128, "tile rows");
    static_assert(P % 32 == 0 && P <= 64 && R * P <= 256, "p: multiple of 32, r*p <= 256");
    static_assert(NT * Q <= 256 && NT * Q % 32 == 0, "T' columns");
    static_assert(M1 % 32 == 0 && Q % 32 == 0, "32-column TMEM loads");
    static_assert(M1 * E % 32 == 0 && M1 * E <= 128, "an x row block of m1 must fit one swizzle row");
    static_assert(Q * E % 32 == 0 && (Q * E <= 128 || Q * E % 128 == 0), "q bytes");
    static_assert(P * E % 32 == 0 && (P * E <= 128 || P * E % 128 == 0), "p bytes");
    static_assert(TM_USED <= 512, "TMEM budget");
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

// (row, kbyte) of a K-major swizzled operand region: K split in chunks of sw bytes
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

// one operand element (as stored: tf32-rounded fp32 or bf16)
template <typename T>
__device__ __forceinline__ void st1(uint32_t addr, float v) {
    if constexpr (BE<T>::tf32) {
        asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(f32_to_tf32(v)) : "memory");
    } else {
        const __nv_bfloat16 h = __float2bfloat16_rn(v);
        asm volatile("st.shared.b16 [%0], %1;" ::"r"(addr),
                     "h"(*reinterpret_cast<const unsigned short *>(&h))
                     : "memory");
    }
}

template <typename T>
__device__ __forceinline__ float ld1(uint32_t addr) {
    if constexpr (BE<T>::tf32) {
        float v;
        asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
        return v;
    } else {
        unsigned short h;
        asm volatile("ld.shared.b16 %0, [%1];" : "=h"(h) : "r"(addr) : "memory");
        return __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(&h));
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
    const uint32_t sBP = sb + Cfg::OFF_BP, sCS = sb + Cfg::OFF_CS, sCDX = sb + Cfg::OFF_CDX;
    const uint32_t sG = sb + Cfg::OFF_G, sX = sb + Cfg::OFF_X, sGT = sb + Cfg::OFF_GT;
    const uint32_t sA = sb + Cfg::OFF_A, sBb = sb + Cfg::OFF_B;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + Cfg::OFF_BAR);
    enum {
        G_FULL, X_FULL,       // TMA landed
        G_FREE, X_FREE,       // G / X tile may be overwritten
        GT_FULL, GT_FREE,     // G^T written / consumed by the U MMA
        TP_FULL,              // T' accumulator ready (read out before TT_FULL)
        U_FULL,               // U accumulator ready (read out before UX_FULL)
        TT_FULL,              // T'1 and T'2 written
        AB_FREE1,             // dX + dC MMAs done: buffers A, B and the X tile (for dC) free
        DX_FULL, DX_FREE,     // dX accumulator ready / read out
        UX_FULL,              // U2 and X^T written
        AB_FREE2,             // dB MMAs done: buffers A and B free
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
        mbar_init(bar(G_FREE), 1 + 128);  // T' MMA commit + transpose warps
        mbar_init(bar(X_FREE), 1 + 128);  // dC MMA commit + transpose warps (X^T written)
        mbar_init(bar(GT_FULL), 128);
        mbar_init(bar(GT_FREE), 1);
        mbar_init(bar(TP_FULL), 1);
        mbar_init(bar(U_FULL), 1);
        mbar_init(bar(TT_FULL), 256);
        mbar_init(bar(AB_FREE1), 1);
        mbar_init(bar(DX_FULL), 1);
        mbar_init(bar(DX_FREE), 128);
        mbar_init(bar(UX_FULL), 256 + 128);
        mbar_init(bar(AB_FREE2), 1);
        mbar_init(bar(DRAIN), 1);
        *ab.flag = 0;
        mbar_init_fence();
        prefetch_tmap(&tmap_g);
        prefetch_tmap(&tmap_x);
    }
    if (warp == 1) tmem_alloc(smem_u32(tmem_slot), Cfg::TM_COLS);
    // factors: B'[(i,j)][k] = B_i[j][k]; C_stack[(i,a)][c] = C_i[a][c]; Cdx[a][(i,c)] = C_i[a][c]
    for (int e = threadIdx.x; e < 128 * (M2 / VPC); e += blockDim.x) {
        const int row = e / (M2 / VPC), k0 = (e % (M2 / VPC)) * VPC;
        float v[8];
#pragma unroll
        for (int t = 0; t < VPC; ++t) v[t] = bld<T>(args.B, (size_t)row * M2 + k0 + t);
        st16v<T>(sBP + koff(row, k0 * E, 128, Cfg::SWK), v);
    }
    for (int e = threadIdx.x; e < R * P * (Q / VPC); e += blockDim.x) {
        const int row = e / (Q / VPC), c0 = (e % (Q / VPC)) * VPC;  // row = (i,a)
        const int i = row / P, a = row % P;
        float v[8];
#pragma unroll
        for (int t = 0; t < VPC; ++t)
            v[t] = bld<T>(args.S, (size_t)a * Q + c0 + t) * bld<T>(args.A, ((size_t)i * P + a) * Q + c0 + t);
        st16v<T>(sCS + koff(row, c0 * E, R * P, Cfg::SWC), v);
        st16v<T>(sCDX + koff(a, (i * Q + c0) * E, P, Cfg::SWQ), v);
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
                mbar_arrive_expect_tx(bar(G_FULL), Cfg::TILE_G);
                for (int kc = 0; kc < M2 * E / Cfg::SWK; ++kc)
                    tma_load_2d(sG + kc * NT * Q * Cfg::SWK, &tmap_g, kc * (Cfg::SWK / E),
                                tile * NT * Q, bar(G_FULL));
                if (!mbar_wait(bar(X_FREE), ph ^ 1, ab)) break;
                mbar_arrive_expect_tx(bar(X_FULL), Cfg::TILE_X);
                for (int kc = 0; kc < M1 * E / Cfg::SWJ; ++kc)
                    tma_load_2d(sX + kc * NT * P * Cfg::SWJ, &tmap_x, kc * (Cfg::SWJ / E),
                                tile * NT * P, bar(X_FULL));
                issued = u + 1;
            }
            if (issued > 0) {
                mbar_wait_drain(bar(G_FULL), (issued - 1) & 1);
                mbar_wait_drain(bar(X_FULL), (issued - 1) & 1);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            auto mma = [&](uint32_t d, uint64_t a, uint64_t b, uint32_t id, uint32_t acc) {
                mma_ss<BE<T>::tf32>(d, a, b, id, acc);
            };
            // T'(u): D[(i,j),(n,c)] = B'[(i,j)][k] . G[(n,c)][k]
            auto issue_tp = [&]() {
                for (int kb = 0; kb < M2 * E; kb += 32) {
                    const int ch = kb / Cfg::SWK, in = kb % Cfg::SWK;
                    mma(tmem + Cfg::TM_TP, sdesc_kmajor(sBP + ch * 128 * Cfg::SWK + in, Cfg::SWK),
                        sdesc_kmajor(sG + ch * NT * Q * Cfg::SWK + in, Cfg::SWK), Cfg::ID_TP, kb > 0);
                }
            };
            // U(u): D[(n,k),(i,a)] = G^T[(n,k)][c] . C_stack[(i,a)][c]
            auto issue_u = [&]() {
                for (int kb = 0; kb < Q * E; kb += 32) {
                    const int ch = kb / Cfg::SWC, in = kb % Cfg::SWC;
                    mma(tmem + Cfg::TM_U, sdesc_kmajor(sGT + ch * 128 * Cfg::SWC + in, Cfg::SWC),
                        sdesc_kmajor(sCS + ch * R * P * Cfg::SWC + in, Cfg::SWC), Cfg::ID_U, kb > 0);
                }
            };
            bool ok = true;
            // prologue: T'(0) and U(0)
            if (nt > 0) {
                ok = mbar_wait(bar(G_FULL), 0, ab) && mbar_wait(bar(GT_FULL), 0, ab);
                if (ok) {
                    tc_fence_after();
                    issue_tp();
                    mma_commit(bar(TP_FULL));
                    mma_commit(bar(G_FREE));
                    issue_u();
                    mma_commit(bar(U_FULL));
                    mma_commit(bar(GT_FREE));
                }
            }
            for (int u = 0; u < nt && ok; ++u) {
                const uint32_t ph = u & 1;
                // dX and dC of tile u
                if (!mbar_wait(bar(TT_FULL), ph, ab) || !mbar_wait(bar(X_FULL), ph, ab) ||
                    !mbar_wait(bar(DX_FREE), ph ^ 1, ab)) { ok = false; break; }
                tc_fence_after();
                for (int kb = 0; kb < R * Q * E; kb += 32) {  // K = (i,c)
                    const int ch = kb / Cfg::SWQ, in = kb % Cfg::SWQ;
                    mma(tmem + Cfg::TM_DX, sdesc_kmajor(sA + ch * 128 * Cfg::SWQ + in, Cfg::SWQ),
                        sdesc_kmajor(sCDX + ch * P * Cfg::SWQ + in, Cfg::SWQ), Cfg::ID_DX, kb > 0);
                }
                mma_commit(bar(DX_FULL));
                for (int kb = 0; kb < NT * M1 * E; kb += 32) {  // K = (n,j)
                    const int ch = kb / Cfg::SWJ, in = kb % Cfg::SWJ;
                    mma(tmem + Cfg::TM_DC, sdesc_kmajor(sBb + ch * 128 * Cfg::SWJ + in, Cfg::SWJ),
                        sdesc_kmajor(sX + ch * P * Cfg::SWJ + in, Cfg::SWJ), Cfg::ID_DC,
                        (u > 0 || kb > 0) ? 1u : 0u);
                }
                mma_commit(bar(AB_FREE1));
                mma_commit(bar(X_FREE));
                // T' of tile u+1 (its accumulator was read out before TT_FULL(u))
                if (u + 1 < nt) {
                    if (!mbar_wait(bar(G_FULL), ph ^ 1, ab)) { ok = false; break; }
                    tc_fence_after();
                    issue_tp();
                    mma_commit(bar(TP_FULL));
                    mma_commit(bar(G_FREE));
                }
                // dB of tile u
                if (!mbar_wait(bar(UX_FULL), ph, ab)) { ok = false; break; }
                tc_fence_after();
                for (int kb = 0; kb < NT * P * E; kb += 32) {  // K = (n,a)
                    const int ch = kb / Cfg::SWA, in = kb % Cfg::SWA;
                    mma(tmem + Cfg::TM_DB, sdesc_kmajor(sA + ch * 128 * Cfg::SWA + in, Cfg::SWA),
                        sdesc_kmajor(sBb + ch * M1 * Cfg::SWA + in, Cfg::SWA), Cfg::ID_DB,
                        (u > 0 || kb > 0) ? 1u : 0u);
                }
                mma_commit(bar(AB_FREE2));
                // U of tile u+1 (its accumulator was read out before UX_FULL(u))
                if (u + 1 < nt) {
                    if (!mbar_wait(bar(GT_FULL), ph ^ 1, ab)) { ok = false; break; }
                    tc_fence_after();
                    issue_u();
                    mma_commit(bar(U_FULL));
                    mma_commit(bar(GT_FREE));
                }
            }
            mma_commit(bar(DRAIN));
            mbar_wait_drain(bar(DRAIN), 0);
        }
    } else if (warp < 6) {
        // ---------------- transposes, dbias, dX epilogue (128 threads) ----------------
        const int tid = threadIdx.x - 64;         // 0..127
        const int quad = warp & 3;
        const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
        float dbias[Q * M2 / 128];
#pragma unroll
        for (int e = 0; e < Q * M2 / 128; ++e) dbias[e] = 0.f;
        for (int u = 0; u < nt; ++u) {
            const uint32_t ph = u & 1;
            const int64_t row0 = (int64_t)(t0 + u) * NT;
            // G^T(u) and the dbias partial, once G(u) has landed and G^T(u-1) is consumed
            if (!mbar_wait(bar(G_FULL), ph, ab) || !mbar_wait(bar(GT_FREE), ph ^ 1, ab)) break;
            {
                // thread (n,k) for two n per pass: reads G[(n,c)][k] for all c, writes row (n,k)
                for (int rr = tid; rr < NT * M2; rr += 128) {
                    const int n = rr / M2, k = rr % M2;
                    for (int c0 = 0; c0 < Q; c0 += VPC) {
                        float v[8];
#pragma unroll
                        for (int t = 0; t < VPC; ++t)
                            v[t] = ld1<T>(sG + koff(n * Q + c0 + t, k * E, NT * Q, Cfg::SWK));
                        st16v<T>(sGT + koff(rr, c0 * E, NT * M2, Cfg::SWC), v);
                    }
                }
#pragma unroll
                for (int e = 0; e < Q * M2 / 128; ++e) {
                    const int o = tid + 128 * e, c = o / M2, k = o % M2;
                    float s = 0.f;
                    for (int n = 0; n < NT; ++n)
                        if (row0 + n < args.N) s += ld1<T>(sG + koff(n * Q + c, k * E, NT * Q, Cfg::SWK));
                    dbias[e] += s;
                }
            }
            fence_proxy_async();
            mbar_arrive(bar(GT_FULL));
            mbar_arrive(bar(G_FREE));
            // dX(u): D[(n,j), a] -> dx[row n][a*m1 + j]
            if (!mbar_wait(bar(DX_FULL), ph, ab)) break;
            tc_fence_after();
            {
                const int L = quad * 32 + lane, n = L / M1, j = L % M1;
                const int64_t row = row0 + n;
#pragma unroll
                for (int a0 = 0; a0 < P; a0 += 32) {
                    uint32_t r[32];
                    tmem_load32(tmem + lane_addr + Cfg::TM_DX + a0, r);
                    if (a0 + 32 >= P) {
                        tc_fence_before();
                        mbar_arrive(bar(DX_FREE));
                    }
                    if (args.dX && row < args.N) {
#pragma unroll
                        for (int t = 0; t < 32; ++t) {
                            const size_t o = (size_t)row * (P * M1) + (size_t)(a0 + t) * M1 + j;
                            if constexpr (BE<T>::tf32) static_cast<float *>(args.dX)[o] = __uint_as_float(r[t]);
                            else static_cast<__nv_bfloat16 *>(args.dX)[o] = __float2bfloat16_rn(__uint_as_float(r[t]));
                        }
                    }
                }
            }
            // X^T(u) into buffer B once dC(u) has consumed T'2 (buffer B) and X(u) has landed
            if (!mbar_wait(bar(AB_FREE1), ph, ab)) break;
            for (int rr = tid; rr < NT * M1; rr += 128) {
                const int n = rr / M1, j = rr % M1;  // reads X[(n,a)][j] for all a
                for (int a0 = 0; a0 < P; a0 += VPC) {
                    float v[8];
#pragma unroll
                    for (int t = 0; t < VPC; ++t)
                        v[t] = ld1<T>(sX + koff(n * P + a0 + t, j * E, NT * P, Cfg::SWJ));
                    st16v<T>(sBb + koff(j, (n * P + a0) * E, M1, Cfg::SWA), v);
                }
            }
            fence_proxy_async();
            mbar_arrive(bar(UX_FULL));
            mbar_arrive(bar(X_FREE));
        }
        // dbias partial of this row range
        const size_t off = (size_t)R * P * Q + (size_t)R * M1 * M2;
        float *part = args.ws + (size_t)blockIdx.x * args.ws_stride;
#pragma unroll
        for (int e = 0; e < Q * M2 / 128; ++e) part[off + tid + 128 * e] = dbias[e];
    } else {
        // ---------------- T' and U epilogues (256 threads) ----------------
        const int half = (warp - 6) / 4;
        const int quad = warp & 3;
        const int L = quad * 32 + lane;
        const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
        for (int u = 0; u < nt; ++u) {
            const uint32_t ph = u & 1;
            // T'(u): lanes (i,j), columns (n,c) -> T'1 [(n,j)][(i,c)] (buffer A) and
            // T'2 [(i,c)][(n,j)] (buffer B), once dB(u-1) has released both buffers
            if (!mbar_wait(bar(TP_FULL), ph, ab) || !mbar_wait(bar(AB_FREE2), ph ^ 1, ab)) break;
            tc_fence_after();
            {
                const int i = L / M1, j = L % M1;
                constexpr int HC = NT * Q / 2;
                for (int c0 = half * HC; c0 < (half + 1) * HC; c0 += 32) {
                    uint32_t r[32];
                    tmem_load32(tmem + lane_addr + Cfg::TM_TP + c0, r);
#pragma unroll
                    for (int g = 0; g < 32 / VPC; ++g) {
                        const int col = c0 + g * VPC, n = col / Q, c = col % Q;
                        float v[8];
#pragma unroll
                        for (int t = 0; t < VPC; ++t) v[t] = __uint_as_float(r[g * VPC + t]);
                        st16v<T>(sA + koff(n * M1 + j, (i * Q + c) * E, 128, Cfg::SWQ), v);
#pragma unroll
                        for (int t = 0; t < VPC; ++t)
                            st1<T>(sBb + koff(i * Q + c + t, (n * M1 + j) * E, 128, Cfg::SWJ), v[t]);
                    }
                }
            }
            tc_fence_before();
            fence_proxy_async();
            mbar_arrive(bar(TT_FULL));
            // U(u): lanes (n,k), columns (i,a) -> U2 [(i,k)][(n,a)] (buffer A), once dX(u)
            // has consumed T'1
            if (!mbar_wait(bar(U_FULL), ph, ab) || !mbar_wait(bar(AB_FREE1), ph, ab)) break;
            tc_fence_after();
            {
                const int n = L / M2, k = L % M2;
                constexpr int HC = R * P / 2;
                for (int c0 = half * HC; c0 < (half + 1) * HC; c0 += 32) {
                    uint32_t r[32];
                    tmem_load32(tmem + lane_addr + Cfg::TM_U + c0, r);
#pragma unroll
                    for (int g = 0; g < 32 / VPC; ++g) {
                        const int col = c0 + g * VPC, i = col / P, a = col % P;
                        float v[8];
#pragma unroll
                        for (int t = 0; t < VPC; ++t) v[t] = __uint_as_float(r[g * VPC + t]);
                        st16v<T>(sA + koff(i * M2 + k, (n * P + a) * E, 128, Cfg::SWA), v);
                    }
                }
            }
            tc_fence_before();
            fence_proxy_async();
            mbar_arrive(bar(UX_FULL));
        }
        // dC and dB partials of this row range, once the last dB MMAs are done
        if (nt > 0 && mbar_wait(bar(AB_FREE2), (nt - 1) & 1, ab)) {
            tc_fence_after();
            float *part = args.ws + (size_t)blockIdx.x * args.ws_stride;
            const int cols = half == 0 ? 0 : 16;   // each half writes 16 of the 32 columns
            {   // dC: lanes (i,c), columns a -> dC_i[a][c] at i*p*q + a*q + c
                const int i = L / Q, c = L % Q;
                for (int a0 = 0; a0 < P; a0 += 32) {
                    uint32_t r[32];
                    tmem_load32(tmem + lane_addr + Cfg::TM_DC + a0, r);
#pragma unroll
                    for (int t = 0; t < 32; ++t)
                        if ((t >= cols) && (t < cols + 16))
                            part[(size_t)i * P * Q + (size_t)(a0 + t) * Q + c] = __uint_as_float(r[t]);
                }
            }
            {   // dB: lanes (i,k), columns j -> dB_i[j][k] at r*p*q + i*m1*m2 + j*m2 + k
                const int i = L / M2, k = L % M2;
                for (int j0 = 0; j0 < M1; j0 += 32) {
                    uint32_t r[32];
                    tmem_load32(tmem + lane_addr + Cfg::TM_DB + j0, r);
#pragma unroll
                    for (int t = 0; t < 32; ++t)
                        if ((t >= cols) && (t < cols + 16))
                            part[(size_t)R * P * Q + (size_t)i * M1 * M2 + (size_t)(j0 + t) * M2 + k] =
                                __uint_as_float(r[t]);
                }
            }
        } else if (nt == 0) {
            float *part = args.ws + (size_t)blockIdx.x * args.ws_stride;
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
    cudaError_t e = make_tmap_2d(&tg, dY, bf16, (uint64_t)s.N * Cfg::Q, Cfg::M2,
                                 Cfg::SWK / Cfg::E, Cfg::NT * Cfg::Q, Cfg::SWK);
    if (e != cudaSuccess) return e;
    e = make_tmap_2d(&tx, x, bf16, (uint64_t)s.N * Cfg::P, Cfg::M1, Cfg::SWJ / Cfg::E,
                     Cfg::NT * Cfg::P, Cfg::SWJ);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kron_bwd_tc_kernel<Cfg>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Cfg::SMEM);
    if (e != cudaSuccess) return e;
    BwdTcArgs a;
    a.S = S; a.A = A; a.B = B; a.dX = dX; a.ws = ws;
    a.ws_stride = partial_stride(s);
    a.N = s.N;
    a.num_tiles = (int)((s.N + Cfg::NT - 1) / Cfg::NT);
    a.tiles_per_part = (a.num_tiles + parts - 1) / parts;
    a.device_error = device_error_ptr();
    kron_bwd_tc_kernel<Cfg><<<parts, 448, Cfg::SMEM, st>>>(tg, tx, a);
    return cudaGetLastError();
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

int tc_backward_tile_rows(const Shape &s) { return 128 / s.m1; }

cudaError_t tc_backward(const void *x, const void *S, const void *A, const void *B,
                        const void *dY, void *dX, float *ws, int parts, const Shape &s,
                        bool bf16, cudaStream_t st) {
    tc::BwdFn fn = tc::find_bwd(s, bf16);
    if (!fn) return cudaErrorNotSupported;
    return fn(x, S, A, B, dY, dX, ws, parts, s, st);
}

}  // namespace kron
