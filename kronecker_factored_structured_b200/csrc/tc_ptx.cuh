// tc_ptx.cuh -- thin inline-PTX layer for sm_100a: mbarriers with bounded waits, TMA
// tile loads, tcgen05 (TMEM alloc, MMA, commit, loads) and the shared-memory matrix
// and instruction descriptors of the 5th-generation tensor cores.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace kron {
namespace tc {

constexpr uint64_t kWaitTimeoutNs = 2000000000ull;  // 2 s without progress = deadlock

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// ---------------------------------------------------------------- mbarriers
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_init_fence() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// One arrival per warp: every lane has already fenced its own writes; __syncwarp orders
// them before lane 0's arrival (a 32-lane arrive on one barrier would serialise).
__device__ __forceinline__ void mbar_arrive_warp(uint32_t bar) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Block-wide abort state of one CTA: a shared flag plus the library's device error
// word (bit 0 = a bounded wait gave up), whose address the host passes in.
struct Abort {
    volatile int *flag;
    int *device_error;
};

// Wait for the phase with the given parity to complete.  Gives up (returns false)
// when the CTA's abort flag is raised by another thread or after kWaitTimeoutNs
// without progress, in which case it raises the flag and the device error word.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, const Abort &abort) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 255u) == 0) {
            if (*abort.flag) return false;
            if (globaltimer() - t0 > kWaitTimeoutNs) {
                *abort.flag = 1;
                if (abort.device_error) atomicOr(abort.device_error, 1);
                return false;
            }
        }
    }
}

// mbar_wait by every lane of a warp, with one verdict for the whole warp (so a warp
// that issues tensor-core work stays converged).
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, const Abort &abort) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort)) != 0;
}

// True in exactly one lane of a converged warp (the lowest).  MMA bursts are issued as
//   if (elect_one()) { mma...; commit...; }  __syncwarp();
// from a loop that the whole warp runs: descriptors and addresses then stay warp-uniform,
// which issues several times faster than a loop run by one lane alone.
__device__ __forceinline__ bool elect_one() {
    uint32_t e;
    asm volatile(
        "{\n\t.reg .pred e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "selp.u32 %0, 1, 0, e;\n\t}"
        : "=r"(e));
    return e != 0;
}

// Bounded wait that ignores the abort flag: used to let this thread's own asynchronous
// work (MMAs, copies) finish before shared memory or TMEM is released.
__device__ __forceinline__ bool mbar_wait_drain(uint32_t bar, uint32_t parity) {
    const uint64_t t0 = globaltimer();
    for (uint32_t it = 0;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 255u) == 255u && globaltimer() - t0 > kWaitTimeoutNs) return false;
    }
}

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int32_t x,
                                            int32_t y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

// Pull the tile at (x, y) of a 2-D tensor map into L2 (no shared memory, no completion
// tracking): a later TMA load of the same tile then waits on L2 instead of HBM.
__device__ __forceinline__ void tma_prefetch_l2_2d(const CUtensorMap *map, int32_t x, int32_t y) {
    asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(x), "r"(y)
                 : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     dst_smem),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T ; kind selects TF32 (4-byte) or BF16 operands.
template <bool kTF32>
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
    if constexpr (kTF32) {
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
            "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
            : "memory");
    } else {
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
            "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
            : "memory");
    }
}

// D[tmem] (+)= A[tmem] * B[smem]^T: the A operand (M rows x K) is read from TMEM, row m in
// lane m, K along consecutive 32-bit columns (two BF16 values per column).
template <bool kTF32>
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
    if constexpr (kTF32) {
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
            "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
            : "memory");
    } else {
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
            "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
            : "memory");
    }
}

// 32 lanes x 32 consecutive 32-bit columns from registers (layout as tmem_load32); the
// store is complete when the call returns.
__device__ __forceinline__ void tmem_store32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
        "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};\n\t"
        "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
        "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
        "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

// 32 lanes x 8 consecutive 32-bit columns from registers; complete on return.
__device__ __forceinline__ void tmem_store8(uint32_t taddr, const uint32_t *r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};\n\t"
        "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
        : "memory");
}

// Arrive once on the mbarrier when every tcgen05 op issued so far by this thread is done.
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
        : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: register j of thread t = column (col + j) of
// lane (lane_base + t).  The warp may only address its own quadrant of 32 lanes.  The
// load and its wait are one asm statement, so no use of r[] can be scheduled before
// the data has arrived.
__device__ __forceinline__ void tmem_load32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, "
        "[%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr)
        : "memory");
}

// Paired lane order of an accumulator whose epilogue stores BF16 pairs of adjacent M
// indices: in each aligned group of 16 TMEM lanes, lanes 0-7 hold the even and lanes 8-15
// the odd M indices of the group, so that a 16x256b load (below) gives every thread the
// values of M indices 2g and 2g + 1 side by side.  Returns the M index held by lane L.
__device__ __forceinline__ int pair_lane_index(int L) {
    const int l = L & 15;
    return (L & ~15) + (l < 8 ? 2 * l : 2 * (l - 8) + 1);
}

// 16 lanes x 32 consecutive 32-bit columns in the 16x256b pattern (four repetitions of
// 8 columns): with g = t / 4 and c = 2 * (t % 4), registers 4*rep .. 4*rep + 3 of thread
// t hold (lane g, column 8*rep + c), (lane g, 8*rep + c + 1), (lane g + 8, 8*rep + c) and
// (lane g + 8, 8*rep + c + 1), lanes counted from the 16-lane base in taddr (which lies in
// the warp's own quadrant).  Load and wait are one asm statement, as in tmem_load32.
__device__ __forceinline__ void tmem_load16x256_x4(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.16x256b.x4.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}

// 32 lanes x N (8 or 16) consecutive 32-bit columns, layout as tmem_load32.
template <int N>
__device__ __forceinline__ void tmem_load_n(uint32_t taddr, uint32_t (&r)[N]);
template <>
__device__ __forceinline__ void tmem_load_n<8>(uint32_t taddr, uint32_t (&r)[8]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7])
        : "r"(taddr)
        : "memory");
}
template <>
__device__ __forceinline__ void tmem_load_n<16>(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}
template <>
__device__ __forceinline__ void tmem_load_n<32>(uint32_t taddr, uint32_t (&r)[32]) {
    tmem_load32(taddr, r);
}

// ---------------------------------------------------------------- descriptors
// Swizzle width (bytes) -> UMMA layout type (3 bits at 61..63 of the smem descriptor).
__host__ __device__ constexpr uint32_t layout_type(int sw) {
    return sw == 128 ? 2u : sw == 64 ? 4u : sw == 32 ? 6u : 0u;
}

// K-major operand tile in the canonical swizzled layout: rows of `sw` bytes along K,
// 8-row atoms of 8*sw bytes (stride byte offset), swizzle applied on address bits.
__device__ __forceinline__ uint64_t sdesc_kmajor(uint32_t saddr, int sw) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);              // start address
    d |= (uint64_t)(((8u * sw) >> 4) & 0x3FFFu) << 32;     // stride byte offset
    d |= (uint64_t)1 << 46;                                // descriptor version (sm100)
    d |= (uint64_t)layout_type(sw) << 61;
    return d;
}

// A descriptor for the same operand layout starting byte_off bytes further on.  The start
// address field holds (address >> 4) in 14 bits; every shared-memory address of a CTA is
// below 2^18 bytes, so the addition never carries out of the field.
__device__ __forceinline__ uint64_t desc_add(uint64_t desc, uint32_t byte_off) {
    return desc + (uint64_t)(byte_off >> 4);
}

// MN-major operand tile: the M (or N) dimension runs along rows of 128 B (TF32, layout
// type 1 = 128-byte swizzle with 32-byte atoms, 4-row K groups) or of `sw` bytes (16-bit
// types, the ordinary swizzles, 8-row K groups); `lbo` = byte stride between successive
// MN blocks of one row width, `sbo` = byte stride between successive K groups.
__device__ __forceinline__ uint64_t sdesc_mn(uint32_t saddr, uint32_t layout, uint32_t lbo,
                                             uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)layout << 61;
    return d;
}
constexpr uint32_t kLayoutSw128Atom32 = 1u;  // the only MN-major layout for TF32 operands

// Instruction descriptor: FP32 accumulator, A/B of format fmt (1 = BF16, 2 = TF32), both
// K-major, shape M x N.  OR in kBMajorMN when B is MN-major.
__host__ __device__ constexpr uint32_t idesc_f32acc(int M, int N, uint32_t fmt) {
    return (1u << 4) | (fmt << 7) | (fmt << 10) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}
constexpr uint32_t kBMajorMN = 1u << 16;

// Byte offset of (row, byte-in-row) inside a K-major swizzled region whose rows are `sw`
// bytes, with 1024-byte-aligned base: the 16-byte chunk index is XORed with address
// bits 7.. (the TMA / UMMA swizzle pattern).
__device__ __forceinline__ uint32_t swz(uint32_t off, int sw) {
    return off ^ (((off >> 7) & (uint32_t)(sw / 16 - 1)) << 4);
}

// fp32 -> TF32 operand (10 explicit mantissa bits), rounded to nearest with ties away
// from zero: add half a TF32 unit in the last place to the magnitude bits and clear the
// 13 dropped bits (a carry out of the mantissa moves the exponent up, as rounding
// should).  Infinities and NaNs pass through unchanged.  Two integer operations, where
// the conversion instruction costs several times more in the epilogues.
__device__ __forceinline__ uint32_t f32_to_tf32(float v) {
    const uint32_t u = __float_as_uint(v);
    return (u & 0x7F800000u) == 0x7F800000u ? u : ((u + 0x1000u) & 0xFFFFE000u);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ void ld_shared_v4(uint32_t addr, uint32_t (&v)[4]) {
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3])
                 : "r"(addr)
                 : "memory");
}

__device__ __forceinline__ void st_shared_u16(uint32_t addr, uint16_t v) {
    asm volatile("st.shared.b16 [%0], %1;" ::"r"(addr), "h"(v) : "memory");
}

// Named barrier that also returns the AND of `pred` over its threads, so a group of warps
// leaves a loop together (none is left waiting at a later barrier of the group).
__device__ __forceinline__ bool named_bar_and(int id, int threads, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.and.pred p, %2, %3, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(threads)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ void st_shared_u32(uint32_t addr, uint32_t v) {
    asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}

}  // namespace tc
}  // namespace kron
