// tc_gen_common.cuh -- element traits and shared-memory layout helpers of the generic
// tensor-core kernels (tc_gen_fwd.cu, tc_gen_pgrad.cu).
#pragma once

#include "tc_ptx.cuh"

#include <cuda_bf16.h>

namespace kron {
namespace tc {
namespace gen {

template <typename T> struct GE;
template <> struct GE<float> {
    static constexpr int bytes = 4;
    static constexpr uint32_t fmt = 2;   // TF32 operands
    static constexpr bool tf32 = true;
};
template <> struct GE<__nv_bfloat16> {
    static constexpr int bytes = 2;
    static constexpr uint32_t fmt = 1;   // BF16 operands
    static constexpr bool tf32 = false;
};

constexpr int gmin(int a, int b) { return a < b ? a : b; }
constexpr int gmax(int a, int b) { return a > b ? a : b; }
constexpr int up(int a, int b) { return (a + b - 1) / b * b; }
constexpr int cdiv(int a, int b) { return (a + b - 1) / b; }
constexpr int tmem_cols_pow2(int n) {
    return n <= 32 ? 32 : n <= 64 ? 64 : n <= 128 ? 128 : n <= 256 ? 256 : 512;
}

template <typename T>
__device__ __forceinline__ float ld_elt(const void *p, size_t i) {
    if constexpr (GE<T>::tf32) return static_cast<const float *>(p)[i];
    else return __bfloat162float(static_cast<const __nv_bfloat16 *>(p)[i]);
}

// One operand value for a TMEM A operand column pair / shared store: TF32 operands are
// rounded to nearest (ties away) once when the factors are packed.
__device__ __forceinline__ uint32_t tf32_bits(float v) { return f32_to_tf32(v); }

// Byte offset of element (row, kbyte) in a K-major operand region of `rows` rows whose K
// runs in chunk-columns of `sw` bytes (chunk-major), 8-row atoms of 8*sw bytes, swizzled.
__device__ __forceinline__ uint32_t kmaj(int row, int kbyte, int rows, int sw) {
    const int chunk = kbyte / sw, inner = kbyte % sw;
    return swz((uint32_t)chunk * rows * sw + (uint32_t)(row >> 3) * 8 * sw +
                   (uint32_t)(row & 7) * sw + inner,
               sw);
}

// Store one fp32 accumulator value as an operand element (TF32: the fp32 bits, whose top
// 19 bits the MMA reads; BF16: rounded to nearest even).
template <typename T>
__device__ __forceinline__ void st_op(uint32_t addr, uint32_t v) {
    if constexpr (GE<T>::tf32) st_shared_u32(addr, v);
    else st_shared_u16(addr, __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(v))));
}

// 16 bytes of operand values (4 TF32 / 8 BF16) from fp32 accumulator bits.
template <typename T>
__device__ __forceinline__ void st_op16(uint32_t addr, const uint32_t *r) {
    if constexpr (GE<T>::tf32) {
        st_shared_v4(addr, r[0], r[1], r[2], r[3]);
    } else {
        st_shared_v4(addr, pack_bf16x2(__uint_as_float(r[0]), __uint_as_float(r[1])),
                     pack_bf16x2(__uint_as_float(r[2]), __uint_as_float(r[3])),
                     pack_bf16x2(__uint_as_float(r[4]), __uint_as_float(r[5])),
                     pack_bf16x2(__uint_as_float(r[6]), __uint_as_float(r[7])));
    }
}

// Zero `bytes` (a multiple of 16) of shared memory from `base`, by the whole CTA.
__device__ __forceinline__ void zero_smem(uint32_t base, int bytes) {
    for (int o = threadIdx.x * 16; o < bytes; o += blockDim.x * 16) st_shared_v4(base + o, 0, 0, 0, 0);
}

}  // namespace gen
}  // namespace tc
}  // namespace kron
