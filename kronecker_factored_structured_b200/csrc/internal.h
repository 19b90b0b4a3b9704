// internal.h -- declarations shared by the translation units of libkronlinear.so.
// Not part of the public ABI (include/kron_linear.h is).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace kron {

// Name of the host-side step that failed in the last launcher call on this thread.
const char *&launch_step();

// Host helpers of the tensor-core kernels (tc_host.cu).
namespace tc {
// Multiprocessor count of the current device.
int num_sms();
// The current device and the id of the CUDA context current on this thread (after making
// the runtime's context current if none is).  Keys caches of device addresses, which
// belong to one context.
cudaError_t current_context_id(int *dev, unsigned long long *id);
// Address of the device error word in the current context (nullptr if it cannot be read).
int *device_error_ptr();
// 2-D tensor map of a row-major [rows][cols] fp32 (bf16 = false) or bf16 matrix with a
// box of box_cols x box_rows, swizzled by sw bytes (128, 64, 32 or 0); atom32 selects the
// 128-byte swizzle with 32-byte atoms (the layout of MN-major TF32 MMA operands).
cudaError_t make_tmap_2d(CUtensorMap *map, const void *base, bool bf16, uint64_t rows,
                         uint64_t cols, uint32_t box_cols, uint32_t box_rows, int sw,
                         bool atom32);
}  // namespace tc

struct Shape {
    int64_t N;
    int p, q, m1, m2, r;
    int64_t d_in() const { return (int64_t)p * m1; }
    int64_t d_out() const { return (int64_t)q * m2; }
};

// Number of contiguous row ranges the backward splits N into.  A fixed constant
// (the SM count of a B200), so the partition, and with it the summation order of
// dS/dA/dB/dbias, does not depend on scheduling or on the device.
constexpr int kRowParts = 148;

// Floats of one row range's partial sums in the workspace:
// [dC: r*p*q][dB: r*m1*m2][dbias: q*m2], each range padded to 64 floats.
inline size_t partial_stride(const Shape &s) {
    size_t n = (size_t)s.r * s.p * s.q + (size_t)s.r * s.m1 * s.m2 + (size_t)s.q * s.m2;
    return (n + 63) & ~(size_t)63;
}

// ---- exact FP32 path on the CUDA cores (simt_f32.cu) ----
// Rows per tile for the SIMT kernels; 0 when the shape does not fit shared memory.
int simt_forward_rows(const Shape &s);
int simt_backward_rows(const Shape &s);
// Every tensor fp32, FP32 arithmetic.  skip drops the products with a zero S entry
// (KRON_FLAG_SKIP_ZERO_BLOCKS; same results).
cudaError_t simt_forward(const void *x, const void *S, const void *A, const void *B,
                         const void *bias, void *y, const Shape &s, bool skip, cudaStream_t st);
// Writes dX (if non-null) and the per-range partials into ws (parts x partial_stride).
cudaError_t simt_backward(const void *x, const void *S, const void *A, const void *B,
                          const void *dY, void *dX, float *ws, int parts, const Shape &s,
                          bool skip, cudaStream_t st);

// ---- tensor-core paths (tc_fwd.cu, tc_bwd.cu, tc_gen.cu): TF32 (fp32 I/O) or BF16 ----
// A shape runs on the tuned kernels of the tutorial layer (p = q = m1 = m2 = 32, r = 4)
// or on the generic kernels where their tiles fit TMEM and shared memory.
bool tc_forward_supported(const Shape &s, bool bf16);
cudaError_t tc_forward(const void *x, const void *S, const void *A, const void *B,
                       const void *bias, void *y, const Shape &s, bool bf16, bool skip,
                       cudaStream_t st);
bool tc_backward_supported(const Shape &s, bool bf16);
// Rows per tile of the backward's row-range split, and the largest number of row ranges.
int tc_backward_tile_rows(const Shape &s, bool bf16);
int tc_backward_max_parts(const Shape &s, bool bf16);
// Writes dX (if non-null) and the final dS, dA, dB, dbias (dbias may be null).  ws holds
// parts x partial_stride floats of row-range partials followed by one grid-barrier word
// (tc_backward_workspace_extra bytes).  l1 != 0 adds l1 * sign(S) to dS.
cudaError_t tc_backward(const void *x, const void *S, const void *A, const void *B,
                        const void *dY, void *dX, float *ws, int parts, const Shape &s,
                        float *dS, float *dA, float *dB, float *dbias, bool bf16, bool skip,
                        double l1, cudaStream_t st);
constexpr size_t tc_backward_workspace_extra = 256;
// Device error word of the tensor-core kernels (bounded waits); -1 if unreadable.
int tc_read_device_error(bool clear);

namespace tc {
// The kernel shape of dX = dY W^T: the layer's shape with (p, q) and (m1, m2) swapped (the
// forward's vec trick with C_i^T and B_i^T).
inline Shape transposed(const Shape &s) { return Shape{s.N, s.q, s.p, s.m2, s.m1, s.r}; }
// Tuned kernels of the tutorial layer (tc_fwd.cu, tc_bwd.cu).  ks is the kernel's shape:
// the layer's for the forward (tr = false), transposed(layer) for dX (tr = true).
bool tuned_fwd_supported(const Shape &ks, bool bf16, bool tr);
cudaError_t tuned_fwd(const void *x, const void *S, const void *A, const void *B,
                      const void *bias, void *y, const Shape &ks, bool bf16, bool tr,
                      cudaStream_t st);
bool tuned_pgrad_supported(const Shape &s, bool bf16);
// Parameter gradients with the fixed-order reduction fused after a grid barrier
// (cooperative launch of `parts` CTAs, which must all be resident at once).
cudaError_t tuned_pgrad(const void *x, const void *S, const void *A, const void *B,
                        const void *dY, float *ws, int parts, const Shape &s, float *dS,
                        float *dA, float *dB, float *dbias, bool bf16, double l1,
                        cudaStream_t st);
// Generic tensor-core kernels (tc_gen_fwd.cu, tc_gen_pgrad.cu) for the other compiled
// shapes.  skip = KRON_FLAG_SKIP_ZERO_BLOCKS.
bool generic_fwd_supported(const Shape &ks, bool bf16, bool tr);
cudaError_t generic_fwd(const void *x, const void *S, const void *A, const void *B,
                        const void *bias, void *y, const Shape &ks, bool bf16, bool tr,
                        bool skip, cudaStream_t st);
// Parameter gradients: row-range partials of dC, dB and dbias into ws (parts x
// partial_stride floats, then the grid-barrier word), summed in a fixed order by the same
// cooperative launch of parts x (rank groups) CTAs, which writes dS, dA, dB and dbias.
bool generic_pgrad_supported(const Shape &s, bool bf16);
int generic_pgrad_tile_rows(const Shape &s, bool bf16);
int generic_pgrad_max_parts(const Shape &s, bool bf16);
cudaError_t generic_pgrad(const void *x, const void *S, const void *A, const void *B,
                          const void *dY, float *ws, int parts, const Shape &s, float *dS,
                          float *dA, float *dB, float *dbias, bool bf16, double l1,
                          cudaStream_t st);
}  // namespace tc

// ---- deterministic reduction of the row-range partials (reduce.cu) ----
// S and A are float (is_bf16 = false) or bfloat16 (is_bf16 = true).  l1 != 0 adds
// l1 * sign(S) to dS.  parts == 0 reads nothing from ws (every partial sum is zero).
cudaError_t reduce_partials(const float *ws, int parts, const void *S, const void *A,
                            bool is_bf16, float *dS, float *dA, float *dB, float *dbias,
                            const Shape &s, double l1, cudaStream_t st);

// sign(v) in {-1, 0, +1} (0 for zero and NaN): the subgradient of |v| that autograd takes.
__host__ __device__ inline double sign_of(float v) { return (double)((v > 0.f) - (v < 0.f)); }

}  // namespace kron
