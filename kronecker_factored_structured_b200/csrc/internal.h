// internal.h -- declarations shared by the translation units of libkronlinear.so.
// Not part of the public ABI (include/kron_linear.h is).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace kron {

// Name of the host-side step that failed in the last launcher call on this thread.
const char *&launch_step();

// Multiprocessor count of the current device (tc_fwd.cu).
namespace tc { int num_sms(); }

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
// I/O tensors fp32, or bf16 when bf16 is set (arithmetic fp32 either way).  skip drops
// the products with a zero S entry (KRON_FLAG_SKIP_ZERO_BLOCKS; same results).
cudaError_t simt_forward(const void *x, const void *S, const void *A, const void *B,
                         const void *bias, void *y, const Shape &s, bool bf16, bool skip,
                         cudaStream_t st);
// Writes dX (if non-null) and the per-range partials into ws (parts x partial_stride).
cudaError_t simt_backward(const void *x, const void *S, const void *A, const void *B,
                          const void *dY, void *dX, float *ws, int parts, const Shape &s,
                          bool bf16, bool skip, cudaStream_t st);

// ---- tensor-core paths (tc_fwd.cu, tc_bwd.cu): TF32 (fp32 I/O) or BF16 ----
bool tc_forward_supported(const Shape &s, bool bf16);
cudaError_t tc_forward(const void *x, const void *S, const void *A, const void *B,
                       const void *bias, void *y, const Shape &s, bool bf16, cudaStream_t st);
// dX = dY W^T by the forward kernel with transposed factors (s is the layer's shape).
bool tc_dx_supported(const Shape &s, bool bf16);
cudaError_t tc_dx(const void *dY, const void *S, const void *A, const void *B, void *dX,
                  const Shape &s, bool bf16, cudaStream_t st);
bool tc_backward_supported(const Shape &s, bool bf16);
int tc_backward_tile_rows(const Shape &s);
// Writes dX (if non-null) and the final dS, dA, dB, dbias (dbias may be null).  ws holds
// parts x partial_stride floats of row-range partials followed by one grid-barrier word
// (tc_backward_workspace_extra bytes).  l1 != 0 adds l1 * sign(S) to dS.
cudaError_t tc_backward(const void *x, const void *S, const void *A, const void *B,
                        const void *dY, void *dX, float *ws, int parts, const Shape &s,
                        float *dS, float *dA, float *dB, float *dbias, bool bf16, double l1,
                        cudaStream_t st);
constexpr size_t tc_backward_workspace_extra = 256;
// Device error word of the tensor-core kernels (bounded waits); -1 if unreadable.
int tc_read_device_error(bool clear);

// ---- deterministic reduction of the row-range partials (reduce.cu) ----
// S and A are float (is_bf16 = false) or bfloat16 (is_bf16 = true).  l1 != 0 adds
// l1 * sign(S) to dS.  parts == 0 reads nothing from ws (every partial sum is zero).
cudaError_t reduce_partials(const float *ws, int parts, const void *S, const void *A,
                            bool is_bf16, float *dS, float *dA, float *dB, float *dbias,
                            const Shape &s, double l1, cudaStream_t st);

// sign(v) in {-1, 0, +1} (0 for zero and NaN): the subgradient of |v| that autograd takes.
__host__ __device__ inline double sign_of(float v) { return (double)((v > 0.f) - (v < 0.f)); }

}  // namespace kron
