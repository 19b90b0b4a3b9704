// api.cu -- the extern "C" entry points of libkronlinear.so (include/kron_linear.h):
// host-side validation, then dispatch to the kernels of the requested path.
// Nothing here computes any part of the layer.
#include "../../include/kron_linear.h"
#include "internal.h"

#include <stdarg.h>
#include <stdio.h>
#include <string.h>

namespace kron {
const char *&launch_step() {
    thread_local const char *step = "launch";
    return step;
}
}  // namespace kron

namespace {

thread_local char g_last_error[256] = "";

kron_status_t fail(kron_status_t st, const char *fmt, ...) __attribute__((format(printf, 2, 3)));
kron_status_t fail(kron_status_t st, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
    va_end(ap);
    return st;
}

kron_status_t cuda_fail(cudaError_t e, const char *what) {
    return fail(KRON_ERR_CUDA, "%s (%s): %s", what, kron::launch_step(), cudaGetErrorString(e));
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

kron_status_t check_shape(int64_t N, int p, int q, int m1, int m2, int r, kron_dtype_t dtype,
                          unsigned flags) {
    if (dtype != KRON_F32 && dtype != KRON_TF32 && dtype != KRON_BF16)
        return fail(KRON_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
    if (flags & ~KRON_FLAG_SKIP_ZERO_BLOCKS)
        return fail(KRON_ERR_INVALID_ARG, "unknown flag bits 0x%x", flags);
    if (N < 0 || p < 1 || q < 1 || m1 < 1 || m2 < 1 || r < 1)
        return fail(KRON_ERR_INVALID_ARG,
                    "sizes must be N >= 0 and p, q, m1, m2, r >= 1 (got N=%lld p=%d q=%d m1=%d "
                    "m2=%d r=%d)", (long long)N, p, q, m1, m2, r);
    if ((int64_t)p * m1 > (1 << 20) || (int64_t)q * m2 > (1 << 20) || r > 4096 ||
        N > ((int64_t)1 << 40))
        return fail(KRON_ERR_INVALID_ARG, "sizes out of range");
    const int mult = dtype == KRON_BF16 ? 8 : 4;
    if (m1 % mult || m2 % mult)
        return fail(KRON_ERR_UNSUPPORTED, "m1 and m2 must be multiples of %d for this dtype", mult);
    return KRON_OK;
}

// True when the backward of this shape and dtype runs on the tensor-core kernels (the TF32
// and BF16 paths); KRON_F32 always runs the CUDA-core kernels.
bool tc_backward_path(const kron::Shape &s, kron_dtype_t dtype) {
    return dtype != KRON_F32 && kron::tc_backward_supported(s, dtype == KRON_BF16);
}

// True when some kernel of the requested path takes this shape.
bool backward_path_exists(const kron::Shape &s, kron_dtype_t dtype) {
    return dtype == KRON_F32 ? kron::simt_backward_rows(s) > 0 : tc_backward_path(s, dtype);
}

// Number of contiguous row ranges of the backward: at most the path's maximum, none empty.
// A function of the shape and path only, so the summation order is fixed.
int backward_parts(const kron::Shape &s, kron_dtype_t dtype) {
    int rows_per_tile = 0, max_parts = kron::kRowParts;
    if (tc_backward_path(s, dtype)) {
        rows_per_tile = kron::tc_backward_tile_rows(s, dtype == KRON_BF16);
        max_parts = kron::tc_backward_max_parts(s, dtype == KRON_BF16);
    } else if (dtype == KRON_F32) {
        rows_per_tile = kron::simt_backward_rows(s);
    }
    if (rows_per_tile <= 0 || max_parts <= 0) return 0;
    int64_t tiles = (s.N + rows_per_tile - 1) / rows_per_tile;
    if (tiles < 1) tiles = 1;
    const int64_t parts0 = tiles < max_parts ? tiles : max_parts;
    const int64_t per = (tiles + parts0 - 1) / parts0;
    return (int)((tiles + per - 1) / per);
}

}  // namespace

// Host-side checks shared by every backward entry point: sizes, dtype, flags, the l1
// weight, pointers, alignment, and that the requested path has a kernel for the shape.
// Touches no CUDA state.
static kron_status_t check_backward(const void *x, const void *S, const void *A, const void *B,
                                    const void *dY, const void *dX, const void *dS,
                                    const void *dA, const void *dB, const void *dbias, int64_t N,
                                    int p, int q, int m1, int m2, int r, kron_dtype_t dtype,
                                    unsigned flags, double l1) {
    kron_status_t st = check_shape(N, p, q, m1, m2, r, dtype, flags);
    if (st != KRON_OK) return st;
    if (!(l1 >= 0.0 && l1 <= 1e30))
        return fail(KRON_ERR_INVALID_ARG, "the l1 weight must be in [0, 1e30] (got %g)", l1);
    if (!S || !A || !B || !dS || !dA || !dB || (N > 0 && (!x || !dY)))
        return fail(KRON_ERR_INVALID_ARG,
                    "S, A, B, dS, dA, dB (and x, dY when N > 0) must be non-null");
    if (!aligned16(x) || !aligned16(S) || !aligned16(A) || !aligned16(B) || !aligned16(dY) ||
        !aligned16(dS) || !aligned16(dA) || !aligned16(dB) || (dX && !aligned16(dX)) ||
        (dbias && !aligned16(dbias)))
        return fail(KRON_ERR_ALIGNMENT, "all tensors must be 16-byte aligned");
    const kron::Shape s{N, p, q, m1, m2, r};
    if (N > 0 && !backward_path_exists(s, dtype)) {
        if (dtype == KRON_F32)
            return fail(KRON_ERR_UNSUPPORTED,
                        "no kernel for p=%d q=%d m1=%d m2=%d r=%d: the FP32 tile does not fit "
                        "shared memory", p, q, m1, m2, r);
        return fail(KRON_ERR_UNSUPPORTED,
                    "no tensor-core kernel for p=%d q=%d m1=%d m2=%d r=%d on the %s path "
                    "(KRON_F32 runs any shape)", p, q, m1, m2, r,
                    dtype == KRON_BF16 ? "BF16" : "TF32");
    }
    return KRON_OK;
}

namespace kron {
// Records a failure in this thread's last-error string (for entry points in other files).
kron_status_t report_failure(kron_status_t st, const char *msg) { return fail(st, "%s", msg); }
}  // namespace kron

namespace kron {
// The backward's host-side checks, for entry points in other files (clears the thread's
// last-error string first, as every entry point does).
kron_status_t validate_backward(const void *x, const void *S, const void *A, const void *B,
                                const void *dY, const void *dX, const void *dS, const void *dA,
                                const void *dB, const void *dbias, int64_t N, int p, int q,
                                int m1, int m2, int r, kron_dtype_t dtype, unsigned flags) {
    g_last_error[0] = 0;
    return check_backward(x, S, A, B, dY, dX, dS, dA, dB, dbias, N, p, q, m1, m2, r, dtype,
                          flags, 0.0);
}
}  // namespace kron

extern "C" {

int kron_linear_abi_version(void) { return KRON_LINEAR_ABI_VERSION; }

const char *kron_last_error(void) { return g_last_error; }

const char *kron_status_string(kron_status_t status) {
    switch (status) {
        case KRON_OK: return "KRON_OK";
        case KRON_ERR_INVALID_ARG: return "KRON_ERR_INVALID_ARG: invalid argument";
        case KRON_ERR_UNSUPPORTED: return "KRON_ERR_UNSUPPORTED: shape or dtype not implemented";
        case KRON_ERR_ALIGNMENT: return "KRON_ERR_ALIGNMENT: pointer not 16-byte aligned";
        case KRON_ERR_WORKSPACE: return "KRON_ERR_WORKSPACE: workspace missing or too small";
        case KRON_ERR_CUDA: return "KRON_ERR_CUDA: CUDA error";
        case KRON_ERR_TIMEOUT: return "KRON_ERR_TIMEOUT: device-side wait timed out";
    }
    return "unknown kron_status_t";
}

size_t kron_linear_workspace_size(int64_t N, int p, int q, int m1, int m2, int r,
                                  kron_dtype_t dtype) {
    if (check_shape(N, p, q, m1, m2, r, dtype, 0) != KRON_OK) return 0;
    const kron::Shape s{N, p, q, m1, m2, r};
    const int parts = backward_parts(s, dtype);
    if (parts <= 0) return 0;
    return (size_t)parts * kron::partial_stride(s) * sizeof(float) +
           (tc_backward_path(s, dtype) ? kron::tc_backward_workspace_extra : 0);
}

kron_status_t kron_linear_forward(const void *x, const void *S, const void *A, const void *B,
                                  const void *bias, void *y, int64_t N, int p, int q, int m1,
                                  int m2, int r, kron_dtype_t dtype, unsigned flags,
                                  void *stream) {
    g_last_error[0] = 0;
    kron_status_t st = check_shape(N, p, q, m1, m2, r, dtype, flags);
    if (st != KRON_OK) return st;
    if (!S || !A || !B || (N > 0 && (!x || !y)))
        return fail(KRON_ERR_INVALID_ARG, "S, A, B (and x, y when N > 0) must be non-null");
    if (!aligned16(x) || !aligned16(S) || !aligned16(A) || !aligned16(B) || !aligned16(y) ||
        (bias && !aligned16(bias)))
        return fail(KRON_ERR_ALIGNMENT, "all tensors must be 16-byte aligned");
    if (N == 0) return KRON_OK;
    const kron::Shape s{N, p, q, m1, m2, r};
    cudaStream_t cs = (cudaStream_t)stream;
    cudaError_t e = cudaSuccess;
    if (dtype == KRON_F32) {
        // exact FP32 on the CUDA cores: any shape whose tile fits shared memory
        if (kron::simt_forward_rows(s) <= 0)
            return fail(KRON_ERR_UNSUPPORTED,
                        "no kernel for p=%d q=%d m1=%d m2=%d r=%d: the FP32 tile does not "
                        "fit shared memory", p, q, m1, m2, r);
        e = kron::simt_forward(x, S, A, B, bias, y, s,
                               (flags & KRON_FLAG_SKIP_ZERO_BLOCKS) != 0, cs);
    } else {
        // the tensor-core paths run only where a tcgen05 kernel exists for the shape
        const bool bf16 = dtype == KRON_BF16;
        if (!kron::tc_forward_supported(s, bf16))
            return fail(KRON_ERR_UNSUPPORTED,
                        "no tensor-core kernel for p=%d q=%d m1=%d m2=%d r=%d on the %s path "
                        "(KRON_F32 runs any shape)", p, q, m1, m2, r, bf16 ? "BF16" : "TF32");
        e = kron::tc_forward(x, S, A, B, bias, y, s, bf16,
                             (flags & KRON_FLAG_SKIP_ZERO_BLOCKS) != 0, cs);
    }
    if (e != cudaSuccess) return cuda_fail(e, "forward launch");
    return KRON_OK;
}

// Both backward entry points.  l1 is the weight of the penalty l1 * sum|S| whose gradient
// the dS epilogue adds (0: none, and then no term is added at all).
static kron_status_t backward_impl(const void *x, const void *S, const void *A, const void *B,
                                   const void *dY, void *dX, void *dS, void *dA, void *dB,
                                   void *dbias, int64_t N, int p, int q, int m1, int m2, int r,
                                   kron_dtype_t dtype, unsigned flags, double l1,
                                   void *workspace, size_t workspace_bytes, void *stream) {
    g_last_error[0] = 0;
    kron_status_t st = check_backward(x, S, A, B, dY, dX, dS, dA, dB, dbias, N, p, q, m1, m2, r,
                                      dtype, flags, l1);
    if (st != KRON_OK) return st;
    const kron::Shape s{N, p, q, m1, m2, r};
    cudaStream_t cs = (cudaStream_t)stream;
    if (N == 0 && l1 != 0.0) {  // empty batch: only the penalty's gradient l1 * sign(S)
        const cudaError_t e = kron::reduce_partials(nullptr, 0, S, A, dtype == KRON_BF16,
                                                    (float *)dS, (float *)dA, (float *)dB,
                                                    (float *)dbias, s, l1, cs);
        return e == cudaSuccess ? KRON_OK : cuda_fail(e, "penalty gradient");
    }
    if (N == 0) {  // empty batch: every gradient is zero
        cudaError_t e = cudaMemsetAsync(dS, 0, (size_t)p * q * sizeof(float), cs);
        if (e == cudaSuccess) e = cudaMemsetAsync(dA, 0, (size_t)r * p * q * sizeof(float), cs);
        if (e == cudaSuccess) e = cudaMemsetAsync(dB, 0, (size_t)r * m1 * m2 * sizeof(float), cs);
        if (e == cudaSuccess && dbias)
            e = cudaMemsetAsync(dbias, 0, (size_t)q * m2 * sizeof(float), cs);
        return e == cudaSuccess ? KRON_OK : cuda_fail(e, "zero gradients");
    }
    const bool on_tc = tc_backward_path(s, dtype);
    const size_t need = kron_linear_workspace_size(N, p, q, m1, m2, r, dtype);
    if (!workspace || workspace_bytes < need)
        return fail(KRON_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need,
                    workspace ? workspace_bytes : (size_t)0);
    if ((uintptr_t)workspace & 255u)
        return fail(KRON_ERR_ALIGNMENT, "workspace must be 256-byte aligned");
    const int parts = backward_parts(s, dtype);
    const bool skip = (flags & KRON_FLAG_SKIP_ZERO_BLOCKS) != 0;
    cudaError_t e = cudaSuccess;
    if (on_tc) {
        e = kron::tc_backward(x, S, A, B, dY, dX, (float *)workspace, parts, s, (float *)dS,
                              (float *)dA, (float *)dB, (float *)dbias, dtype == KRON_BF16, skip,
                              l1, cs);
        if (e != cudaSuccess) return cuda_fail(e, "backward launch");
    } else {
        // exact FP32 on the CUDA cores, then the fixed-order reduction of the partials
        e = kron::simt_backward(x, S, A, B, dY, dX, (float *)workspace, parts, s, skip, cs);
        if (e != cudaSuccess) return cuda_fail(e, "backward launch");
        e = kron::reduce_partials((const float *)workspace, parts, S, A, false, (float *)dS,
                                  (float *)dA, (float *)dB, (float *)dbias, s, l1, cs);
    }
    if (e != cudaSuccess) return cuda_fail(e, "reduction launch");
    return KRON_OK;
}

kron_status_t kron_linear_backward(const void *x, const void *S, const void *A, const void *B,
                                   const void *dY, void *dX, void *dS, void *dA, void *dB,
                                   void *dbias, int64_t N, int p, int q, int m1, int m2, int r,
                                   kron_dtype_t dtype, unsigned flags, void *workspace,
                                   size_t workspace_bytes, void *stream) {
    return backward_impl(x, S, A, B, dY, dX, dS, dA, dB, dbias, N, p, q, m1, m2, r, dtype, flags,
                         0.0, workspace, workspace_bytes, stream);
}

kron_status_t kron_linear_backward_l1(const void *x, const void *S, const void *A, const void *B,
                                      const void *dY, void *dX, void *dS, void *dA, void *dB,
                                      void *dbias, int64_t N, int p, int q, int m1, int m2, int r,
                                      kron_dtype_t dtype, unsigned flags, double l1,
                                      void *workspace, size_t workspace_bytes, void *stream) {
    return backward_impl(x, S, A, B, dY, dX, dS, dA, dB, dbias, N, p, q, m1, m2, r, dtype, flags,
                         l1, workspace, workspace_bytes, stream);
}

kron_status_t kron_linear_device_error(int clear) {
    const int v = kron::tc_read_device_error(clear != 0);
    if (v < 0) return fail(KRON_ERR_CUDA, "could not read the device error word");
    if (v) return fail(KRON_ERR_TIMEOUT, "a kernel's bounded wait gave up (device error 0x%x)", v);
    return KRON_OK;
}

}  // extern "C"
