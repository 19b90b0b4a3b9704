// noalloc.cu -- kron_linear_backward_noalloc: the backward for callers that cannot
// allocate device memory at the time they call it.
//
// The backward needs device scratch for its row-range partial sums.  Here that scratch
// is a fixed array compiled into the library (every GPU that loads the library holds
// it until the process exits), so the caller passes only inputs and outputs.  All
// calls share the array; calls that overlap on the GPU (e.g. on two streams) race on
// it.  Nothing in it has to start at zero except the grid-barrier word of the
// tensor-core backward, which the backward itself zeroes with an asynchronous memset on
// the caller's stream before every launch; every other value is written before it is
// read.
#include "../../include/kron_linear.h"
#include "internal.h"

#include <mutex>
#include <stdio.h>

namespace kron {
kron_status_t report_failure(kron_status_t st, const char *msg);
kron_status_t validate_backward(const void *x, const void *S, const void *A, const void *B,
                                const void *dY, const void *dX, const void *dS, const void *dA,
                                const void *dB, const void *dbias, int64_t N, int p, int q,
                                int m1, int m2, int r, kron_dtype_t dtype, unsigned flags);
}  // namespace kron

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[KRON_NOALLOC_SCRATCH_BYTES];

// Device address of the scratch array in the current context.  In host code the name
// g_noalloc_scratch is only a host-side stand-in; the device address comes from
// cudaGetSymbolAddress, called with the device current.  The address belongs to one
// context, so it is cached per device together with that context's id and looked up
// again whenever the context changes (after cudaDeviceReset, or under a context the
// caller made current through the driver API).
cudaError_t scratch_address(void **out) {
    struct Slot { unsigned long long ctx; void *addr; };
    static Slot slots[64] = {};
    static std::mutex mu;
    int dev = 0;
    unsigned long long ctx = 0;
    cudaError_t e = kron::tc::current_context_id(&dev, &ctx);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!slots[dev].addr || slots[dev].ctx != ctx) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        slots[dev] = Slot{ctx, p};
    }
    *out = slots[dev].addr;
    return cudaSuccess;
}

}  // namespace

extern "C" kron_status_t kron_linear_backward_noalloc(
    const void *x, const void *S, const void *A, const void *B, const void *dY, void *dX,
    void *dS, void *dA, void *dB, void *dbias, int64_t N, int p, int q, int m1, int m2, int r,
    kron_dtype_t dtype, unsigned flags, void *stream) {
    // 1. the same host-side checks as kron_linear_backward, before any CUDA call
    const kron_status_t st = kron::validate_backward(x, S, A, B, dY, dX, dS, dA, dB, dbias, N, p,
                                                     q, m1, m2, r, dtype, flags);
    if (st != KRON_OK) return st;
    // an empty batch needs no scratch: the workspace entry point zeroes the gradients
    if (N == 0)
        return kron_linear_backward(x, S, A, B, dY, dX, dS, dA, dB, dbias, N, p, q, m1, m2, r,
                                    dtype, flags, nullptr, 0, stream);
    // 2. the size limit of the fixed array
    const size_t need = kron_linear_workspace_size(N, p, q, m1, m2, r, dtype);
    if (need > KRON_NOALLOC_SCRATCH_BYTES) {
        char msg[200];
        snprintf(msg, sizeof(msg),
                 "this problem needs %zu bytes of scratch; the library's fixed scratch holds %zu "
                 "(use kron_linear_backward with a caller-owned workspace)",
                 need, (size_t)KRON_NOALLOC_SCRATCH_BYTES);
        return kron::report_failure(KRON_ERR_WORKSPACE, msg);
    }
    // 3. the array's device address in the current context
    void *ws = nullptr;
    const cudaError_t e = scratch_address(&ws);
    if (e != cudaSuccess) {
        char msg[200];
        snprintf(msg, sizeof(msg), "address of the fixed scratch: %s", cudaGetErrorString(e));
        return kron::report_failure(KRON_ERR_CUDA, msg);
    }
    return kron_linear_backward(x, S, A, B, dY, dX, dS, dA, dB, dbias, N, p, q, m1, m2, r, dtype,
                                flags, ws, KRON_NOALLOC_SCRATCH_BYTES, stream);
}
