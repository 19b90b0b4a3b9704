// noalloc.cu -- kron_linear_backward_noalloc: the backward for callers that cannot
// allocate device memory at the time they call it.
//
// The backward needs device scratch for its row-range partial sums.  Here that scratch
// is a fixed array compiled into the library (every GPU that loads the library holds
// it until the process exits), so the caller passes only inputs and outputs.  All
// calls share the array; calls that overlap on the GPU (e.g. on two streams) race on
// it.  Nothing in it has to start at zero: the backward kernels overwrite every value
// they later read.
#include "../../include/kron_linear.h"
#include "internal.h"

#include <mutex>
#include <stdio.h>

namespace kron {
kron_status_t report_failure(kron_status_t st, const char *msg);
}

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[KRON_NOALLOC_SCRATCH_BYTES];

// Device address of the scratch array on the current device.  In host code the name
// g_noalloc_scratch is only a host-side stand-in; the device address comes from
// cudaGetSymbolAddress, looked up once per device with that device current.
cudaError_t scratch_address(void **out) {
    static void *addr[64] = {};
    static std::mutex mu;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        addr[dev] = p;
    }
    *out = addr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" kron_status_t kron_linear_backward_noalloc(
    const void *x, const void *S, const void *A, const void *B, const void *dY, void *dX,
    void *dS, void *dA, void *dB, void *dbias, int64_t N, int p, int q, int m1, int m2, int r,
    kron_dtype_t dtype, unsigned flags, void *stream) {
    const size_t need = kron_linear_workspace_size(N, p, q, m1, m2, r, dtype);
    // need == 0: the sizes or dtype are invalid, or no kernel takes this shape; the
    // workspace entry point reports which before touching the device (and with N == 0
    // zeroes the gradients, which needs no scratch)
    if (need == 0)
        return kron_linear_backward(x, S, A, B, dY, dX, dS, dA, dB, dbias, N, p, q, m1, m2, r,
                                    dtype, flags, nullptr, 0, stream);
    if (need > KRON_NOALLOC_SCRATCH_BYTES) {
        char msg[200];
        snprintf(msg, sizeof(msg),
                 "this problem needs %zu bytes of scratch; the library's fixed scratch holds %zu "
                 "(use kron_linear_backward with a caller-owned workspace)",
                 need, (size_t)KRON_NOALLOC_SCRATCH_BYTES);
        return kron::report_failure(KRON_ERR_WORKSPACE, msg);
    }
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
