// tc_host.cu -- host-side helpers of the tensor-core kernels: TMA tensor maps, the device
// error word of the bounded waits, and the identity of the current CUDA context that keys
// every cached device address.
#include "internal.h"

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <mutex>

namespace kron {
namespace tc {

// Device error word: bit 0 = an mbarrier wait gave up, bit 1 = the grid barrier gave up.
__device__ int g_device_error = 0;

namespace {

template <typename F>
F driver_entry(const char *name) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
        return reinterpret_cast<F>(p);
    return nullptr;
}

using CtxGetCurrentFn = CUresult (*)(CUcontext *);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);

}  // namespace

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        fn = driver_entry<PFN_cuTensorMapEncodeTiled_v12000>("cuTensorMapEncodeTiled");
    });
    return fn;
}

cudaError_t current_context_id(int *dev, unsigned long long *id) {
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        get_current = driver_entry<CtxGetCurrentFn>("cuCtxGetCurrent");
        get_id = driver_entry<CtxGetIdFn>("cuCtxGetId");
    });
    cudaError_t e = cudaGetDevice(dev);
    if (e != cudaSuccess) return e;
    if (!get_current || !get_id) return cudaErrorNotSupported;
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS) return cudaErrorDeviceUninitialized;
    if (!ctx) {
        // no context bound to this thread yet (its first CUDA call): bind the device's
        // primary context, as the runtime does for a launch (legal under stream capture,
        // unlike calls that synchronise)
        e = cudaSetDevice(*dev);
        if (e != cudaSuccess) return e;
        if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return cudaErrorDeviceUninitialized;
    }
    if (get_id(ctx, id) != CUDA_SUCCESS) return cudaErrorDeviceUninitialized;
    return cudaSuccess;
}

// 2-D tensor map of a row-major [rows][cols] matrix, box = box_cols x box_rows, swizzled
// by sw bytes (128, 64, 32 or 0); atom32 selects the 128-byte swizzle with 32-byte atoms
// (the shared-memory layout of MN-major TF32 MMA operands).
cudaError_t make_tmap_2d(CUtensorMap *map, const void *base, bool bf16, uint64_t rows,
                         uint64_t cols, uint32_t box_cols, uint32_t box_rows, int sw,
                         bool atom32) {
    auto enc = get_encode();
    if (!enc) return cudaErrorNotSupported;
    // The encoder is a driver-API call: make the current device's primary context current
    // on this host thread first (a thread whose first CUDA call this is has none bound).
    int dev = 0;
    cudaError_t ce = cudaGetDevice(&dev);
    if (ce == cudaSuccess) ce = cudaSetDevice(dev);
    if (ce != cudaSuccess) return ce;
    const int E = bf16 ? 2 : 4;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * E};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUtensorMapSwizzle swm = atom32      ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B
                           : sw == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                           : sw == 64  ? CU_TENSOR_MAP_SWIZZLE_64B
                           : sw == 32  ? CU_TENSOR_MAP_SWIZZLE_32B
                                       : CU_TENSOR_MAP_SWIZZLE_NONE;
    CUresult r = enc(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                     2, const_cast<void *>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, swm, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// Address of the device error word in the current context.  Cached per device together
// with the context's id, and looked up again whenever the context changes (a context
// created after cudaDeviceReset, or one the caller made current through the driver API).
int *device_error_ptr() {
    struct Slot { unsigned long long ctx; int *ptr; };
    static Slot slots[64] = {};
    static std::mutex mu;
    int dev = 0;
    unsigned long long id = 0;
    if (current_context_id(&dev, &id) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!slots[dev].ptr || slots[dev].ctx != id) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
        slots[dev] = Slot{id, static_cast<int *>(p)};
    }
    return slots[dev].ptr;
}

int num_sms() {
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

}  // namespace tc

int tc_read_device_error(bool clear) {
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, tc::g_device_error, sizeof(int)) != cudaSuccess) return -1;
    if (clear && v) {
        const int z = 0;
        cudaMemcpyToSymbol(tc::g_device_error, &z, sizeof(int));
    }
    return v;
}

}  // namespace kron
