// tc_dispatch.cu -- which tensor-core kernels run a TF32 or BF16 call.
//
// The tutorial layer's shape (p = q = m1 = m2 = 32, r = 4) runs the tuned kernels of
// tc_fwd.cu and tc_bwd.cu.  Every shape without a tensor-core kernel is refused with
// KRON_ERR_UNSUPPORTED by the caller (api.cu); nothing falls back to another path.
#include "internal.h"

namespace kron {

bool tc_forward_supported(const Shape &s, bool bf16) {
    return tc::tuned_fwd_supported(s, bf16, false);
}

cudaError_t tc_forward(const void *x, const void *S, const void *A, const void *B,
                       const void *bias, void *y, const Shape &s, bool bf16, bool skip,
                       cudaStream_t st) {
    // the tuned kernels' shape has an element-wise sparse S and no all-zero tile to skip
    (void)skip;
    if (tc::tuned_fwd_supported(s, bf16, false))
        return tc::tuned_fwd(x, S, A, B, bias, y, s, bf16, false, st);
    return cudaErrorNotSupported;
}

bool tc_backward_supported(const Shape &s, bool bf16) {
    return tc::tuned_pgrad_supported(s, bf16) &&
           tc::tuned_fwd_supported(tc::transposed(s), bf16, true);
}

int tc_backward_tile_rows(const Shape &, bool) { return 2; }

int tc_backward_max_parts(const Shape &, bool) { return kRowParts; }

cudaError_t tc_backward(const void *x, const void *S, const void *A, const void *B,
                        const void *dY, void *dX, float *ws, int parts, const Shape &s,
                        float *dS, float *dA, float *dB, float *dbias, bool bf16, bool skip,
                        double l1, cudaStream_t st) {
    (void)skip;
    if (!tc_backward_supported(s, bf16)) return cudaErrorNotSupported;
    if (dX) {
        const cudaError_t e =
            tc::tuned_fwd(dY, S, A, B, nullptr, dX, tc::transposed(s), bf16, true, st);
        if (e != cudaSuccess) return e;
    }
    return tc::tuned_pgrad(x, S, A, B, dY, ws, parts, s, dS, dA, dB, dbias, bf16, l1, st);
}

}  // namespace kron
