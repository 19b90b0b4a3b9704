// tc_dispatch.cu -- which tensor-core kernels run a TF32 or BF16 call.
//
// The tutorial layer's shape (p = q = m1 = m2 = 32, r = 4) runs the tuned kernels of
// tc_fwd.cu and tc_bwd.cu; the other compiled shapes run the generic kernels of
// tc_gen_fwd.cu and tc_gen_pgrad.cu.  Every other shape is refused with
// KRON_ERR_UNSUPPORTED by the caller (api.cu); nothing falls back to another path.
#include "internal.h"

namespace kron {

namespace {

bool tuned_backward(const Shape &s, bool bf16) {
    return tc::tuned_pgrad_supported(s, bf16) &&
           tc::tuned_fwd_supported(tc::transposed(s), bf16, true);
}

bool generic_backward(const Shape &s, bool bf16) {
    return tc::generic_pgrad_supported(s, bf16) &&
           tc::generic_fwd_supported(tc::transposed(s), bf16, true);
}

}  // namespace

bool tc_forward_supported(const Shape &s, bool bf16) {
    return tc::tuned_fwd_supported(s, bf16, false) || tc::generic_fwd_supported(s, bf16, false);
}

cudaError_t tc_forward(const void *x, const void *S, const void *A, const void *B,
                       const void *bias, void *y, const Shape &s, bool bf16, bool skip,
                       cudaStream_t st) {
    // the tuned kernels' shape has an element-wise sparse S (no all-zero MMA tile to skip)
    if (tc::tuned_fwd_supported(s, bf16, false))
        return tc::tuned_fwd(x, S, A, B, bias, y, s, bf16, false, st);
    if (tc::generic_fwd_supported(s, bf16, false))
        return tc::generic_fwd(x, S, A, B, bias, y, s, bf16, false, skip, st);
    return cudaErrorNotSupported;
}

bool tc_backward_supported(const Shape &s, bool bf16) {
    return tuned_backward(s, bf16) || generic_backward(s, bf16);
}

int tc_backward_tile_rows(const Shape &s, bool bf16) {
    if (tuned_backward(s, bf16)) return 2;
    return tc::generic_pgrad_tile_rows(s, bf16);
}

int tc_backward_max_parts(const Shape &s, bool bf16) {
    if (tuned_backward(s, bf16)) return kRowParts;
    return tc::generic_pgrad_max_parts(s, bf16);
}

cudaError_t tc_backward(const void *x, const void *S, const void *A, const void *B,
                        const void *dY, void *dX, float *ws, int parts, const Shape &s,
                        float *dS, float *dA, float *dB, float *dbias, bool bf16, bool skip,
                        double l1, cudaStream_t st) {
    cudaError_t e = cudaSuccess;
    if (tuned_backward(s, bf16)) {
        if (dX) {
            e = tc::tuned_fwd(dY, S, A, B, nullptr, dX, tc::transposed(s), bf16, true, st);
            if (e != cudaSuccess) return e;
        }
        return tc::tuned_pgrad(x, S, A, B, dY, ws, parts, s, dS, dA, dB, dbias, bf16, l1, st);
    }
    if (!generic_backward(s, bf16)) return cudaErrorNotSupported;
    if (dX) {
        e = tc::generic_fwd(dY, S, A, B, nullptr, dX, tc::transposed(s), bf16, true, skip, st);
        if (e != cudaSuccess) return e;
    }
    return tc::generic_pgrad(x, S, A, B, dY, ws, parts, s, dS, dA, dB, dbias, bf16, l1, st);
}

}  // namespace kron
