// rq_gemv_rb_p8.cu -- row-block decode kernels for the int8 preset
// (symmetric, groups of 16).
#include "rq_gemv_rb.cuh"

namespace rq {

cudaError_t rb_run_p8(RbParams& prm, const RbPlan& P, const uint16_t* const* x,
                      const void* const* codes, int nmat, cudaStream_t s) {
    if (prm.M <= 8) return rb_dispatch_mt<FMT_P8, 8, 1, true>(prm, P, x, codes, nmat, s);
    if (prm.M <= 16) return rb_dispatch_mt<FMT_P8, 8, 2, true>(prm, P, x, codes, nmat, s);
    return rb_dispatch_mt<FMT_P8, 8, 4, true>(prm, P, x, codes, nmat, s);
}

}  // namespace rq
