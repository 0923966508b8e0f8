// rq_gemv_rb_p4a.cu -- row-block decode kernels for the int4 preset
// (asymmetric, groups of 32 in super-blocks).
#include "rq_gemv_rb.cuh"

namespace rq {

cudaError_t rb_run_p4a(RbParams& prm, const RbPlan& P, const uint16_t* const* x,
                       const void* const* codes, int nmat, cudaStream_t s) {
    if (prm.M <= 8) return rb_dispatch_mt<FMT_P4A, 4, 1, true>(prm, P, x, codes, nmat, s);
    if (prm.M <= 16) return rb_dispatch_mt<FMT_P4A, 4, 2, true>(prm, P, x, codes, nmat, s);
    return rb_dispatch_mt<FMT_P4A, 4, 4, true>(prm, P, x, codes, nmat, s);
}

}  // namespace rq
