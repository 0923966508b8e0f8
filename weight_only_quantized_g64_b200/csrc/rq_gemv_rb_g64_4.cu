// rq_gemv_rb_g64_4.cu -- row-block decode kernels for the group-64 format, int4.
#include "rq_gemv_rb.cuh"

namespace rq {

cudaError_t rb_run_g64_4(RbParams& prm, const RbPlan& P, const uint16_t* const* x,
                         const void* const* codes, int nmat, cudaStream_t s) {
    const bool ssc = prm.ssc != 0;
    if (prm.M <= 8)
        return ssc ? rb_dispatch_mt<FMT_G64, 4, 1, true>(prm, P, x, codes, nmat, s)
                   : rb_dispatch_mt<FMT_G64, 4, 1, false>(prm, P, x, codes, nmat, s);
    if (prm.M <= 16)
        return ssc ? rb_dispatch_mt<FMT_G64, 4, 2, true>(prm, P, x, codes, nmat, s)
                   : rb_dispatch_mt<FMT_G64, 4, 2, false>(prm, P, x, codes, nmat, s);
    return ssc ? rb_dispatch_mt<FMT_G64, 4, 4, true>(prm, P, x, codes, nmat, s)
               : rb_dispatch_mt<FMT_G64, 4, 4, false>(prm, P, x, codes, nmat, s);
}

}  // namespace rq
