// rq_gemv_rb_g64_8.cu -- row-block decode kernels for the group-64 format, int8.
#include "rq_gemv_rb.cuh"

namespace rq {

cudaError_t rb_run_g64_8(RbParams& prm, const RbPlan& P, const uint16_t* const* x,
                         const void* const* codes, int nmat, cudaStream_t s) {
    const bool ssc = prm.ssc != 0;
    if (prm.M <= 8)
        return ssc ? rb_dispatch_mt<FMT_G64, 8, 1, true>(prm, P, x, codes, nmat, s)
                   : rb_dispatch_mt<FMT_G64, 8, 1, false>(prm, P, x, codes, nmat, s);
    if (prm.M <= 16)
        return ssc ? rb_dispatch_mt<FMT_G64, 8, 2, true>(prm, P, x, codes, nmat, s)
                   : rb_dispatch_mt<FMT_G64, 8, 2, false>(prm, P, x, codes, nmat, s);
    return ssc ? rb_dispatch_mt<FMT_G64, 8, 4, true>(prm, P, x, codes, nmat, s)
               : rb_dispatch_mt<FMT_G64, 8, 4, false>(prm, P, x, codes, nmat, s);
}

}  // namespace rq
