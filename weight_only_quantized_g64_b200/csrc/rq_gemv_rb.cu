// rq_gemv_rb.cu -- host side of the row-block decode kernel (rq_gemv_rb.cuh):
// how a product is cut into blocks and slots, and the launch entry points.
#include <cstring>

#include "rq_gemv_rb.cuh"

namespace rq {

int num_sms() {
    static int sms[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (sms[dev] == 0) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) v = 0;
        sms[dev] = v > 0 ? v : 148;
    }
    return sms[dev];
}

#ifndef RQ_RB_SMEM_BUDGET
#define RQ_RB_SMEM_BUDGET (227 * 1024)
#endif
constexpr int kRbMaxTC = 8;                       // m-tiles per block at most

static int rb_align(int v, int a) { return (v + a - 1) / a * a; }

// fmt: FMT_G64 (bits 4 or 8), FMT_P8 (bits 8), FMT_P4A (bits 4).
static bool rb_plan(int64_t M, int64_t K, int64_t N, int bits, int nmat, int fmt, RbPlan* P) {
    const int GPS = bits == 4 ? 4 : 2;
    const int sms = num_sms();
    const int64_t tm = (N + 15) / 16;                 // m-tiles per matrix
    const int64_t T = tm * nmat;
    int64_t tc = (T + sms - 1) / sms;
    if (tc > kRbMaxTC) tc = kRbMaxTC;
    if (fmt != FMT_G64 && M > 16 && tc > 4) tc = 4;   // (taller preset blocks spill at M > 16)
    if (tc < 1) tc = 1;
    P->tc = static_cast<int>(tc);
    P->bpm = static_cast<int>((tm + tc - 1) / tc);
    P->nblocks = P->bpm * nmat;
    P->grid = P->nblocks < sms ? P->nblocks : sms;
    const int RB = 16 * P->tc;
    const int64_t row_bytes = K * bits / 8;
    P->stages = static_cast<int>((row_bytes + 127) / 128);
    P->three_d = row_bytes % 128 == 0;
    // stages per slot: about 16 KB of codes, at least 16 group columns (two
    // per warp, processed together) for M <= 8 and 8 otherwise, when the row
    // has them, and at most 16 KB of x (32 KB for M > 16).  Short blocks (one
    // or two m-tiles) take at least 32 columns and up to 32 KB of x: their
    // slots are small, and fewer, larger slots measured faster on B200.
    const bool short_blk = P->tc <= 2;
    const int smin = (M <= 8 ? (short_blk ? 32 : 16) : 8) / GPS;
    const int64_t x_cap = M > 16 || short_blk ? 32768 : 16384;
    int S = 1;
    while (S * 2 * RB * 128 <= 16384 && S < 16) S *= 2;
    if (S < smin) S = smin;
    while (S > smin && static_cast<int64_t>(S) * GPS * M * 128 > x_cap) S /= 2;
    // the int8 preset stages 4 scales per column in a row of kRbSrowP8
    if (fmt == FMT_P8)
        while (S * GPS > 16) S /= 2;
    if (S > P->stages) S = P->stages;
    P->S = S;
    P->J = S * GPS;
    P->slots = (P->stages + S - 1) / S;
    // staged metadata row: elements of the scale map's box and its bytes
    int srow_bytes;
    if (fmt == FMT_P8) {
        if (P->J > 16) return false;
        P->srow = kRbSrowP8;
        srow_bytes = 2 * kRbSrowP8;
    } else if (fmt == FMT_P4A) {
        P->srow = 4 * P->J;          // (a, b) of the slot's 2 J groups
        srow_bytes = P->srow;
    } else {
        P->srow = kRbSrow;
        srow_bytes = 2 * kRbSrow;
    }
    const int cbytes = RB * 128 * S;
    P->s_off = cbytes;
    P->x_off = rb_align(P->s_off + RB * srow_bytes, 1024);
    P->slot_bytes = rb_align(P->x_off + P->J * static_cast<int>(M) * 128, 1024);
    P->red_stride = RB + 4;
    const int red_bytes = kRbWarps * 8 * P->red_stride * 4;
    const int per_cta = (P->nblocks + P->grid - 1) / P->grid;
    int want = P->slots * per_cta;
    if (want > kRbMaxSG) want = kRbMaxSG;
    for (int sg = want; sg >= 1; --sg) {
        const int ring = sg * P->slot_bytes > red_bytes ? sg * P->slot_bytes : rb_align(red_bytes, 1024);
        const int bar_off = ring;
        const int smem = 1024 + bar_off + static_cast<int>(sizeof(RbBars));
        if (smem <= RQ_RB_SMEM_BUDGET) {
            P->sg = sg;
            P->bar_off = bar_off;
            P->smem = smem;
            return true;
        }
    }
    return false;
}

bool gemv_rowblock_fits(int64_t M, int64_t K, int64_t N, int bits, int nmat, int fmt) {
    if (M < 1 || M > 32) return false;
    if (fmt == FMT_P8 && (bits != 8 || K % 128 != 0)) return false;
    if (fmt == FMT_P4A && (bits != 4 || K % 256 != 0)) return false;
    RbPlan P;
    return rb_plan(M, K, N, bits, nmat, fmt, &P);
}

cudaError_t launch_gemv_rowblock(const uint16_t* x, int64_t M, int64_t K, int64_t N, int bits,
                                 const WOperand* w, int nmat, cudaStream_t s) {
    const uint16_t* xs[1] = {x};
    return launch_gemv_rowblock_ex(xs, 1, M, K, N, bits, w, nmat, false, 0, s);
}

cudaError_t launch_gemv_rowblock_ex(const uint16_t* const* xs, int nx, int64_t M, int64_t K,
                                    int64_t N, int bits, const WOperand* w, int nmat, bool y_half,
                                    int epilogue, cudaStream_t s) {
    return launch_gemv_rowblock_fmt(xs, nx, M, K, N, bits, FMT_G64, w, nullptr, nmat, y_half,
                                    epilogue, s);
}

cudaError_t launch_gemv_rowblock_fmt(const uint16_t* const* xs, int nx, int64_t M, int64_t K,
                                     int64_t N, int bits, int fmt, const WOperand* w,
                                     const uint32_t* const* sup, int nmat, bool y_half,
                                     int epilogue, cudaStream_t s) {
    RbPlan P;
    const uint16_t* const* x = xs;
    if (!gemv_rowblock_fits(M, K, N, bits, nmat, fmt) || !rb_plan(M, K, N, bits, nmat, fmt, &P))
        return cudaErrorInvalidValue;
    if (fmt == FMT_P4A && sup == nullptr) return cudaErrorInvalidValue;
    RbParams prm;
    memset(&prm, 0, sizeof(prm));
    prm.M = static_cast<int>(M);
    prm.N = static_cast<int>(N);
    prm.K = static_cast<int>(K);
    prm.groups = static_cast<int>(K / kGroup);
    prm.stages = P.stages;
    prm.tc = P.tc;
    prm.bpm = P.bpm;
    prm.nblocks = P.nblocks;
    prm.S = P.S;
    prm.J = P.J;
    prm.slots = P.slots;
    prm.sg = P.sg;
    prm.three_d = P.three_d ? 1 : 0;
    // presets always stage their metadata (their K keeps every row 16-byte aligned)
    prm.ssc = fmt != FMT_G64 || (prm.groups * 2) % 16 == 0 ? 1 : 0;
    prm.srow = P.srow;
    prm.slot_bytes = P.slot_bytes;
    prm.s_off = P.s_off;
    prm.x_off = P.x_off;
    prm.bar_off = P.bar_off;
    prm.red_stride = P.red_stride;
    prm.nx = nx;
    prm.nsb = static_cast<int>(K / 256);
    prm.yh = y_half ? 1 : 0;
    prm.epi = epilogue;
    prm.status = device_status_ptr();
    prm.timeout_ns = wait_limit_ns();
    const void* codes[3] = {nullptr, nullptr, nullptr};
    for (int i = 0; i < nmat; ++i) {
        codes[i] = w[i].codes;
        prm.scales[i] = w[i].scales;
        prm.y[i] = w[i].y;
        prm.sup[i] = fmt == FMT_P4A ? sup[i] : nullptr;
    }
    if (fmt == FMT_P8) return rb_run_p8(prm, P, x, codes, nmat, s);
    if (fmt == FMT_P4A) return rb_run_p4a(prm, P, x, codes, nmat, s);
    return bits == 4 ? rb_run_g64_4(prm, P, x, codes, nmat, s) : rb_run_g64_8(prm, P, x, codes, nmat, s);
}

}  // namespace rq
