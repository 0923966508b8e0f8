// rq_api.cu -- the C ABI of include/rq.h: argument validation, dispatch to
// the kernels, TMA descriptor creation, status strings.
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>

#include "rq_internal.h"

namespace rq {

// Library-wide device status word (one per device that loads the module):
// bounded waits raise RQ_ERR_TIMEOUT here.
__device__ int g_device_status = 0;

static constexpr int kMaxDevices = 64;
static int* g_status_ptr[kMaxDevices] = {};
static std::mutex g_mu;
static bool g_pdl = false;
static uint64_t g_wait_limit_ns = 1000000000ull;  // 1 s

int* device_status_ptr() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    if (g_status_ptr[dev] == nullptr) {
        std::lock_guard<std::mutex> lk(g_mu);
        if (g_status_ptr[dev] == nullptr) {
            void* p = nullptr;
            if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
            g_status_ptr[dev] = static_cast<int*>(p);
        }
    }
    return g_status_ptr[dev];
}

uint64_t wait_limit_ns() { return g_wait_limit_ns; }
bool pdl_enabled() { return g_pdl; }

static int g_decode_kernel = RQ_DECODE_AUTO;

int decode_kernel_for(int64_t M, int64_t K, int64_t N, int bits, int nmat) {
    const bool fits = gemv_cluster_fits(M, K, bits);
    if (g_decode_kernel == RQ_DECODE_CLUSTER) return fits ? RQ_DECODE_CLUSTER : -1;
    if (g_decode_kernel == RQ_DECODE_ROWTILE) return RQ_DECODE_ROWTILE;
    if (g_decode_kernel == RQ_DECODE_ROWBLOCK)
        return gemv_rowblock_fits(M, K, N, bits, nmat) ? RQ_DECODE_ROWBLOCK : -1;
    if (g_decode_kernel == RQ_DECODE_TENSOR) return tcs_fits(M, K, N, bits) ? RQ_DECODE_TENSOR : -1;
    // measured on B200 (graph-replayed chains with PDL, int4 and int8):
    // * at least one 16-row m-tile per SM: the row-block kernel, except for
    //   M > 16 on rows of >= 16384 k or launches of >= 16384 rows, where the
    //   MMA work of mma.sync makes the tensor-core kernel faster (at M = 32:
    //   4096 x 16384 23.8 vs 29.5 us, 16384 x 4096 20.4 vs 20.9 us);
    // * fewer m-tiles than SMs: the row-tile kernel (which also splits K) for
    //   M <= 8; the row-block kernel for M 9..16 and for M > 16 on rows of
    //   <= 4096 k; the cluster kernel for M > 16 on longer rows.
    const int64_t mtiles = static_cast<int64_t>(nmat) * ((N + 15) / 16);
    if (mtiles >= num_sms()) {
        if (M > 16 && (K >= 16384 || static_cast<int64_t>(nmat) * N >= 16384) &&
            tcs_fits(M, K, N, bits))
            return RQ_DECODE_TENSOR;
        if (gemv_rowblock_fits(M, K, N, bits, nmat)) return RQ_DECODE_ROWBLOCK;
    } else if (M > 8 && (M <= 16 || K <= 4096) && gemv_rowblock_fits(M, K, N, bits, nmat)) {
        return RQ_DECODE_ROWBLOCK;
    }
    if (fits && M > 16) return RQ_DECODE_CLUSTER;
    return RQ_DECODE_ROWTILE;
}


// ------------------------------------------------------------- workspace --
// Per-device scratch of the row-tile decode kernel.  When a launch needs more
// than the current buffers hold, larger ones are allocated and the old ones
// are kept (never freed before the process exits): a CUDA graph captured
// earlier may still hold their addresses, and replaying it must not touch
// freed memory.  The old counters stay zero (every completed launch leaves
// them so), and the old slots are only ever written by replays of such graphs.
struct Workspace {
    float* ws = nullptr;
    size_t ws_bytes = 0;
    int* cnt = nullptr;
    size_t n_cnt = 0;
    int retired = 0;   // buffers replaced by larger ones and kept alive
};
static Workspace g_ws[kMaxDevices];

cudaError_t workspace_get(size_t ws_bytes, size_t n_counters, float** ws, int** cnt) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(g_mu);
    Workspace& w = g_ws[dev];
    if (w.ws_bytes < ws_bytes) {
        const size_t want = ws_bytes > (size_t{32} << 20) ? ws_bytes : (size_t{32} << 20);
        void* p = nullptr;
        e = cudaMalloc(&p, want);
        if (e != cudaSuccess) return e;
        if (w.ws != nullptr) ++w.retired;
        w.ws = static_cast<float*>(p);
        w.ws_bytes = want;
    }
    if (w.n_cnt < n_counters) {
        const size_t want = n_counters > (size_t{1} << 18) ? n_counters : (size_t{1} << 18);
        void* p = nullptr;
        e = cudaMalloc(&p, want * sizeof(int));
        if (e != cudaSuccess) return e;
        e = cudaMemset(p, 0, want * sizeof(int));
        if (e != cudaSuccess) return e;
        e = cudaDeviceSynchronize();
        if (e != cudaSuccess) return e;
        if (w.cnt != nullptr) ++w.retired;
        w.cnt = static_cast<int*>(p);
        w.n_cnt = want;
    }
    *ws = w.ws;
    *cnt = w.cnt;
    return cudaSuccess;
}

cudaError_t workspace_reset_counters() {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(g_mu);
    Workspace& w = g_ws[dev];
    if (w.cnt == nullptr) return cudaSuccess;
    e = cudaMemset(w.cnt, 0, w.n_cnt * sizeof(int));
    if (e != cudaSuccess) return e;
    return cudaDeviceSynchronize();
}

// ------------------------------------------------------------ tensor maps --
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

bool make_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base,
                  uint64_t inner_elems, uint64_t rows, uint64_t row_stride_bytes,
                  uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle swz) {
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return false;
    cuuint64_t dims[2] = {inner_elems, rows};
    cuuint64_t strides[1] = {row_stride_bytes};
    cuuint32_t box[2] = {box_inner, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool make_tmap_3d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t d0,
                  uint64_t d1, uint64_t d2, uint64_t s1, uint64_t s2, uint32_t b0, uint32_t b1,
                  uint32_t b2, CUtensorMapSwizzle swz) {
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return false;
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {s1, s2};
    cuuint32_t box[3] = {b0, b1, b2};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, dtype, 3, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace rq

using namespace rq;

static thread_local std::string t_last_cuda_error;

void rq::record_cuda_error(cudaError_t e) { t_last_cuda_error = cudaGetErrorString(e); }

static rq_status cuda_fail(cudaError_t e) {
    t_last_cuda_error = cudaGetErrorString(e);
    return RQ_ERR_CUDA;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static rq_status check_weight_shape(int64_t N, int64_t K, int bits) {
    if (bits != 4 && bits != 8) return RQ_ERR_BITS;
    if (N < 1 || K < kGroup || K % kGroup != 0) return RQ_ERR_SHAPE;
    if (N > (int64_t{1} << 31) - 1 || K > (int64_t{1} << 30)) return RQ_ERR_SHAPE;
    return RQ_OK;
}

static rq_status check_product(const uint16_t* x, int64_t M, int64_t K, int64_t N, int bits,
                               int64_t max_m) {
    rq_status st = check_weight_shape(N, K, bits);
    if (st != RQ_OK) return st;
    if (M < 1 || M > max_m) return RQ_ERR_SHAPE;
    if (x == nullptr) return RQ_ERR_NULL;
    if (!aligned16(x)) return RQ_ERR_ALIGN;
    return RQ_OK;
}

static rq_status check_operand(const void* codes, const uint16_t* scales, const float* y) {
    if (codes == nullptr || scales == nullptr || y == nullptr) return RQ_ERR_NULL;
    if (!aligned16(codes) || !aligned16(scales) || !aligned16(y)) return RQ_ERR_ALIGN;
    return RQ_OK;
}

static rq_status launch_decode(const uint16_t* x, int64_t M, int64_t K, int64_t N, int bits,
                               const WOperand* w, int nmat, cudaStream_t s) {
    const int which = decode_kernel_for(M, K, N, bits, nmat);
    if (which < 0) return RQ_ERR_SHAPE;
    const uint16_t* xs[1] = {x};
    const cudaError_t e =
        which == RQ_DECODE_CLUSTER    ? launch_gemv_cluster(x, M, K, N, bits, w, nmat, s)
        : which == RQ_DECODE_ROWBLOCK ? launch_gemv_rowblock(x, M, K, N, bits, w, nmat, s)
        : which == RQ_DECODE_TENSOR   ? launch_tcs(xs, 1, M, K, N, bits, w, nmat, false, 0, s)
                                      : launch_gemv_product(x, M, K, N, bits, w, nmat, s);
    return e == cudaSuccess ? RQ_OK : cuda_fail(e);
}

// The decode variants (per-matrix inputs, fp16 output, fused epilogue) run on
// the tensor-core kernel when the selection (or the automatic choice) names
// it, else on the row-block kernel.
static rq_status launch_decode_ex(const uint16_t* const* xs, int nx, int64_t M, int64_t K,
                                  int64_t N, int bits, const WOperand* w, int nmat, bool y_half,
                                  int epilogue, cudaStream_t s) {
    cudaError_t e;
    if (decode_kernel_for(M, K, N, bits, nmat) == RQ_DECODE_TENSOR)
        e = launch_tcs(xs, nx, M, K, N, bits, w, nmat, y_half, epilogue, s);
    else if (gemv_rowblock_fits(M, K, N, bits, nmat))
        e = launch_gemv_rowblock_ex(xs, nx, M, K, N, bits, w, nmat, y_half, epilogue, s);
    else
        return RQ_ERR_SHAPE;
    return e == cudaSuccess ? RQ_OK : cuda_fail(e);
}

extern "C" {

size_t rq_codes_bytes(int64_t N, int64_t K, int bits) {
    if (check_weight_shape(N, K, bits) != RQ_OK) return 0;
    return static_cast<size_t>(N) * static_cast<size_t>(K) * static_cast<size_t>(bits) / 8;
}

size_t rq_scales_bytes(int64_t N, int64_t K) {
    if (check_weight_shape(N, K, 4) != RQ_OK) return 0;
    return static_cast<size_t>(N) * static_cast<size_t>(K / kGroup) * 2;
}

rq_status rq_quantize_g64(const float* W, int64_t N, int64_t K, int bits, void* codes,
                          uint16_t* scales, int* dev_status, rq_stream_t stream) {
    rq_status st = check_weight_shape(N, K, bits);
    if (st != RQ_OK) return st;
    if (W == nullptr || codes == nullptr || scales == nullptr) return RQ_ERR_NULL;
    if (!aligned16(W) || !aligned16(codes) || !aligned16(scales)) return RQ_ERR_ALIGN;
    if (dev_status != nullptr && (reinterpret_cast<uintptr_t>(dev_status) & 3u)) return RQ_ERR_ALIGN;
    cudaError_t e = launch_quantize(W, N * (K / kGroup), bits, codes, scales, dev_status,
                                    reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? RQ_OK : cuda_fail(e);
}

rq_status rq_quantize_g64_ex2(const float* W, int64_t N, int64_t K, int bits, const float* e2,
                              const float* factors, int nf, void* codes, uint16_t* scales,
                              int32_t* chosen, int* dev_status, rq_stream_t stream) {
    rq_status st = check_weight_shape(N, K, bits);
    if (st != RQ_OK) return st;
    if (nf < 1 || nf > 16) return RQ_ERR_RANGE;
    if (W == nullptr || e2 == nullptr || factors == nullptr || codes == nullptr || scales == nullptr)
        return RQ_ERR_NULL;
    if (!aligned16(W) || !aligned16(e2) || !aligned16(codes) || !aligned16(scales)) return RQ_ERR_ALIGN;
    const auto mis4 = [](const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 3u); };
    if (mis4(factors) || mis4(chosen) || mis4(dev_status)) return RQ_ERR_ALIGN;
    cudaError_t e = launch_quantize_ex2(W, N, K, bits, e2, factors, nf, codes, scales, chosen,
                                        dev_status, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? RQ_OK : cuda_fail(e);
}

static rq_status check_search(const float* e2, const float* factors, int nf) {
    if (e2 == nullptr) return RQ_OK;
    if (nf < 1 || nf > 16) return RQ_ERR_RANGE;
    if (factors == nullptr) return RQ_ERR_NULL;
    if (!aligned16(e2) || (reinterpret_cast<uintptr_t>(factors) & 3u)) return RQ_ERR_ALIGN;
    return RQ_OK;
}

rq_status rq_quantize_p8_g16(const float* W, int64_t N, int64_t K, const float* e2,
                             const float* factors, int nf, void* codes, uint16_t* scales,
                             int32_t* chosen, int* dev_status, rq_stream_t stream) {
    rq_status st = check_weight_shape(N, K, 8);
    if (st != RQ_OK) return st;
    if ((st = check_search(e2, factors, nf)) != RQ_OK) return st;
    if (W == nullptr || codes == nullptr || scales == nullptr) return RQ_ERR_NULL;
    if (!aligned16(W) || !aligned16(codes) || !aligned16(scales)) return RQ_ERR_ALIGN;
    const auto mis4 = [](const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 3u); };
    if (mis4(chosen) || mis4(dev_status)) return RQ_ERR_ALIGN;
    const cudaError_t e = launch_quantize_p8(W, N, K, e2, factors, nf, codes, scales, chosen, dev_status,
                                             reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? RQ_OK : cuda_fail(e);
}

rq_status rq_quantize_p4a_g32(const float* W, int64_t N, int64_t K, const float* e2,
                              const float* factors, int nf, void* codes, uint8_t* sub, uint16_t* sup,
                              int32_t* chosen, int* dev_status, rq_stream_t stream) {
    rq_status st = check_weight_shape(N, K, 4);
    if (st != RQ_OK) return st;
    if (K % 256 != 0) return RQ_ERR_SHAPE;
    if ((st = check_search(e2, factors, nf)) != RQ_OK) return st;
    if (W == nullptr || codes == nullptr || sub == nullptr || sup == nullptr) return RQ_ERR_NULL;
    if (!aligned16(W) || !aligned16(codes) || !aligned16(sub) || !aligned16(sup)) return RQ_ERR_ALIGN;
    const auto mis4 = [](const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 3u); };
    if (mis4(chosen) || mis4(dev_status)) return RQ_ERR_ALIGN;
    const cudaError_t e = launch_quantize_p4a(W, N, K, e2, factors, nf, codes, sub, sup, chosen, dev_status,
                                              reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? RQ_OK : cuda_fail(e);
}

rq_status rq_gptq_hessian(const uint16_t* X, int64_t T, int64_t K, double* H, rq_stream_t stream) {
    if (K < kGroup || K % kGroup != 0 || K > (int64_t{1} << 16) || T < 1 || T > (int64_t{1} << 31))
        return RQ_ERR_SHAPE;
    if (X == nullptr || H == nullptr) return RQ_ERR_NULL;
    if (!aligned16(X) || !aligned16(H)) return RQ_ERR_ALIGN;
    const cudaError_t e = launch_gptq_hessian(X, T, K, H, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? RQ_OK : cuda_fail(e);
}

rq_status rq_gptq_factor(double* H, int64_t K, double damp, float* U, uint8_t* dead, double* work,
                         rq_stream_t stream) {
    if (K < kGroup || K % kGroup != 0 || K > (int64_t{1} << 16)) return RQ_ERR_SHAPE;
    if (!(damp >= 0.0) || !(damp < 1e6)) return RQ_ERR_RANGE;
    if (H == nullptr || U == nullptr || dead == nullptr || work == nullptr) return RQ_ERR_NULL;
    if (!aligned16(H) || !aligned16(U) || !aligned16(work)) return RQ_ERR_ALIGN;
    const cudaError_t e = launch_gptq_factor(H, K, damp, U, dead, work,
                                             reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? RQ_OK : cuda_fail(e);
}

rq_status rq_gptq_g64(float* W, int64_t N, int64_t K, int bits, const float* U, const uint8_t* dead,
                      void* codes, uint16_t* scales, float* work, int* dev_status, rq_stream_t stream) {
    rq_status st = check_weight_shape(N, K, bits);
    if (st != RQ_OK) return st;
    if (K > (int64_t{1} << 16)) return RQ_ERR_SHAPE;
    if (W == nullptr || U == nullptr || codes == nullptr || scales == nullptr || work == nullptr)
        return RQ_ERR_NULL;
    if (!aligned16(W) || !aligned16(U) || !aligned16(codes) || !aligned16(scales) || !aligned16(work))
        return RQ_ERR_ALIGN;
    if (dev_status != nullptr && (reinterpret_cast<uintptr_t>(dev_status) & 3u)) return RQ_ERR_ALIGN;
    const cudaError_t e = launch_gptq_quantize(W, N, K, bits, U, dead, codes, scales, work, dev_status,
                                               reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? RQ_OK : cuda_fail(e);
}

rq_status rq_gemv_wq(const uint16_t* x, int64_t M, int64_t K, const void* codes,
                     const uint16_t* scales, int64_t N, int bits, float* y, rq_stream_t stream) {
    rq_status st = check_product(x, M, K, N, bits, RQ_MAX_DECODE_M);
    if (st != RQ_OK) return st;
    if ((st = check_operand(codes, scales, y)) != RQ_OK) return st;
    WOperand w = {codes, scales, y};
    return launch_decode(x, M, K, N, bits, &w, 1, reinterpret_cast<cudaStream_t>(stream));
}

rq_status rq_rkv_fused(const uint16_t* x, int64_t M, int64_t K, int64_t N, int bits,
                       const void* codes_r, const uint16_t* scales_r, const void* codes_k,
                       const uint16_t* scales_k, const void* codes_v, const uint16_t* scales_v,
                       float* y_r, float* y_k, float* y_v, rq_stream_t stream) {
    rq_status st = check_product(x, M, K, N, bits, RQ_MAX_DECODE_M);
    if (st != RQ_OK) return st;
    if ((st = check_operand(codes_r, scales_r, y_r)) != RQ_OK) return st;
    if ((st = check_operand(codes_k, scales_k, y_k)) != RQ_OK) return st;
    if ((st = check_operand(codes_v, scales_v, y_v)) != RQ_OK) return st;
    WOperand w[3] = {{codes_r, scales_r, y_r}, {codes_k, scales_k, y_k}, {codes_v, scales_v, y_v}};
    return launch_decode(x, M, K, N, bits, w, 3, reinterpret_cast<cudaStream_t>(stream));
}

rq_status rq_gemv_wq_ex(const uint16_t* x, int64_t M, int64_t K, const void* codes,
                        const uint16_t* scales, int64_t N, int bits, void* y, int out_dtype,
                        int epilogue, rq_stream_t stream) {
    rq_status st = check_product(x, M, K, N, bits, RQ_MAX_DECODE_M);
    if (st != RQ_OK) return st;
    if (out_dtype != RQ_OUT_F32 && out_dtype != RQ_OUT_F16) return RQ_ERR_RANGE;
    if (epilogue != RQ_EPI_NONE && epilogue != RQ_EPI_RELU_SQ) return RQ_ERR_RANGE;
    if ((st = check_operand(codes, scales, static_cast<const float*>(y))) != RQ_OK) return st;
    WOperand w = {codes, scales, static_cast<float*>(y)};
    const uint16_t* xs[1] = {x};
    return launch_decode_ex(xs, 1, M, K, N, bits, &w, 1, out_dtype == RQ_OUT_F16, epilogue,
                            reinterpret_cast<cudaStream_t>(stream));
}

rq_status rq_rkv_fused3(const uint16_t* x_r, const uint16_t* x_k, const uint16_t* x_v, int64_t M,
                        int64_t K, int64_t N, int bits, const void* codes_r, const uint16_t* scales_r,
                        const void* codes_k, const uint16_t* scales_k, const void* codes_v,
                        const uint16_t* scales_v, void* y_r, void* y_k, void* y_v, int out_dtype,
                        rq_stream_t stream) {
    rq_status st = check_product(x_r, M, K, N, bits, RQ_MAX_DECODE_M);
    if (st != RQ_OK) return st;
    if (x_k == nullptr || x_v == nullptr) return RQ_ERR_NULL;
    if (!aligned16(x_k) || !aligned16(x_v)) return RQ_ERR_ALIGN;
    if (out_dtype != RQ_OUT_F32 && out_dtype != RQ_OUT_F16) return RQ_ERR_RANGE;
    if ((st = check_operand(codes_r, scales_r, static_cast<const float*>(y_r))) != RQ_OK) return st;
    if ((st = check_operand(codes_k, scales_k, static_cast<const float*>(y_k))) != RQ_OK) return st;
    if ((st = check_operand(codes_v, scales_v, static_cast<const float*>(y_v))) != RQ_OK) return st;
    WOperand w[3] = {{codes_r, scales_r, static_cast<float*>(y_r)},
                     {codes_k, scales_k, static_cast<float*>(y_k)},
                     {codes_v, scales_v, static_cast<float*>(y_v)}};
    const uint16_t* xs[3] = {x_r, x_k, x_v};
    return launch_decode_ex(xs, 3, M, K, N, bits, w, 3, out_dtype == RQ_OUT_F16, RQ_EPI_NONE,
                            reinterpret_cast<cudaStream_t>(stream));
}

rq_status rq_gemv_p8_g16(const uint16_t* x, int64_t M, int64_t K, const void* codes,
                         const uint16_t* scales, int64_t N, float* y, rq_stream_t stream) {
    rq_status st = check_product(x, M, K, N, 8, RQ_MAX_DECODE_M);
    if (st != RQ_OK) return st;
    if (K % 128 != 0) return RQ_ERR_SHAPE;
    if ((st = check_operand(codes, scales, y)) != RQ_OK) return st;
    if (!gemv_rowblock_fits(M, K, N, 8, 1, FMT_P8)) return RQ_ERR_SHAPE;
    WOperand w = {codes, scales, y};
    const uint16_t* xs[1] = {x};
    const cudaError_t e = launch_gemv_rowblock_fmt(xs, 1, M, K, N, 8, FMT_P8, &w, nullptr, 1, false,
                                                   RQ_EPI_NONE, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? RQ_OK : cuda_fail(e);
}

rq_status rq_gemv_p4a_g32(const uint16_t* x, int64_t M, int64_t K, const void* codes,
                          const uint8_t* sub, const uint16_t* sup, int64_t N, float* y,
                          rq_stream_t stream) {
    rq_status st = check_product(x, M, K, N, 4, RQ_MAX_DECODE_M);
    if (st != RQ_OK) return st;
    if (K % 256 != 0) return RQ_ERR_SHAPE;
    if ((st = check_operand(codes, reinterpret_cast<const uint16_t*>(sub), y)) != RQ_OK) return st;
    if (sup == nullptr) return RQ_ERR_NULL;
    if (!aligned16(sup)) return RQ_ERR_ALIGN;
    if (!gemv_rowblock_fits(M, K, N, 4, 1, FMT_P4A)) return RQ_ERR_SHAPE;
    WOperand w = {codes, reinterpret_cast<const uint16_t*>(sub), y};
    const uint16_t* xs[1] = {x};
    const uint32_t* sp[1] = {reinterpret_cast<const uint32_t*>(sup)};
    const cudaError_t e = launch_gemv_rowblock_fmt(xs, 1, M, K, N, 4, FMT_P4A, &w, sp, 1, false,
                                                   RQ_EPI_NONE, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? RQ_OK : cuda_fail(e);
}

rq_status rq_gemm_wq(const uint16_t* x, int64_t M, int64_t K, const void* codes,
                     const uint16_t* scales, int64_t N, int bits, float* y, rq_stream_t stream) {
    rq_status st = check_product(x, M, K, N, bits, (int64_t{1} << 31) - 1);
    if (st != RQ_OK) return st;
    if ((st = check_operand(codes, scales, y)) != RQ_OK) return st;
    if (M * K > (int64_t{1} << 40)) return RQ_ERR_SHAPE;
    WOperand w = {codes, scales, y};
    cudaError_t e = launch_tc_product(x, M, K, N, bits, &w, 1, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? RQ_OK : cuda_fail(e);
}

rq_status rq_set_pdl(int enable) {
    g_pdl = enable != 0;
    return RQ_OK;
}

rq_status rq_set_decode_kernel(int kernel) {
    if (kernel != RQ_DECODE_AUTO && kernel != RQ_DECODE_ROWTILE && kernel != RQ_DECODE_CLUSTER &&
        kernel != RQ_DECODE_ROWBLOCK && kernel != RQ_DECODE_TENSOR)
        return RQ_ERR_RANGE;
    g_decode_kernel = kernel;
    return RQ_OK;
}

rq_status rq_decode_kernel_for(int64_t M, int64_t K, int64_t N, int bits, int nmat, int* kernel) {
    rq_status st = check_weight_shape(N, K, bits);
    if (st != RQ_OK) return st;
    if (M < 1 || M > RQ_MAX_DECODE_M || (nmat != 1 && nmat != 3)) return RQ_ERR_SHAPE;
    if (kernel == nullptr) return RQ_ERR_NULL;
    const int which = decode_kernel_for(M, K, N, bits, nmat);
    if (which < 0) return RQ_ERR_SHAPE;
    *kernel = which;
    return RQ_OK;
}

rq_status rq_set_wait_limit_ns(uint64_t limit_ns) {
    if (limit_ns == 0) return RQ_ERR_RANGE;
    g_wait_limit_ns = limit_ns;
    return RQ_OK;
}

rq_status rq_read_device_status(int* out, int reset) {
    if (out == nullptr) return RQ_ERR_NULL;
    cudaError_t e = cudaMemcpyFromSymbol(out, g_device_status, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e);
    if (reset) {
        const int zero = 0;
        e = cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int));
        if (e != cudaSuccess) return cuda_fail(e);
        e = workspace_reset_counters();
        if (e != cudaSuccess) return cuda_fail(e);
    }
    return RQ_OK;
}

rq_status rq_selftest_bounded_wait(uint64_t limit_ns, rq_stream_t stream) {
    if (limit_ns == 0) return RQ_ERR_RANGE;
    cudaError_t e = launch_wait_selftest(limit_ns, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? RQ_OK : cuda_fail(e);
}

const char* rq_status_string(rq_status s) {
    switch (s) {
        case RQ_OK: return "ok";
        case RQ_ERR_NULL: return "a required pointer is NULL";
        case RQ_ERR_BITS: return "bits must be 4 or 8";
        case RQ_ERR_SHAPE: return "bad shape (K % 64 != 0, N < 1, M out of range, or too large)";
        case RQ_ERR_ALIGN: return "a pointer is not 16-byte aligned";
        case RQ_ERR_NONFINITE: return "a weight is NaN or infinite";
        case RQ_ERR_RANGE: return "a value is out of range (fp16 scale overflow or bad limit)";
        case RQ_ERR_TIMEOUT: return "a bounded on-chip wait timed out";
        case RQ_ERR_CUDA: return "a CUDA call failed";
    }
    return "unknown status";
}

const char* rq_last_cuda_error(void) { return t_last_cuda_error.c_str(); }

const char* rq_version(void) { return "0.1.0"; }

}  // extern "C"
