// rq_noalloc.cu -- rq_gemv_wq_noalloc: the decode product with its scratch in
// a fixed, statically sized device array instead of memory the library
// allocates.
//
// The decode product splits its work evenly over the SMs; a row tile shared
// by several CTAs leaves partial sums in scratch, and a per-tile counter says
// which CTA adds them up.  rq_gemv_wq keeps that scratch in a workspace it
// allocates on first use.  Some callers cannot let a library allocate:
// a caller recording a CUDA graph (allocation is not a stream operation and is
// refused or goes unrecorded while a stream is being captured), a serving
// runtime that reserves the device's memory up front for weights and caches
// and accounts for every byte, or a latency-critical loop that must not hit
// the implicit synchronisation of cudaMalloc / cudaFree.  This entry point
// calls no allocator at all.
//
// Scratch: one file-scope array per device that loads the library, held until
// the process exits: kSlotBytes of partial-tile slots followed by
// kMaxTiles per-tile counters.  Host code never dereferences the array's name
// (on the host it is only a stand-in for the device symbol); the device
// address is obtained once per device with cudaGetSymbolAddress.
#include <cstring>
#include <mutex>

#include "rq_internal.h"

namespace rq {

constexpr size_t kSlotBytes = size_t{5} << 20;          // partial-tile slots: 5 MiB
constexpr size_t kMaxTiles = 16384;                       // per-tile counters
constexpr size_t kScratchBytes = kSlotBytes + kMaxTiles * sizeof(int);

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

static constexpr int kMaxDev = 64;
static unsigned char* g_scratch_addr[kMaxDev] = {};
static std::mutex g_scratch_mu;

// Device address of the scratch array on the current device (set-up on the
// first call per device).
static cudaError_t scratch_address(unsigned char** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (g_scratch_addr[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        if (p == nullptr) return cudaErrorInvalidSymbol;
        g_scratch_addr[dev] = static_cast<unsigned char*>(p);
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

}  // namespace rq

using namespace rq;

extern "C" rq_status rq_gemv_wq_noalloc(const uint16_t* x, int64_t M, int64_t K,
                                        const void* codes, const uint16_t* scales, int64_t N,
                                        int bits, float* y, rq_stream_t stream) {
    // same argument rules as rq_gemv_wq
    if (bits != 4 && bits != 8) return RQ_ERR_BITS;
    if (N < 1 || K < kGroup || K % kGroup != 0) return RQ_ERR_SHAPE;
    if (N > (int64_t{1} << 31) - 1 || K > (int64_t{1} << 30)) return RQ_ERR_SHAPE;
    if (M < 1 || M > RQ_MAX_DECODE_M) return RQ_ERR_SHAPE;
    if (x == nullptr || codes == nullptr || scales == nullptr || y == nullptr) return RQ_ERR_NULL;
    const auto mis = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; };
    if (mis(x) || mis(codes) || mis(scales) || mis(y)) return RQ_ERR_ALIGN;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    WOperand w = {codes, scales, y};
    const int which = decode_kernel_for(M, K, N, bits, 1);
    if (which < 0) return RQ_ERR_SHAPE;
    if (which == RQ_DECODE_CLUSTER || which == RQ_DECODE_ROWBLOCK || which == RQ_DECODE_TENSOR) {
        // these kernels keep their partial sums on chip: no scratch at all
        const uint16_t* xs[1] = {x};
        cudaError_t ec = which == RQ_DECODE_CLUSTER  ? launch_gemv_cluster(x, M, K, N, bits, &w, 1, s)
                         : which == RQ_DECODE_TENSOR ? launch_tcs(xs, 1, M, K, N, bits, &w, 1, false, 0, s)
                                                     : launch_gemv_rowblock(x, M, K, N, bits, &w, 1, s);
        if (ec != cudaSuccess) {
            record_cuda_error(ec);
            return RQ_ERR_CUDA;
        }
        return RQ_OK;
    }

    unsigned char* base = nullptr;
    cudaError_t e = scratch_address(&base);
    if (e != cudaSuccess) {
        record_cuda_error(e);
        return RQ_ERR_CUDA;
    }
    float* ws = reinterpret_cast<float*>(base);
    int* cnt = reinterpret_cast<int*>(base + kSlotBytes);
    // the launcher checks the scratch it needs against these sizes before it
    // enqueues anything (then clears the counters it uses)
    bool too_large = false;
    GemvScratch sc = {ws, kSlotBytes, cnt, kMaxTiles, &too_large};
    e = launch_gemv_product_scratch(x, M, K, N, bits, &w, 1, s, &sc);
    if (too_large) return RQ_ERR_SHAPE;
    if (e != cudaSuccess) {
        record_cuda_error(e);
        return RQ_ERR_CUDA;
    }
    return RQ_OK;
}
