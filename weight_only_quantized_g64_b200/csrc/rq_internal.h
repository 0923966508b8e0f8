// rq_internal.h -- declarations shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "../../include/rq.h"

namespace rq {

// Group size of the format (64 consecutive k of one row share a scale).
constexpr int kGroup = 64;

// Quantizer: flat over all N*K/64 groups (groups are contiguous in W, codes
// and scales when all three are row-major).
cudaError_t launch_quantize(const float* W, int64_t n_groups, int bits, void* codes,
                            uint16_t* scales, int* dev_status, cudaStream_t s);

// Quantizer with an E[x^2]-weighted scale search (nf <= 16 candidates).
cudaError_t launch_quantize_ex2(const float* W, int64_t N, int64_t K, int bits, const float* e2,
                                const float* factors, int nf, void* codes, uint16_t* scales,
                                int32_t* chosen, int* dev_status, cudaStream_t s);

// One weight operand of a product: its TMA descriptor (codes), scales, output.
struct WOperand {
    const void* codes;
    const uint16_t* scales;
    float* y;
};

// Tensor-core product (dequantise into TMEM, tcgen05.mma with fp32
// accumulation).  nmat = 1 (single projection) or 3 (fused R/K/V).
cudaError_t launch_tc_product(const uint16_t* x, int64_t M, int64_t K, int64_t N, int bits,
                              const WOperand* w, int nmat, cudaStream_t s);

// Decode product (M <= 32): TMA-staged codes, in-register dequantisation,
// warp-level tensor-core MMA (mma.sync), stream-K split over the SMs.
cudaError_t launch_gemv_product(const uint16_t* x, int64_t M, int64_t K, int64_t N, int bits,
                                const WOperand* w, int nmat, cudaStream_t s);

// Decode product (M <= 32), K split over the CTAs of a cluster, partial sums
// added through distributed shared memory.  Needs no workspace.
cudaError_t launch_gemv_cluster(const uint16_t* x, int64_t M, int64_t K, int64_t N, int bits,
                                const WOperand* w, int nmat, cudaStream_t s);

// Whether the cluster kernel's shared memory holds a product with this M and
// K (each CTA keeps the x of its K range on chip).
bool gemv_cluster_fits(int64_t M, int64_t K, int bits);

// Decode product (M <= 32), row blocks over the full K range: every output is
// finished inside one CTA.  Needs no workspace.
cudaError_t launch_gemv_rowblock(const uint16_t* x, int64_t M, int64_t K, int64_t N, int bits,
                                 const WOperand* w, int nmat, cudaStream_t s);

// The row-block kernel with nx inputs (1 shared, or one per matrix), y as
// fp16 when y_half (WOperand::y then points to fp16), and an epilogue
// (0 none, 1 relu(y)^2) applied before the store.
cudaError_t launch_gemv_rowblock_ex(const uint16_t* const* xs, int nx, int64_t M, int64_t K,
                                    int64_t N, int bits, const WOperand* w, int nmat, bool y_half,
                                    int epilogue, cudaStream_t s);

// Weight formats of the row-block kernel: the symmetric group-64 format, and
// the two rwkv-quant presets (int8 symmetric in groups of 16: codes int8
// [N, K], scales fp16 [N, K/16], K % 128 == 0; int4 asymmetric in groups of
// 32 under super-blocks of 256: codes u8 [N, K/2], sub-codes u8 [N, K/32, 2]
// in place of the scales, (ds, dm) fp16 [N, K/256, 2], K % 256 == 0).
constexpr int FMT_G64 = 0, FMT_P8 = 1, FMT_P4A = 2;

// The row-block kernel for weights of format fmt (bits 8 for FMT_P8, 4 for
// FMT_P4A); sup[i]: the (ds, dm) pairs of matrix i for FMT_P4A, else unused.
cudaError_t launch_gemv_rowblock_fmt(const uint16_t* const* xs, int nx, int64_t M, int64_t K,
                                     int64_t N, int bits, int fmt, const WOperand* w,
                                     const uint32_t* const* sup, int nmat, bool y_half,
                                     int epilogue, cudaStream_t s);

// Streaming tensor-core product for 1 <= M <= 64 (tcgen05, dequantised
// weights in TMEM, 256-row blocks with K split over a thread-block cluster,
// partial sums added through distributed shared memory; needs no workspace).
// Inputs and outputs as launch_gemv_rowblock_ex.
cudaError_t launch_tcs(const uint16_t* const* xs, int nx, int64_t M, int64_t K, int64_t N,
                       int bits, const WOperand* w, int nmat, bool y_half, int epilogue,
                       cudaStream_t s);
bool tcs_fits(int64_t M, int64_t K, int64_t N, int bits);
// Its K split (cluster size) for a shape.
int tcs_ksplit(int64_t K, int64_t N, int nmat, int bits);

// Whether the row-block kernel takes a product of this shape and format.
bool gemv_rowblock_fits(int64_t M, int64_t K, int64_t N, int bits, int nmat, int fmt = FMT_G64);

// The decode kernel a product of this shape runs on: RQ_DECODE_ROWTILE,
// RQ_DECODE_CLUSTER, RQ_DECODE_ROWBLOCK or RQ_DECODE_TENSOR (the selection of
// rq_set_decode_kernel, or the automatic choice), or -1 when the selected
// kernel cannot take the shape.
int decode_kernel_for(int64_t M, int64_t K, int64_t N, int bits, int nmat);

// Caller-provided scratch for the decode product instead of the library's
// workspace: partial-tile slots (ws, ws_bytes) and per-tile counters (cnt,
// n_cnt, zero between launches).  If a launch would need more, nothing is
// launched and *too_large is set.
struct GemvScratch {
    float* ws;
    size_t ws_bytes;
    int* cnt;
    size_t n_cnt;
    bool* too_large;
};
cudaError_t launch_gemv_product_scratch(const uint16_t* x, int64_t M, int64_t K, int64_t N,
                                        int bits, const WOperand* w, int nmat, cudaStream_t s,
                                        const GemvScratch* scratch);

// GPTQ on the group-64 grid: H = (2/T) X^T X (fp64); the damped inverse-
// Hessian factor U (fp32 upper, H^-1 = U^T U) and the dead-input mask (work:
// K*K + K doubles, H consumed); the column loop (W in/out, work: N*128 fp32).
cudaError_t launch_gptq_hessian(const uint16_t* X, int64_t T, int64_t K, double* H, cudaStream_t s);
cudaError_t launch_gptq_factor(double* H, int64_t K, double damp, float* U, uint8_t* dead,
                               double* work, cudaStream_t s);
cudaError_t launch_gptq_quantize(float* W, int64_t N, int64_t K, int bits, const float* U,
                                 const uint8_t* dead, void* codes, uint16_t* scales, float* work,
                                 int* dev_status, cudaStream_t s);

// Quantizers of the rwkv-quant preset formats: symmetric int8 with groups of
// 16 (scales fp16 [N, K/16]); asymmetric int4 with groups of 32 in
// super-blocks of 8 (sub uint8 [N, K/32, 2], sup fp16 [N, K/256, 2]).
// e2 NULL: no search (RTN).
cudaError_t launch_quantize_p8(const float* W, int64_t N, int64_t K, const float* e2,
                               const float* factors, int nf, void* codes, uint16_t* scales,
                               int32_t* chosen, int* dev_status, cudaStream_t s);
cudaError_t launch_quantize_p4a(const float* W, int64_t N, int64_t K, const float* e2,
                                const float* factors, int nf, void* codes, uint8_t* sub, uint16_t* sup,
                                int32_t* chosen, int* dev_status, cudaStream_t s);

// Bounded-wait self test: a kernel waits on an mbarrier nothing completes.
cudaError_t launch_wait_selftest(uint64_t limit_ns, cudaStream_t s);

// Tensor map creation (driver entry point fetched once through the runtime).
bool make_tmap_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base,
                  uint64_t inner_elems, uint64_t rows, uint64_t row_stride_bytes,
                  uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle swz);

// 3D tiled tensor map: dims {d0 (contiguous), d1, d2}, byte strides s1, s2
// (any order), box {b0, b1, b2}.
bool make_tmap_3d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t d0,
                  uint64_t d1, uint64_t d2, uint64_t s1, uint64_t s2, uint32_t b0, uint32_t b1,
                  uint32_t b2, CUtensorMapSwizzle swz);

// Whether programmatic dependent launch is requested for kernel launches.
bool pdl_enabled();

// Device address of the library status word on the current device.
// SMs of the current device (148 when it cannot be queried), cached per device.
int num_sms();

int* device_status_ptr();

// Time limit of every bounded on-chip wait, in nanoseconds.
uint64_t wait_limit_ns();

// Per-device scratch of the decode product: partial-tile slots and per-tile
// arrival counters (zero between launches).  Grows on demand; growing
// allocates device memory, so the first call at a new size must not be made
// while a stream is being captured.
cudaError_t workspace_get(size_t ws_bytes, size_t n_counters, float** ws, int** cnt);

// Zero the current device's arrival counters (after an aborted launch).
cudaError_t workspace_reset_counters();

// Remember e as this thread's last CUDA error (returned by rq_last_cuda_error).
void record_cuda_error(cudaError_t e);

}  // namespace rq
