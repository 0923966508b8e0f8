/*
 * rq.h -- C ABI of librq: weight-only, group-64, symmetric int4/int8
 * quantized projections on NVIDIA B200 (sm_100a).
 *
 * The operation: a projection weight W[N, K] (N output features, K input
 * features, row-major) is stored group-wise with GROUP = 64 consecutive k of
 * one row sharing one fp16 scale, symmetric (no zero point), as packed signed
 * codes plus scales -- the ".qweight + .scale" format of the
 * "Hakureirm/rwkv7-sglang-w4gptq-1.5b" model card ("Format & loading
 * (important)"), in its int4 form and the int8 "w8g64" tier of its
 * "Accuracy warning" section.  Products are taken directly on those codes
 * ("RWKV-7 Quantization Toolkit", rwkv-quant-nv 1.2.1, "Key Design": no
 * dequantised weight matrix is materialised), in three kernel families named
 * by the model card's opening summary: a GEMV for decode, a small-M product
 * and a tensor-core GEMM for prefill.  The fused R/K/V call follows the same
 * "Key Design" list (three projections in one kernel launch).
 *
 * Layouts (all row-major, all device memory owned by the caller):
 *   W       fp32 [N, K]
 *   codes   int4: uint8 [N, K/2]; byte j of row n holds k = 2j in its low
 *           nibble and k = 2j+1 in its high nibble, 4-bit two's complement,
 *           values in [-7, 7].  int8: int8 [N, K], values in [-127, 127].
 *   scales  fp16 bit patterns [N, K/64]; scales[n, g] covers k in [64g, 64g+64).
 *   x       fp16 [M, K]            y  fp32 [M, N]
 *   Dequantised weight: w_hat[n, k] = code[n, k] * scales[n, k/64].
 *   y[m, n] = sum_k x[m, k] * w_hat[n, k], accumulated in fp32; the result is
 *   within 2e-3 * sum_k |x[m, k]| * |w_hat[n, k]| of the exact value.
 *
 * Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 * stream).  Argument errors are found before any launch and returned
 * synchronously; nothing is launched then.  The library allocates no device
 * memory per call, except the decode products' workspace, allocated the
 * first time a shape needs it (see rq_gemv_wq); pointers must stay valid
 * until the stream reaches the call.  Inputs and outputs must not overlap.
 * Array pointers must be 16-byte aligned unless a call states otherwise.  A
 * call that fails to launch returns RQ_ERR_CUDA (the CUDA error string is
 * available from rq_last_cuda_error()).
 */
#ifndef RQ_H_
#define RQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t, declared without the CUDA headers. */
typedef struct CUstream_st *rq_stream_t;

typedef enum {
    RQ_OK = 0,
    RQ_ERR_NULL = 1,       /* a required pointer is NULL */
    RQ_ERR_BITS = 2,       /* bits is not 4 or 8 */
    RQ_ERR_SHAPE = 3,      /* K % 64 != 0, N < 1, K < 64, M out of range, or sizes too large */
    RQ_ERR_ALIGN = 4,      /* a pointer is not 16-byte aligned */
    RQ_ERR_NONFINITE = 5,  /* (device status) a weight is NaN or +-inf */
    RQ_ERR_RANGE = 6,      /* (device status) a group scale overflows fp16 */
    RQ_ERR_TIMEOUT = 7,    /* (device status) a bounded on-chip wait gave up */
    RQ_ERR_CUDA = 8        /* a CUDA call or kernel launch failed */
} rq_status;

#define RQ_GROUP 64
#define RQ_MAX_DECODE_M 32

/* Bytes of packed codes for an N x K matrix: N*K*bits/8. 0 on bad arguments. */
size_t rq_codes_bytes(int64_t N, int64_t K, int bits);

/* Bytes of fp16 scales for an N x K matrix: N*(K/64)*2. 0 on bad arguments. */
size_t rq_scales_bytes(int64_t N, int64_t K);

/*
 * rq_quantize_g64 -- round-to-nearest group-64 symmetric quantization (the
 * "calibration-free RTN" of the model card's accuracy bullet).
 *
 * For every row n and group g, with qmax = 7 (bits 4) or 127 (bits 8):
 *   amax = max |W[n, k]| over the group          (fp32, exact)
 *   s32  = amax / qmax                           (IEEE fp32 division)
 *   s16  = fp16(s32), round to nearest even     -> scales[n, g]
 *   code = clamp(rint(W[n, k] / float(s16)), -qmax, qmax)
 *          (IEEE fp32 division by the STORED scale, rint = half to even);
 *          code = 0 for every k when s16 == 0.
 * W: fp32 [N, K] device.  codes: rq_codes_bytes(N, K, bits) bytes device.
 * scales: N*(K/64) fp16 device.  dev_status: optional device int that the
 * caller zeroes beforehand; the kernel sets it to RQ_ERR_NONFINITE if any
 * weight is NaN/inf (that group gets scale 0x7E00, codes 0), otherwise to
 * RQ_ERR_RANGE if any group scale overflows fp16 (that group gets scale +inf,
 * codes 0); it stays RQ_OK otherwise.  Bandwidth-bound: reads 4 B and writes 0.53 / 1.03 B per weight.
 * Requires K % 64 == 0, N >= 1.
 */
rq_status rq_quantize_g64(const float *W, int64_t N, int64_t K, int bits,
                          void *codes, uint16_t *scales, int *dev_status,
                          rq_stream_t stream);

/*
 * rq_quantize_g64_ex2 -- group-64 symmetric quantization with the scale of
 * each group chosen by an E[x^2]-weighted search ("rwkv-quant: uma matriz em
 * bf16 elimina 39% das perdas na quantização do RWKV-7 2.9B", "Dois presets e
 * seis tamanhos": the groups' scale is chosen by a search weighted by the mean
 * square of the input channel's activation).  Same stored format as
 * rq_quantize_g64.  Per group, candidate j (0 <= j < nf) has scale
 * s16_j = fp16_rn(fp32(amax * factors[j]) / qmax) and RTN codes against it;
 * its error is sum_k e2[k] * (w_k - c_k * s16_j)^2 over the group's 64 k in k
 * order, every operation one IEEE fp32 rounding; the smallest error wins, the
 * earlier candidate on a tie; a candidate whose scale overflows fp16 is never
 * chosen (if all do, the group is quantized by RTN).  factors[0] = 1 makes
 * the result never worse than RTN by this measure; nf = 1 with factor 1 is
 * exactly rq_quantize_g64.
 *
 * W: fp32 [N, K] device, 16-byte aligned.  e2: fp32 [K] device, 16-byte
 * aligned, E[x^2] per input channel (finite, >= 0; the caller's estimate).
 * factors: fp32 [nf] device, 4-byte aligned, 1 <= nf <= 16 (else
 * RQ_ERR_RANGE).  codes, scales: outputs as for rq_quantize_g64.  chosen:
 * nullable int32 [N, K/64] device, 4-byte aligned, receives each group's
 * winning candidate (0 for groups RTN handled).  dev_status: as for
 * rq_quantize_g64.  Other argument errors as
 * rq_quantize_g64.  Asynchronous on `stream`.
 */
rq_status rq_quantize_g64_ex2(const float *W, int64_t N, int64_t K, int bits, const float *e2,
                              const float *factors, int nf, void *codes, uint16_t *scales,
                              int32_t *chosen, int *dev_status, rq_stream_t stream);

/*
 * The two preset formats of "rwkv-quant: uma matriz em bf16 elimina 39% das
 * perdas na quantização do RWKV-7 2.9B" ("Dois presets e seis tamanhos"):
 * REDUCTION stores projections in 8 bits, symmetric, groups of 16 weights;
 * COMPRESSION in 4 bits, asymmetric, in super-blocks, groups of 32; in both
 * the groups' scale (and offset) is chosen by a search weighted by E[x^2].
 * Where the article is silent, this library reads (and its oracle follows):
 *
 * rq_quantize_p8_g16 -- int8 symmetric, groups of 16 consecutive k: per group
 *   amax; candidate j: s16 = fp16_rn(fp32(amax * factors[j]) / 127), codes
 *   clamp(rint(w / s16), +-127) (IEEE fp32 division, ties to even), error
 *   sum_k e2[k] (w - c s16)^2 in k order (each operation one fp32 rounding);
 *   the smallest error wins, the earlier candidate on a tie; a candidate whose
 *   scale overflows is never chosen (all overflow: RTN).  e2 NULL: RTN (one
 *   candidate, factor 1).  codes int8 [N, K]; scales fp16 [N, K/16]; chosen
 *   (nullable) int32 [N, K/16].
 *
 * rq_quantize_p4a_g32 -- int4 asymmetric, groups of 32 in super-blocks of 8
 *   groups (256 k).  Per group: lo = min(0, min w), hi = max(0, max w);
 *   candidate j: lo_j = lo f_j, hi_j = hi f_j, s_j = (hi_j - lo_j) / 15, codes
 *   clamp(rint((w - lo_j) / s_j), 0, 15), error sum e2 (w - (q s_j + lo_j))^2;
 *   the chosen group's (s, o = lo_j).  Per super-block: ds =
 *   fp16_rn(max s / 63), dm = fp16_rn(max(-o) / 63); per group 6-bit
 *   sub-codes a = clamp(rint(s / ds), 0, 63), b = clamp(rint(-o / dm), 0, 63);
 *   stored scale S = ds a and offset O = -(dm b); codes q = clamp(rint((w - O) /
 *   S), 0, 15); w_hat = S q + O.  Layout: codes uint8 [N, K/2], unsigned
 *   nibbles, k = 2j in the low nibble of byte j; sub uint8 [N, K/32, 2] = (a,
 *   b); sup fp16 [N, K/256, 2] = (ds, dm); chosen (nullable) int32 [N, K/32].
 *   K % 256 == 0.  A super-block holding a non-finite weight: ds = dm =
 *   0x7E00, sub-codes and codes 0; an overflowing ds or dm: kept (+inf),
 *   sub-codes and codes 0.
 *
 * Both: W fp32 [N, K] device, 16-byte aligned; e2 fp32 [K] (E[x^2] per input
 * channel, >= 0) or NULL; factors fp32 [nf], 1 <= nf <= 16 (else
 * RQ_ERR_RANGE), read only with e2; dev_status as rq_quantize_g64
 * (RQ_ERR_NONFINITE over RQ_ERR_RANGE).  Every operation is one IEEE fp32
 * rounding in the order stated, so results are reproducible bit for bit.
 */
rq_status rq_quantize_p8_g16(const float *W, int64_t N, int64_t K, const float *e2,
                             const float *factors, int nf, void *codes, uint16_t *scales,
                             int32_t *chosen, int *dev_status, rq_stream_t stream);
rq_status rq_quantize_p4a_g32(const float *W, int64_t N, int64_t K, const float *e2,
                              const float *factors, int nf, void *codes, uint8_t *sub,
                              uint16_t *sup, int32_t *chosen, int *dev_status,
                              rq_stream_t stream);

/*
 * Decode products of the two preset formats (the formats above, as their
 * quantizers write them): y[M, N] = x[M, K] W_hat^T with
 *
 * rq_gemv_p8_g16  -- W_hat[n, k] = codes[n, k] * scales[n, k / 16];
 * rq_gemv_p4a_g32 -- W_hat[n, k] = S q + O, q the unsigned nibble of k,
 *   S = ds a and O = -(dm b) with (a, b) = sub[n, k / 32] and (ds, dm) =
 *   sup[n, k / 256], each product one fp32 rounding.
 *
 * Each group's sum x * codes is exact in fp32 before its scale (and, for the
 * asymmetric format, its offset times the group's sum of x) is applied in
 * fp32; groups are added in an order fixed per shape, so results are
 * deterministic.  x fp16 [M, K] row-major, 1 <= M <= 32 (else RQ_ERR_SHAPE);
 * y fp32 [M, N].  K % 128 == 0 (int8 preset) or K % 256 == 0 (int4 preset),
 * else RQ_ERR_SHAPE; x, codes, scales / sub, sup and y 16-byte aligned (else
 * RQ_ERR_ALIGN); NULL pointers: RQ_ERR_NULL.  Non-finite scales or x give
 * non-finite outputs.  Same kernel, data path and wait bound as the row-block
 * decode kernel of rq_gemv_wq; needs no workspace; asynchronous on `stream`.
 */
rq_status rq_gemv_p8_g16(const uint16_t *x, int64_t M, int64_t K, const void *codes,
                         const uint16_t *scales, int64_t N, float *y, rq_stream_t stream);
rq_status rq_gemv_p4a_g32(const uint16_t *x, int64_t M, int64_t K, const void *codes,
                          const uint8_t *sub, const uint16_t *sup, int64_t N, float *y,
                          rq_stream_t stream);

/*
 * GPTQ on the same group-64 grid -- the "GPTQ-calibrated, symmetric, group
 * 64" int4 of the "Hakureirm/rwkv7-sglang-w4gptq-1.5b" model card (opening
 * summary), run "on the preset's grid without changing the format or the
 * kernels" ("rwkv-quant: uma matriz em bf16 elimina 39% das perdas na
 * quantização do RWKV-7 2.9B", "Vazamento de calibração e medições
 * honestas").  The method is the published GPTQ (Frantar et al.,
 * arXiv:2210.17323): columns of W are quantized in order, each column's
 * rounding error spread over the later columns through U, the upper Cholesky
 * factor of the damped inverse Hessian of the layer input.  Three calls, on
 * one stream in this order; the stored codes and scales are the format of
 * rq_quantize_g64 and feed the same products.
 *
 * rq_gptq_hessian -- H = (2/T) X^T X in fp64.  X: fp16 [T, K] device (the
 * calibration inputs of the layer, one row per token), 16-byte aligned.
 * H: fp64 [K, K] device, fully overwritten.  64 <= K <= 65536, K % 64 == 0,
 * 1 <= T < 2^31, else RQ_ERR_SHAPE.
 *
 * rq_gptq_factor -- from H (consumed: overwritten): every input j whose
 * H[j][j] is 0 is dead (dead[j] = 1, H[j][j] = 1); H += damp * mean(diag H) * I;
 * U = the upper Cholesky factor of H^-1 (H^-1 = U^T U), fp64 arithmetic, U
 * written as fp32 [K, K] (zeros below the diagonal).  dead: uint8 [K] device.
 * work: fp64, K*K + K values, device, 16-byte aligned.  damp: the relative
 * damping (GPTQ's usual 0.01), 0 <= damp < 1e6 else RQ_ERR_RANGE.  The
 * factorisation is right-looking with one kernel launch per column (K
 * launches): offline cost, about K^3 / 3 fp64 operations.
 *
 * rq_gptq_g64 -- the column loop.  W: fp32 [N, K] device, overwritten with the
 * error-compensated weights each column was quantized from (dead inputs'
 * columns start at 0).  U, dead: from rq_gptq_factor (dead may be NULL: no
 * dead inputs).  codes, scales: outputs in the layout of rq_quantize_g64.
 * work: fp32 [N, 128] device.  Per row, for j = 0 .. K-1: at a group's first
 * column its scale s16 = fp16_rn(fp32 amax / qmax) is found from the group's
 * CURRENT weights; code c_j = clamp(rint(w_j / s16), +-qmax) (IEEE fp32
 * division, ties to even); e_j = (w_j - c_j s16) / U[j][j]; w_k =
 * fmaf(-e_j, U[j][k], w_k) for every k > j in ascending j.  Every operation
 * is one fp32 rounding in that order, so the result is reproducible bit for
 * bit.  A group with a non-finite weight gets scale 0x7E00 and codes 0, one
 * whose scale overflows fp16 gets 0x7C00 and codes 0; neither spreads error;
 * dev_status (optional, caller-zeroed device int) receives RQ_ERR_NONFINITE /
 * RQ_ERR_RANGE as for rq_quantize_g64.  K <= 65536.
 */
rq_status rq_gptq_hessian(const uint16_t *X, int64_t T, int64_t K, double *H,
                          rq_stream_t stream);
rq_status rq_gptq_factor(double *H, int64_t K, double damp, float *U, uint8_t *dead,
                         double *work, rq_stream_t stream);
rq_status rq_gptq_g64(float *W, int64_t N, int64_t K, int bits, const float *U,
                      const uint8_t *dead, void *codes, uint16_t *scales, float *work,
                      int *dev_status, rq_stream_t stream);

/*
 * rq_gemv_wq -- decode product y[M, N] = x[M, K] * w_hat^T for 1 <= M <= 32.
 * Streams each code and scale byte from HBM once.
 * x: fp16 [M, K] device.  codes/scales: as produced by rq_quantize_g64.
 * y: fp32 [M, N] device, fully overwritten.  Requires K % 64 == 0, N >= 1.
 * Two kernels compute it (rq_set_decode_kernel, rq_decode_kernel_for): the
 * row-tile kernel keeps the partial sums of row tiles shared by several
 * blocks in a device workspace that the library allocates the first time a
 * shape needs it (at least 32 MiB of slots and 2^18 counters per device) --
 * make that first call outside any stream capture, or use
 * rq_gemv_wq_noalloc; the cluster kernel needs no workspace.  When a later
 * shape needs a larger workspace, a larger one is allocated and the old one
 * is kept until the process exits, so CUDA graphs captured earlier stay valid.
 * Workspace sharing: every rq_gemv_wq and rq_rkv_fused call on one device uses
 * the same workspace, so two such calls that may run at the same time on the
 * GPU (e.g. on two streams with no ordering between them) race on it and can
 * give wrong results; order them on one stream or with events.
 */
rq_status rq_gemv_wq(const uint16_t *x, int64_t M, int64_t K, const void *codes,
                     const uint16_t *scales, int64_t N, int bits, float *y,
                     rq_stream_t stream);

/*
 * rq_rkv_fused -- the three receptance/key/value projections of one RWKV-7
 * time-mix block, sharing one input x, in ONE kernel launch:
 *   yR = x * w_hat_R^T,  yK = x * w_hat_K^T,  yV = x * w_hat_V^T.
 * All three weights are N x K with the same bits.  Same rules as rq_gemv_wq
 * (1 <= M <= 32), including its workspace: calls of rq_gemv_wq and
 * rq_rkv_fused that may overlap on the GPU race on it.
 */
rq_status rq_rkv_fused(const uint16_t *x, int64_t M, int64_t K, int64_t N, int bits,
                       const void *codes_r, const uint16_t *scales_r,
                       const void *codes_k, const uint16_t *scales_k,
                       const void *codes_v, const uint16_t *scales_v,
                       float *y_r, float *y_k, float *y_v, rq_stream_t stream);

/*
 * rq_gemv_wq_ex -- the decode product with a choice of output type and a
 * fused epilogue ("fp16-output / fused-epilogue" decode variants).  Same
 * product as rq_gemv_wq (1 <= M <= 32), on the row-block decode kernel, then,
 * per output, before it is stored:
 *   epilogue RQ_EPI_NONE     y
 *   epilogue RQ_EPI_RELU_SQ  max(y, 0)^2 in fp32 -- the squared-ReLU that
 *            follows the channel-mix key projection of an RWKV-7 block, so the
 *            key output can feed the value projection directly;
 *   out_dtype RQ_OUT_F32: y fp32 [M, N]; RQ_OUT_F16: y fp16 [M, N] (fp16 bit
 *            patterns, round to nearest even; values beyond fp16 become inf).
 * Other values of out_dtype / epilogue: RQ_ERR_RANGE.  y: device, 16-byte
 * aligned, fully overwritten.  Needs no workspace.
 */
#define RQ_OUT_F32 0
#define RQ_OUT_F16 1
#define RQ_EPI_NONE 0
#define RQ_EPI_RELU_SQ 1
rq_status rq_gemv_wq_ex(const uint16_t *x, int64_t M, int64_t K, const void *codes,
                        const uint16_t *scales, int64_t N, int bits, void *y, int out_dtype,
                        int epilogue, rq_stream_t stream);

/*
 * rq_rkv_fused3 -- the receptance/key/value projections in ONE launch, each
 * with its OWN input (RWKV-7 mixes a token-shifted copy of the block input
 * into each of r, k and v with its own coefficients, so the three inputs
 * differ): yR = xR * w_hat_R^T, yK = xK * w_hat_K^T, yV = xV * w_hat_V^T.
 * The "RWKV-7 Quantization Toolkit" ("Key Design") runs R/K/V in a single
 * launch; rq_rkv_fused is the shared-input form.  x_*: fp16 [M, K] device,
 * 16-byte aligned.  Outputs fp32 or (out_dtype RQ_OUT_F16) fp16 [M, N].
 * Same rules otherwise as rq_rkv_fused (1 <= M <= 32); row-block kernel, no
 * workspace.
 */
rq_status rq_rkv_fused3(const uint16_t *x_r, const uint16_t *x_k, const uint16_t *x_v,
                        int64_t M, int64_t K, int64_t N, int bits,
                        const void *codes_r, const uint16_t *scales_r,
                        const void *codes_k, const uint16_t *scales_k,
                        const void *codes_v, const uint16_t *scales_v,
                        void *y_r, void *y_k, void *y_v, int out_dtype, rq_stream_t stream);

/*
 * rq_gemm_wq -- prefill product y[M, N] = x[M, K] * w_hat^T on the tcgen05
 * tensor cores (fp16 operands, fp32 accumulation in tensor memory).  Tuned
 * for M >= 64; accepts any M >= 1.  Same layouts and rules as rq_gemv_wq.
 */
rq_status rq_gemm_wq(const uint16_t *x, int64_t M, int64_t K, const void *codes,
                     const uint16_t *scales, int64_t N, int bits, float *y,
                     rq_stream_t stream);

/*
 * rq_gemv_wq_noalloc -- rq_gemv_wq for callers that cannot have a library
 * allocate device memory.  (The pages describe no such variant; it exists for
 * this library's users.)
 *
 * Who needs it: code that records a CUDA graph (allocation is not a stream
 * operation, so while a stream is being captured it is refused or not
 * recorded), serving runtimes that reserve the device memory up front for
 * weights and caches and account for every byte, and hot loops that cannot
 * afford the implicit device synchronisation of cudaMalloc / cudaFree.
 * rq_gemv_wq splits each product over all SMs; rows shared by several blocks
 * leave partial sums in scratch that rq_gemv_wq allocates on first use.  This
 * call keeps that scratch in a fixed array inside the library instead --
 * 5 MiB of partial sums plus 16384 per-tile counters (64 KiB), present on
 * every GPU that loads the library until the process exits -- and calls no
 * allocator.
 *
 * Same arguments, result and rules as rq_gemv_wq (1 <= M <= 32; y fully
 * overwritten).  Only the row-tile kernel (see rq_set_decode_kernel) uses
 * the array: its launch must fit it -- one counter per row tile of 16 to 64
 * rows, at most 16384, and the partial sums within 5 MiB (true for every M
 * on a 148-SM B200) -- else RQ_ERR_SHAPE is returned and nothing is
 * enqueued; such a call clears the counters it uses (an asynchronous memset
 * on `stream`) and then launches the product.  The row-block, cluster and
 * tensor-core kernels keep their partial sums on chip: a call that runs on
 * one of them uses no scratch, launches only the product and has no row
 * limit of its own.
 * The first call on a device looks up the array's device address (once per
 * device, with that device current) -- make it before any stream capture.
 * Each device has its own copy of the array; calls that may overlap on the
 * same device (e.g. on two streams with no ordering between them) race on
 * it and give wrong results.
 */
rq_status rq_gemv_wq_noalloc(const uint16_t *x, int64_t M, int64_t K, const void *codes,
                             const uint16_t *scales, int64_t N, int bits, float *y,
                             rq_stream_t stream);

/*
 * rq_set_pdl -- opt in (enable != 0) or out of programmatic dependent launch
 * for the product kernels launched afterwards by this process.  With it on, a
 * product kernel may start while the previous kernel of the stream is still
 * running: it fetches its codes and scales early and waits for the previous
 * kernel's completion only before it reads x or writes y.  So with it on, the
 * kernel launched immediately before a product call must not write that
 * call's codes or scales.  Off by default.  Not thread-safe.
 */
rq_status rq_set_pdl(int enable);

/*
 * rq_set_decode_kernel -- which kernel computes the decode products
 * (rq_gemv_wq, rq_gemv_wq_noalloc, rq_rkv_fused) launched afterwards by this
 * process.  Both compute the same sums (within the products' tolerance; each
 * is deterministic for a given shape):
 *   RQ_DECODE_AUTO     (0) chosen per shape and batch size (default);
 *   RQ_DECODE_ROWTILE  (1) row tiles dealt over the SMs (stream-K), partial
 *                          tiles summed through a workspace;
 *   RQ_DECODE_CLUSTER  (2) K split over the CTAs of a thread-block cluster,
 *                          each CTA's x held in shared memory, partial sums
 *                          added through distributed shared memory;
 *   RQ_DECODE_ROWBLOCK (3) blocks of rows over the full K range, each output
 *                          finished inside one CTA; needs no workspace;
 *   RQ_DECODE_TENSOR   (4) the fifth-generation tensor cores (tcgen05):
 *                          weights dequantised to fp16(code * s16) in tensor
 *                          memory, 256-row blocks with K split over a
 *                          thread-block cluster, partial sums added through
 *                          distributed shared memory; needs no workspace.
 * Any other value is rejected with RQ_ERR_RANGE.  Not thread-safe.
 */
#define RQ_DECODE_AUTO 0
#define RQ_DECODE_ROWTILE 1
#define RQ_DECODE_CLUSTER 2
#define RQ_DECODE_ROWBLOCK 3
#define RQ_DECODE_TENSOR 4
rq_status rq_set_decode_kernel(int kernel);

/*
 * rq_decode_kernel_for -- which decode kernel (RQ_DECODE_ROWTILE,
 * RQ_DECODE_CLUSTER, RQ_DECODE_ROWBLOCK or RQ_DECODE_TENSOR) a decode
 * product of this shape would run on under the
 * current rq_set_decode_kernel selection; nmat is 1 (rq_gemv_wq) or 3
 * (rq_rkv_fused).  Host-only: launches nothing and needs no GPU.  The same
 * argument checks as the products (RQ_ERR_BITS, RQ_ERR_SHAPE); kernel NULL
 * gives RQ_ERR_NULL; a forced kernel that cannot take the shape gives
 * RQ_ERR_SHAPE, as the product would.
 */
rq_status rq_decode_kernel_for(int64_t M, int64_t K, int64_t N, int bits, int nmat,
                               int *kernel);

/*
 * rq_set_wait_limit_ns -- time limit of every bounded on-chip wait of the
 * library's kernels (default 1 s).  A kernel whose wait exceeds it stops its
 * work, sets the device status word to RQ_ERR_TIMEOUT and exits; its outputs
 * are then undefined.  0 is rejected with RQ_ERR_RANGE.
 */
rq_status rq_set_wait_limit_ns(uint64_t limit_ns);

/*
 * rq_read_device_status -- copy the library's device status word of the
 * current device to *out (RQ_OK or RQ_ERR_TIMEOUT), synchronously (it waits
 * for the device), and reset it to RQ_OK when reset != 0.
 */
rq_status rq_read_device_status(int *out, int reset);

/*
 * rq_selftest_bounded_wait -- launch a one-warp kernel that waits on an
 * mbarrier nothing ever completes.  Its bounded wait must give up after
 * limit_ns and set the device status word to RQ_ERR_TIMEOUT; the kernel then
 * exits normally.  Diagnostic for the timeout path; faults nothing.
 */
rq_status rq_selftest_bounded_wait(uint64_t limit_ns, rq_stream_t stream);

/* Static description of a status code. */
const char *rq_status_string(rq_status s);

/* Message of the last CUDA error a call of this thread returned RQ_ERR_CUDA for. */
const char *rq_last_cuda_error(void);

/* Library version, e.g. "0.1.0". */
const char *rq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* RQ_H_ */
