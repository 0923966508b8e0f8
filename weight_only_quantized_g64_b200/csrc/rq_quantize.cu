// rq_quantize.cu -- round-to-nearest, group-64, symmetric int4/int8 quantizer.
//
// Follows the "calibration-free RTN" of the "Hakureirm/rwkv7-sglang-w4gptq-1.5b"
// model card (opening summary) in its stored format ("Format & loading
// (important)": GROUP = 64, symmetric, packed codes + per-group scale) and the
// int8 w8g64 tier of its "Accuracy warning" section.  Per group:
//   amax = max|w|;  s16 = fp16_rn(amax / qmax);  c = clamp(rint(w / s16), +-qmax)
// with IEEE fp32 divisions (__fdiv_rn), fp16 round-to-nearest-even and rint
// ties-to-even (__float2int_rn), so the result is bit-exact with a scalar
// fp32 implementation of the same steps.  This translation unit must not be
// built with fast-math.
//
// Layout of the work: groups of W are contiguous (row-major W, K % 64 == 0),
// so the kernel runs flat over all N*K/64 groups.  8 threads own one group
// (eight fp32 each, two 16-byte loads, each load instruction covering whole
// 128-byte lines), a warp four groups; the group max is a 3-step
// xor-shuffle inside the 8-lane team, so the per-group work (the max, the
// division, the fp16 rounding, the reciprocal) is shared by 8 weights per
// lane.  256 B read, 34 B (int4) or 66 B (int8) written per group.
#include "rq_internal.h"
#include "rq_ptx.cuh"

namespace rq {

// rint(w / sf) with the quotient an IEEE fp32 division (ties to even), as
// __float2int_rn(__fdiv_rn(w, sf)), but dividing only where it can matter.
// t = w * r with r = 1/sf rounded to nearest lies within |q| * 2^-23 (1 + 2^-25)
// of the exact quotient q, and the rounded quotient fl(q) within |q| * 2^-24
// of it; when t is more than |t| * 2^-21 away from every half-integer, no
// half-integer separates t from fl(q) and both round to the same integer.
// Otherwise (ties and near-ties, e.g. weights on the grid) the exact division
// decides.  sf must be finite and non-zero; |t| stays far below 2^22 here, so
// t - floor(t) is exact.
__device__ __forceinline__ int rint_quotient(float w, float sf, float r) {
    const float t = __fmul_rn(w, r);
    const float f = __fsub_rn(t, floorf(t));
    if (fabsf(__fsub_rn(f, 0.5f)) > fabsf(t) * 4.76837158203125e-7f)   // 2^-21
        return __float2int_rn(t);
    return __float2int_rn(__fdiv_rn(w, sf));
}

// max that propagates NaN (the PTX max.NaN), so one reduction also tells
// whether the group holds a non-finite weight.
__device__ __forceinline__ float max_nan(float a, float b) {
    float d;
    asm("max.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
    return d;
}

// clamp(rint(fl(w / sf)), +-QMAX) without a division where that is provably
// the same value: t = w * r (r = 1/sf rounded to nearest) lies within
// |q| * 2^-23 (1 + 2^-25) of the exact quotient q and fl(q) within |q| * 2^-24
// of it, so when t (clamped to +-QMAX, which both sides would clamp to) is
// more than (QMAX + 1) * 2^-21 away from every half-integer, no half-integer
// separates it from fl(q).  Near ties (weights on the grid) take the IEEE
// division.  Rounding: t + 1.5 * 2^23 rounds to an integer, ties to even, for
// |t| <= 2^22; its bit pattern minus that of 1.5 * 2^23 is the integer.
//
// With a normal fp16 scale the clamp never acts: s16 >= (amax / qmax)(1 -
// 2^-11)(1 - 2^-24), so |t| <= qmax (1 + 5e-4) (1 + 2^-24) < qmax + 0.5, and
// the same bound holds for the IEEE quotient; only subnormal scales (relative
// rounding up to 1/2) need it (CLAMP).
template <int QMAX, bool CLAMP>
__device__ __forceinline__ int rint_quotient_q(float w, float sf, float r) {
    constexpr float kNear = static_cast<float>(QMAX + 1) * 4.76837158203125e-7f;   // 2^-21
    constexpr float kMagic = 12582912.0f;                                          // 1.5 * 2^23
    float t = __fmul_rn(w, r);
    if constexpr (CLAMP) t = fminf(fmaxf(t, static_cast<float>(-QMAX)), static_cast<float>(QMAX));
    const float m = __fadd_rn(t, kMagic);
    const float d = __fsub_rn(t, __fsub_rn(m, kMagic));
    if (fabsf(__fsub_rn(fabsf(d), 0.5f)) > kNear) return __float_as_int(m) - __float_as_int(kMagic);
    const int q = __float2int_rn(__fdiv_rn(w, sf));
    return CLAMP ? max(-QMAX, min(QMAX, q)) : q;
}

// rint_quotient_q<QMAX, true> returned as the float value of the code (for
// the error sums of the scale search): q = (t + 1.5 * 2^23) - 1.5 * 2^23 is
// rint(t) exactly, with no integer conversion on the common path; the
// near-tie test is the one comparison |t - q| >= 1/2 - (QMAX + 1) 2^-21 (t - q
// is exact and at most 1/2 in magnitude), the same decision as above.
template <int QMAX>
__device__ __forceinline__ float rint_quotient_qf(float w, float sf, float r) {
    constexpr float kTie = 0.5f - static_cast<float>(QMAX + 1) * 4.76837158203125e-7f;
    constexpr float kMagic = 12582912.0f;                                          // 1.5 * 2^23
    float t = __fmul_rn(w, r);
    t = fminf(fmaxf(t, static_cast<float>(-QMAX)), static_cast<float>(QMAX));
    const float q = __fsub_rn(__fadd_rn(t, kMagic), kMagic);
    if (fabsf(__fsub_rn(t, q)) < kTie) return q;
    const int qi = __float2int_rn(__fdiv_rn(w, sf));
    return static_cast<float>(max(-QMAX, min(QMAX, qi)));
}

// One group held by 8 lanes, 8 weights per lane (positions 4l..4l+3 and
// 32+4l..32+4l+3 of the group): scale bits, codes (only their low 4 / 8 bits
// are meaningful: the packing keeps just those), status (0, 5 = NONFINITE,
// 6 = RANGE).
template <int BITS>
__device__ __forceinline__ void quantize_group8(const float4 (&v)[2], unsigned mask8,
                                                uint16_t& s_bits, int (&c)[8], int& status) {
    constexpr int kQmax = BITS == 4 ? 7 : 127;
    const float w[8] = {v[0].x, v[0].y, v[0].z, v[0].w, v[1].x, v[1].y, v[1].z, v[1].w};
    float a = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) a = max_nan(a, fabsf(w[i]));
#pragma unroll
    for (int off = 4; off > 0; off >>= 1) a = max_nan(a, __shfl_xor_sync(mask8, a, off));
    // a is NaN or +inf exactly when the group holds a non-finite weight

    const float s32 = __fdiv_rn(a, static_cast<float>(kQmax));
    const __half s16 = __float2half_rn(s32);
    s_bits = __half_as_ushort(s16);
    const float sf = __half2float(s16);
    status = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) c[i] = 0;
    if (!isfinite(a)) {
        s_bits = 0x7E00u;
        status = 5;  // RQ_ERR_NONFINITE
    } else if (s_bits == 0x7C00u) {
        status = 6;  // RQ_ERR_RANGE
    } else if (sf != 0.0f) {
        const float r = __frcp_rn(sf);
        if (sf >= 6.103515625e-05f) {
            // normal fp16 scale: no clamp needed.  The fast value for every
            // weight first; if any of the lane's weights is a near tie, those
            // are redone with the IEEE division afterwards (rare), so the
            // common path has no branch per weight.  d = t - rint(t) is exact
            // and |d| <= 1/2, so "more than kNear away from a half-integer"
            // is |d| < 1/2 - kNear (exact in fp32).  The code is taken from
            // the low bits of m: m's bit pattern is that of 1.5 * 2^23 plus
            // the integer, and 1.5 * 2^23 has zero low bytes.
            constexpr float kTie = 0.5f - static_cast<float>(kQmax + 1) * 4.76837158203125e-7f;
            constexpr float kMagic = 12582912.0f;
            bool any_slow = false;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float t = __fmul_rn(w[i], r);
                const float m = __fadd_rn(t, kMagic);
                const float d = __fsub_rn(t, __fsub_rn(m, kMagic));
                c[i] = __float_as_int(m);
                any_slow |= fabsf(d) >= kTie;
            }
            if (any_slow) {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float t = __fmul_rn(w[i], r);
                    const float d = __fsub_rn(t, __fsub_rn(__fadd_rn(t, kMagic), kMagic));
                    if (fabsf(d) >= kTie) c[i] = __float2int_rn(__fdiv_rn(w[i], sf));
                }
            }
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) c[i] = rint_quotient_q<kQmax, true>(w[i], sf, r);
        }
    }
}

template <int BITS>
__device__ __forceinline__ void store_group8(int64_t gid, int l8, uint16_t s_bits, const int (&c)[8],
                                             uint8_t* __restrict__ codes,
                                             uint16_t* __restrict__ scales) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int* ch = c + 4 * h;
        if (BITS == 4) {
            const uint16_t packed = static_cast<uint16_t>((ch[0] & 0xF) | ((ch[1] & 0xF) << 4) |
                                                          ((ch[2] & 0xF) << 8) | ((ch[3] & 0xF) << 12));
            __stcs(reinterpret_cast<unsigned short*>(codes + gid * 32 + h * 16 + l8 * 2), packed);
        } else {
            const uint32_t packed = (ch[0] & 0xFF) | ((ch[1] & 0xFF) << 8) | ((ch[2] & 0xFF) << 16) |
                                    (static_cast<uint32_t>(ch[3] & 0xFF) << 24);
            __stcs(reinterpret_cast<unsigned int*>(codes + gid * 64 + h * 32 + l8 * 4), packed);
        }
    }
    if (l8 == 0) scales[gid] = s_bits;
}

// NONFINITE overrides everything; RANGE only replaces OK.
__device__ __forceinline__ void raise_status(int* dev_status, int status) {
    if (dev_status == nullptr) return;
    if (status == 5) atomicExch(dev_status, 5);
    else if (status == 6) atomicCAS(dev_status, 0, 6);
}

// Eight lanes per group, four groups per warp.  An 8-lane team takes groups
// t + T*(kQU*i + j), j < kQU, for i = 0, 1, ... (T = teams in the grid): the
// kQU groups' loads (two 16-byte loads per lane each) are issued together.
constexpr int kQU = 2;

template <int BITS>
__global__ void __launch_bounds__(256) quantize_g64_kernel(const float4* __restrict__ W,
                                                           int64_t n_groups,
                                                           uint8_t* __restrict__ codes,
                                                           uint16_t* __restrict__ scales,
                                                           int* __restrict__ dev_status) {
    const int l8 = threadIdx.x & 7;
    const unsigned mask8 = 0xFFu << (threadIdx.x & 24);
    const int64_t first = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 3;
    const int64_t step = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 3;

    for (int64_t g0 = first; g0 < n_groups; g0 += kQU * step) {
        float4 v[kQU][2];
#pragma unroll
        for (int j = 0; j < kQU; ++j) {
            const int64_t gid = g0 + j * step;
#pragma unroll
            for (int h = 0; h < 2; ++h)
                v[j][h] = gid < n_groups ? __ldcs(&W[gid * 16 + h * 8 + l8]) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        int status_any = 0;
#pragma unroll
        for (int j = 0; j < kQU; ++j) {
            const int64_t gid = g0 + j * step;
            if (gid >= n_groups) break;   // uniform over the team
            uint16_t s_bits;
            int c[8], status;
            quantize_group8<BITS>(v[j], mask8, s_bits, c, status);
            store_group8<BITS>(gid, l8, s_bits, c, codes, scales);
            if (status == 5 || (status == 6 && status_any == 0)) status_any = status;
        }
        if (l8 == 0 && status_any != 0) raise_status(dev_status, status_any);
    }
}

// Blocks of 256 threads: as many as are resident on every SM at once (the
// loop walks the rest), no more than the groups need.
static int quantize_grid(int64_t n_groups, const void* kern) {
    int dev = 0, sms = 0, per_sm = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
        sms = 1;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 256, 0) != cudaSuccess ||
        per_sm <= 0)
        per_sm = 1;
    const int64_t need = (n_groups + 31) / 32;
    const int64_t full = static_cast<int64_t>(sms) * per_sm;
    return static_cast<int>(need < full ? need : full);
}

cudaError_t launch_quantize(const float* W, int64_t n_groups, int bits, void* codes,
                            uint16_t* scales, int* dev_status, cudaStream_t s) {
    if (n_groups <= 0) return cudaSuccess;
    const int threads = 256;
    if (bits == 4) {
        const int blocks = quantize_grid(n_groups, reinterpret_cast<const void*>(quantize_g64_kernel<4>));
        quantize_g64_kernel<4><<<static_cast<unsigned>(blocks), threads, 0, s>>>(
            reinterpret_cast<const float4*>(W), n_groups, static_cast<uint8_t*>(codes), scales,
            dev_status);
    } else {
        const int blocks = quantize_grid(n_groups, reinterpret_cast<const void*>(quantize_g64_kernel<8>));
        quantize_g64_kernel<8><<<static_cast<unsigned>(blocks), threads, 0, s>>>(
            reinterpret_cast<const float4*>(W), n_groups, static_cast<uint8_t*>(codes), scales,
            dev_status);
    }
    return cudaGetLastError();
}


// ------------------------------------------- E[x^2]-weighted scale search --
//
// "rwkv-quant: uma matriz em bf16 elimina 39% das perdas na quantização do
// RWKV-7 2.9B", section "Dois presets e seis tamanhos": a group's scale is
// chosen by a search weighted by E[x^2], the mean square of the input
// channel's activation.  On the symmetric g64 grid: candidate j has scale
// s16_j = fp16_rn(fp32(amax * f[j]) / qmax) and RTN codes against it; its
// error is sum_k e2[k] * (w_k - c_k * s16_j)^2 over the group's 64 k, in k
// order, each operation one IEEE fp32 rounding (explicit _rn intrinsics: no
// contraction); the candidate with the smallest error wins, the earlier one
// on a tie, and one whose scale overflows is never chosen (if every one
// does, the group is quantized by RTN).
//
// Layout of the work: a team of TL lanes per group (16, or 8 when there are
// at most 8 candidates, so a warp takes 2 or 4 groups at once).  Lane j
// evaluates candidate j over all 64 weights in k order, reading the weights
// and E[x^2] four at a time (the same address for every lane of the team:
// one broadcast load), so its sum runs in the same order as a scalar loop;
// the team's first lane then scans the candidates in order (the same
// comparisons as a sequential argmin, NaN included).  Each lane also holds
// 64 / TL weights of the group for the max and for the final codes.
template <int BITS, int TL>
__global__ void __launch_bounds__(256) quantize_g64_ex2_kernel(
    const float4* __restrict__ W, int64_t n_groups, int64_t groups_per_row,
    const float4* __restrict__ e2, const float* __restrict__ factors, int nf,
    uint8_t* __restrict__ codes, uint16_t* __restrict__ scales, int32_t* __restrict__ chosen,
    int* __restrict__ dev_status) {
    constexpr int kQmax = BITS == 4 ? 7 : 127;
    constexpr int NV = 16 / TL;                              // float4 of weights per lane
    const int lt = threadIdx.x & (TL - 1);                   // lane in the team
    const int base = threadIdx.x & (31 & ~(TL - 1));         // first lane of the team
    const unsigned tmask = (TL == 32 ? 0xFFFFFFFFu : ((1u << TL) - 1u)) << base;
    const int64_t first = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) / TL;
    const int64_t step = (static_cast<int64_t>(gridDim.x) * blockDim.x) / TL;
    const float fj = lt < nf ? factors[lt] : 1.0f;

    for (int64_t gid = first; gid < n_groups; gid += step) {
        const float4* wg = W + gid * 16;
        const float4* eg = e2 + (gid % groups_per_row) * 16;
        float4 v[NV];
#pragma unroll
        for (int h = 0; h < NV; ++h) v[h] = __ldg(&wg[h * TL + lt]);
        // max |w| over the group; NaN-propagating, so it also flags a
        // non-finite weight (NaN or +inf exactly then)
        float a = 0.0f;
#pragma unroll
        for (int h = 0; h < NV; ++h)
            a = max_nan(max_nan(a, max_nan(fabsf(v[h].x), fabsf(v[h].y))),
                        max_nan(fabsf(v[h].z), fabsf(v[h].w)));
#pragma unroll
        for (int off = TL / 2; off > 0; off >>= 1) a = max_nan(a, __shfl_xor_sync(tmask, a, off));
        const bool all_finite = isfinite(a);

        // ---- candidate lt: scale, then its error over the 64 weights in order
        const float a32 = __fmul_rn(a, fj);
        const __half s16j = __float2half_rn(__fdiv_rn(a32, static_cast<float>(kQmax)));
        const float sfj = __half2float(s16j);
        const bool valid = lt < nf && __half_as_ushort(s16j) != 0x7C00u;
        const float rj = (sfj != 0.0f && valid) ? __frcp_rn(sfj) : 0.0f;
        float err = 0.0f;
        if (all_finite) {
#pragma unroll 2
            for (int k4 = 0; k4 < 16; ++k4) {
                const float4 wq = __ldg(&wg[k4]);
                const float4 eq = __ldg(&eg[k4]);
                const float wk[4] = {wq.x, wq.y, wq.z, wq.w};
                const float ek[4] = {eq.x, eq.y, eq.z, eq.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float cf = sfj != 0.0f ? rint_quotient_qf<kQmax>(wk[i], sfj, rj) : 0.0f;
                    const float t = __fmul_rn(cf, sfj);
                    const float d = __fsub_rn(wk[i], t);
                    err = __fadd_rn(err, __fmul_rn(ek[i], __fmul_rn(d, d)));
                }
            }
        }
        // ---- the team's first lane scans the candidates in order
        int best = -1;
        float best_err = 0.0f;
        for (int j = 0; j < nf; ++j) {
            const float ej = __shfl_sync(tmask, err, base + j);
            const int vj = __shfl_sync(tmask, valid ? 1 : 0, base + j);
            if (vj && (best < 0 || ej < best_err)) {
                best = j;
                best_err = ej;
            }
        }
        best = __shfl_sync(tmask, best, base);

        // ---- the chosen scale (or RTN when no candidate is valid) and codes
        const float fb = best >= 0 ? __shfl_sync(tmask, fj, base + best) : 1.0f;
        const float s32 = best >= 0 ? __fdiv_rn(__fmul_rn(a, fb), static_cast<float>(kQmax))
                                    : __fdiv_rn(a, static_cast<float>(kQmax));
        const __half s16 = __float2half_rn(s32);
        uint16_t s_bits = __half_as_ushort(s16);
        const float sf = __half2float(s16);
        int status = 0;
        int c[4 * NV];
#pragma unroll
        for (int i = 0; i < 4 * NV; ++i) c[i] = 0;
        if (!all_finite) {
            s_bits = 0x7E00u;
            status = 5;  // RQ_ERR_NONFINITE
        } else if (s_bits == 0x7C00u) {
            status = 6;  // RQ_ERR_RANGE
        } else if (sf != 0.0f) {
            const float r = __frcp_rn(sf);
#pragma unroll
            for (int h = 0; h < NV; ++h) {
                const float wv[4] = {v[h].x, v[h].y, v[h].z, v[h].w};
#pragma unroll
                for (int i = 0; i < 4; ++i) c[4 * h + i] = rint_quotient_q<kQmax, true>(wv[i], sf, r);
            }
        }
#pragma unroll
        for (int h = 0; h < NV; ++h) {
            const int* ch = c + 4 * h;
            const int pos = h * TL + lt;                     // float4 index within the group
            if (BITS == 4) {
                const uint16_t packed = static_cast<uint16_t>((ch[0] & 0xF) | ((ch[1] & 0xF) << 4) |
                                                              ((ch[2] & 0xF) << 8) | ((ch[3] & 0xF) << 12));
                __stcs(reinterpret_cast<unsigned short*>(codes + gid * 32 + pos * 2), packed);
            } else {
                const uint32_t packed = (ch[0] & 0xFF) | ((ch[1] & 0xFF) << 8) | ((ch[2] & 0xFF) << 16) |
                                        (static_cast<uint32_t>(ch[3] & 0xFF) << 24);
                __stcs(reinterpret_cast<unsigned int*>(codes + gid * 64 + pos * 4), packed);
            }
        }
        if (lt == 0) {
            scales[gid] = s_bits;
            if (chosen != nullptr) chosen[gid] = (all_finite && best >= 0) ? best : 0;
            if (dev_status != nullptr) {
                if (status == 5) atomicExch(dev_status, 5);
                else if (status == 6) atomicCAS(dev_status, 0, 6);
            }
        }
    }
}

template <int BITS, int TL>
static cudaError_t launch_ex2_cfg(const float* W, int64_t n_groups, int64_t groups_per_row,
                                  const float* e2, const float* factors, int nf, void* codes,
                                  uint16_t* scales, int32_t* chosen, int* dev_status, cudaStream_t s) {
    auto kern = quantize_g64_ex2_kernel<BITS, TL>;
    // (quantize_grid counts 32 groups per block of 256 threads: a block holds
    // 256 / TL groups here)
    const int blocks = quantize_grid(n_groups * TL / 8, reinterpret_cast<const void*>(kern));
    kern<<<static_cast<unsigned>(blocks), 256, 0, s>>>(
        reinterpret_cast<const float4*>(W), n_groups, groups_per_row,
        reinterpret_cast<const float4*>(e2), factors, nf, static_cast<uint8_t*>(codes), scales,
        chosen, dev_status);
    return cudaGetLastError();
}

cudaError_t launch_quantize_ex2(const float* W, int64_t N, int64_t K, int bits, const float* e2,
                                const float* factors, int nf, void* codes, uint16_t* scales,
                                int32_t* chosen, int* dev_status, cudaStream_t s) {
    const int64_t groups_per_row = K / kGroup;
    const int64_t n_groups = N * groups_per_row;
    if (n_groups <= 0) return cudaSuccess;
    if (bits == 4)
        return nf <= 8 ? launch_ex2_cfg<4, 8>(W, n_groups, groups_per_row, e2, factors, nf, codes, scales,
                                              chosen, dev_status, s)
                       : launch_ex2_cfg<4, 16>(W, n_groups, groups_per_row, e2, factors, nf, codes, scales,
                                               chosen, dev_status, s);
    return nf <= 8 ? launch_ex2_cfg<8, 8>(W, n_groups, groups_per_row, e2, factors, nf, codes, scales,
                                          chosen, dev_status, s)
                   : launch_ex2_cfg<8, 16>(W, n_groups, groups_per_row, e2, factors, nf, codes, scales,
                                           chosen, dev_status, s);
}

}  // namespace rq
