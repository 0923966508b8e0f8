// rq_quantize_presets.cu -- quantizers of the two rwkv-quant preset formats.
//
// "rwkv-quant: uma matriz em bf16 elimina 39% das perdas na quantização do
// RWKV-7 2.9B", section "Dois presets e seis tamanhos": REDUCTION keeps the
// projections in 8 bits, symmetric, groups of 16 weights; COMPRESSION in 4
// bits, asymmetric, in super-blocks, groups of 32; in both presets the
// groups' scale (and offset) is chosen by a search weighted by E[x^2], the
// mean square of the input channel.
//
// int8 g16 symmetric: per group of 16 (one thread per group, four float4
//   loads): amax; candidate j: s16 = fp16_rn(fp32(amax * f_j) / 127), codes
//   rint(w / s16) clamped to +-127, error sum_k e2 (w - c s16)^2 in k order;
//   smallest error wins, the earlier candidate on a tie; no search = RTN.
// int4 g32 asymmetric in super-blocks of 8 groups (one warp per super-block,
//   8 weights per lane, group g on lanes 4g..4g+3): lo = min(0, min w), hi =
//   max(0, max w); candidate j: lo_j = lo f_j, hi_j = hi f_j, s_j =
//   (hi_j - lo_j) / 15, codes rint((w - lo_j) / s_j) clamped to [0, 15],
//   error sum_k e2 (w - (q s_j + lo_j))^2 in k order (each group's 32 terms
//   summed by one lane from shared memory); ds = fp16_rn(max s / 63), dm =
//   fp16_rn(max(-o) / 63); 6-bit sub-codes a = rint(s / ds), b = rint(-o / dm);
//   stored scale S = ds a, offset O = -(dm b); codes rint((w - O) / S)
//   clamped to [0, 15].
// Every operation is one IEEE fp32 rounding in the order written (explicit
// _rn intrinsics, no contraction), so codes, scales and sub-codes are
// bit-exact with a scalar fp32 implementation of the same steps.
#include <cuda_fp16.h>

#include "rq_internal.h"

namespace rq {

// rint(w / s) of an IEEE fp32 division: the product with the rounded
// reciprocal decides wherever it lies more than |t| 2^-21 from a
// half-integer (both round alike there); ties and near-ties divide exactly.
__device__ __forceinline__ int preset_rint_quot(float w, float s, float r) {
    const float t = __fmul_rn(w, r);
    const float f = __fsub_rn(t, floorf(t));
    if (fabsf(__fsub_rn(f, 0.5f)) > fabsf(t) * 4.76837158203125e-7f) return __float2int_rn(t);
    return __float2int_rn(__fdiv_rn(w, s));
}

__device__ __forceinline__ void preset_status(int* dev_status, int st) {
    if (dev_status == nullptr || st == 0) return;
    if (st == 5) atomicExch(dev_status, 5);
    else atomicCAS(dev_status, 0, 6);
}

// ------------------------------------------------------- int8, groups of 16 --
__global__ void __launch_bounds__(256) quantize_p8_kernel(const float4* __restrict__ W, int64_t n_groups,
                                                          int64_t groups_per_row,
                                                          const float* __restrict__ e2,
                                                          const float* __restrict__ factors, int nf,
                                                          uint8_t* __restrict__ codes,
                                                          uint16_t* __restrict__ scales,
                                                          int32_t* __restrict__ chosen,
                                                          int* __restrict__ dev_status) {
    constexpr int kQmax = 127;
    const int64_t step = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t gid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; gid < n_groups;
         gid += step) {
        float w[16];
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            const float4 f4 = __ldcs(&W[gid * 4 + v]);
            w[4 * v] = f4.x; w[4 * v + 1] = f4.y; w[4 * v + 2] = f4.z; w[4 * v + 3] = f4.w;
        }
        bool finite = true;
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            finite = finite && isfinite(w[i]);
            amax = fmaxf(amax, fabsf(w[i]));
        }
        const float* e = e2 != nullptr ? e2 + (gid % groups_per_row) * 16 : nullptr;
        uint16_t s_bits = 0;
        int best = -1, status = 0;
        float best_err = 0.0f;
        if (!finite) {
            s_bits = 0x7E00u;
            status = 5;
        } else {
            const int ncand = e != nullptr ? nf : 1;
            for (int j = 0; j < ncand; ++j) {
                const float a32 = e != nullptr ? __fmul_rn(amax, factors[j]) : amax;
                const uint16_t sj = __half_as_ushort(__float2half_rn(__fdiv_rn(a32, static_cast<float>(kQmax))));
                if (sj == 0x7C00u) continue;
                float err = 0.0f;
                if (e != nullptr) {
                    const float sf = __half2float(__ushort_as_half(sj));
                    const float r = sf != 0.0f ? __frcp_rn(sf) : 0.0f;
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        int c = 0;
                        if (sf != 0.0f) c = max(-kQmax, min(kQmax, preset_rint_quot(w[i], sf, r)));
                        const float d = __fsub_rn(w[i], __fmul_rn(static_cast<float>(c), sf));
                        err = __fadd_rn(err, __fmul_rn(__ldg(e + i), __fmul_rn(d, d)));
                    }
                }
                if (best < 0 || err < best_err) {
                    best = j;
                    best_err = err;
                    s_bits = sj;
                }
            }
            if (best < 0) {
                // every candidate's scale overflows: RTN decides
                s_bits = __half_as_ushort(__float2half_rn(__fdiv_rn(amax, static_cast<float>(kQmax))));
                best = 0;
                if (s_bits == 0x7C00u) status = 6;
            }
        }
        const float sf = __half2float(__ushort_as_half(s_bits));
        uint32_t packed[4] = {0u, 0u, 0u, 0u};
        if (status == 0 && sf != 0.0f) {
            const float r = __frcp_rn(sf);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int c = max(-kQmax, min(kQmax, preset_rint_quot(w[i], sf, r)));
                packed[i >> 2] |= static_cast<uint32_t>(c & 0xFF) << (8 * (i & 3));
            }
        }
        *reinterpret_cast<uint4*>(codes + gid * 16) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
        scales[gid] = s_bits;
        if (chosen != nullptr) chosen[gid] = (status == 0 && best >= 0) ? best : 0;
        preset_status(dev_status, status);
    }
}

// ------------------------------------- int4, groups of 32 in super-blocks --
constexpr int kP4Warps = 8;   // super-blocks per CTA (one per warp)

__global__ void __launch_bounds__(kP4Warps * 32) quantize_p4a_kernel(
    const float4* __restrict__ W, int64_t n_sb, int64_t sb_per_row, const float* __restrict__ e2,
    const float* __restrict__ factors, int nf, uint8_t* __restrict__ codes, uint8_t* __restrict__ sub,
    uint16_t* __restrict__ sup, int32_t* __restrict__ chosen, int* __restrict__ dev_status) {
    __shared__ float ws[kP4Warps][256];
    __shared__ float es[kP4Warps][256];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int grp = lane >> 2;              // the lane's group (8 weights per lane)
    const int gl = lane & 3;                // lane within the group
    const int64_t wstep = static_cast<int64_t>(gridDim.x) * kP4Warps;
    for (int64_t sb = static_cast<int64_t>(blockIdx.x) * kP4Warps + warp; sb < n_sb; sb += wstep) {
        const float4 v0 = __ldcs(&W[sb * 64 + 2 * lane]);
        const float4 v1 = __ldcs(&W[sb * 64 + 2 * lane + 1]);
        const float w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        // range seeds +0 and takes a weight only when strictly beyond it, so a
        // range end is +0 or a weight of the right sign, never -0
        bool fin = true;
        float lo = 0.0f, hi = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            fin = fin && isfinite(w[i]);
            if (w[i] < lo) lo = w[i];
            if (w[i] > hi) hi = w[i];
        }
        const bool all_finite = __all_sync(0xffffffffu, fin);
        uint8_t* sub_sb = sub + sb * 16;
        uint16_t* sup_sb = sup + sb * 2;
        uint32_t* code_sb = reinterpret_cast<uint32_t*>(codes + sb * 128);
        if (!all_finite) {
            code_sb[lane] = 0u;
            if (lane < 16) sub_sb[lane] = 0;
            if (lane < 2) sup_sb[lane] = 0x7E00u;
            if (chosen != nullptr && gl == 0) chosen[sb * 8 + grp] = 0;
            if (lane == 0) preset_status(dev_status, 5);
            continue;
        }
        // the group's range over its 4 lanes (min/max are exact in any order)
#pragma unroll
        for (int off = 1; off < 4; off <<= 1) {
            const float lo2 = __shfl_xor_sync(0xffffffffu, lo, off);
            const float hi2 = __shfl_xor_sync(0xffffffffu, hi, off);
            if (lo2 < lo) lo = lo2;
            if (hi2 > hi) hi = hi2;
        }
        // ---- the search: lane gl of group grp evaluates candidates gl, gl+4, ...
        float s_best = 0.0f, o_best = 0.0f;
        int j_best = 0;
        if (e2 != nullptr) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                ws[warp][8 * lane + i] = w[i];
                es[warp][8 * lane + i] = __ldg(e2 + (sb % sb_per_row) * 256 + 8 * lane + i);
            }
            __syncwarp();
            const float* wg = &ws[warp][32 * grp];
            const float* eg = &es[warp][32 * grp];
            float my_err[4];
            for (int c = 0; c < 4; ++c) {
                const int j = gl + 4 * c;
                my_err[c] = 0.0f;
                if (j >= nf) continue;
                const float loj = __fmul_rn(lo, factors[j]);
                const float hij = __fmul_rn(hi, factors[j]);
                const float sj = __fdiv_rn(__fsub_rn(hij, loj), 15.0f);
                const float r = sj != 0.0f ? __frcp_rn(sj) : 0.0f;
                float err = 0.0f;
                for (int i = 0; i < 32; ++i) {
                    int q = 0;
                    if (sj != 0.0f) q = max(0, min(15, preset_rint_quot(__fsub_rn(wg[i], loj), sj, r)));
                    const float u = __fadd_rn(__fmul_rn(static_cast<float>(q), sj), loj);
                    const float d = __fsub_rn(wg[i], u);
                    err = __fadd_rn(err, __fmul_rn(eg[i], __fmul_rn(d, d)));
                }
                my_err[c] = err;
            }
            // sequential argmin over j = 0 .. nf-1 (the first minimum wins)
            int best = -1;
            float best_err = 0.0f;
            for (int j = 0; j < nf; ++j) {
                const int c = j >> 2;
                float ej = 0.0f;
#pragma unroll
                for (int cc = 0; cc < 4; ++cc)
                    if (cc == c) ej = my_err[cc];
                ej = __shfl_sync(0xffffffffu, ej, (lane & ~3) + (j & 3));
                if (best < 0 || ej < best_err) {
                    best = j;
                    best_err = ej;
                }
            }
            j_best = best;
            const float lob = __fmul_rn(lo, factors[best]);
            const float hib = __fmul_rn(hi, factors[best]);
            s_best = __fdiv_rn(__fsub_rn(hib, lob), 15.0f);
            o_best = lob;
            __syncwarp();
        } else {
            s_best = __fdiv_rn(__fsub_rn(hi, lo), 15.0f);
            o_best = lo;
        }
        // ---- super-block scales
        // maxima seeded with +0 and taken only when strictly larger (a -0
        // offset never turns the super-scale into -0)
        float smax = s_best > 0.0f ? s_best : 0.0f;
        float omax = -o_best > 0.0f ? -o_best : 0.0f;
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
            const float s2 = __shfl_xor_sync(0xffffffffu, smax, off);
            const float o2 = __shfl_xor_sync(0xffffffffu, omax, off);
            if (s2 > smax) smax = s2;
            if (o2 > omax) omax = o2;
        }
        const uint16_t ds = __half_as_ushort(__float2half_rn(__fdiv_rn(smax, 63.0f)));
        const uint16_t dm = __half_as_ushort(__float2half_rn(__fdiv_rn(omax, 63.0f)));
        if (lane == 0) {
            sup_sb[0] = ds;
            sup_sb[1] = dm;
        }
        if (ds == 0x7C00u || dm == 0x7C00u) {
            code_sb[lane] = 0u;
            if (lane < 16) sub_sb[lane] = 0;
            if (chosen != nullptr && gl == 0) chosen[sb * 8 + grp] = j_best;
            if (lane == 0) preset_status(dev_status, 6);
            continue;
        }
        const float dsf = __half2float(__ushort_as_half(ds));
        const float dmf = __half2float(__ushort_as_half(dm));
        int a = 0, b = 0;
        if (dsf != 0.0f) a = max(0, min(63, __float2int_rn(__fdiv_rn(s_best, dsf))));
        if (dmf != 0.0f) b = max(0, min(63, __float2int_rn(__fdiv_rn(-o_best, dmf))));
        const float S = __fmul_rn(dsf, static_cast<float>(a));
        const float O = -__fmul_rn(dmf, static_cast<float>(b));
        uint32_t packed = 0;
        if (S != 0.0f) {
            const float r = __frcp_rn(S);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int q = max(0, min(15, preset_rint_quot(__fsub_rn(w[i], O), S, r)));
                packed |= static_cast<uint32_t>(q) << (4 * i);
            }
        }
        code_sb[lane] = packed;
        if (gl == 0) {
            sub_sb[2 * grp] = static_cast<uint8_t>(a);
            sub_sb[2 * grp + 1] = static_cast<uint8_t>(b);
            if (chosen != nullptr) chosen[sb * 8 + grp] = j_best;
        }
    }
}

static int preset_grid(int64_t items_per_block, int64_t items, const void* kern, int threads) {
    int dev = 0, sms = 0, per_sm = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
        sms = 1;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, 0) != cudaSuccess ||
        per_sm <= 0)
        per_sm = 1;
    const int64_t need = (items + items_per_block - 1) / items_per_block;
    const int64_t full = static_cast<int64_t>(sms) * per_sm;
    return static_cast<int>(need < full ? need : full);
}

cudaError_t launch_quantize_p8(const float* W, int64_t N, int64_t K, const float* e2,
                               const float* factors, int nf, void* codes, uint16_t* scales,
                               int32_t* chosen, int* dev_status, cudaStream_t s) {
    const int64_t n_groups = N * (K / 16);
    if (n_groups <= 0) return cudaSuccess;
    const int blocks = preset_grid(256, n_groups, reinterpret_cast<const void*>(quantize_p8_kernel), 256);
    quantize_p8_kernel<<<blocks, 256, 0, s>>>(reinterpret_cast<const float4*>(W), n_groups, K / 16, e2,
                                              factors, nf, static_cast<uint8_t*>(codes), scales, chosen,
                                              dev_status);
    return cudaGetLastError();
}

cudaError_t launch_quantize_p4a(const float* W, int64_t N, int64_t K, const float* e2,
                                const float* factors, int nf, void* codes, uint8_t* sub, uint16_t* sup,
                                int32_t* chosen, int* dev_status, cudaStream_t s) {
    const int64_t n_sb = N * (K / 256);
    if (n_sb <= 0) return cudaSuccess;
    const int blocks = preset_grid(kP4Warps, n_sb, reinterpret_cast<const void*>(quantize_p4a_kernel),
                                   kP4Warps * 32);
    quantize_p4a_kernel<<<blocks, kP4Warps * 32, 0, s>>>(reinterpret_cast<const float4*>(W), n_sb, K / 256,
                                                         e2, factors, nf, static_cast<uint8_t*>(codes),
                                                         sub, sup, chosen, dev_status);
    return cudaGetLastError();
}

}  // namespace rq
