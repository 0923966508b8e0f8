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
// so the kernel runs flat over all N*K/64 groups.  16 threads own one group
// (four fp32 each, one 16-byte load), a warp two groups; the group max is a
// 4-step xor-shuffle inside the 16-lane half.  Bandwidth-bound: 256 B read,
// 34 B (int4) or 66 B (int8) written per group.
#include "rq_internal.h"
#include "rq_ptx.cuh"

namespace rq {

template <int BITS>
__global__ void __launch_bounds__(256) quantize_g64_kernel(const float4* __restrict__ W,
                                                           int64_t n_groups,
                                                           uint8_t* __restrict__ codes,
                                                           uint16_t* __restrict__ scales,
                                                           int* __restrict__ dev_status) {
    constexpr int kQmax = BITS == 4 ? 7 : 127;
    const int lane16 = threadIdx.x & 15;
    const unsigned half_mask = 0xFFFFu << (threadIdx.x & 16);
    const int64_t first = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 4;
    const int64_t step = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 4;

    for (int64_t gid = first; gid < n_groups; gid += step) {
        const float4 v = __ldcs(&W[gid * 16 + lane16]);
        const bool finite = isfinite(v.x) && isfinite(v.y) && isfinite(v.z) && isfinite(v.w);
        float a = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
#pragma unroll
        for (int off = 8; off > 0; off >>= 1) a = fmaxf(a, __shfl_xor_sync(half_mask, a, off));
        const bool all_finite = __all_sync(half_mask, finite);

        const float s32 = __fdiv_rn(a, static_cast<float>(kQmax));
        const __half s16 = __float2half_rn(s32);
        uint16_t s_bits = __half_as_ushort(s16);
        const float sf = __half2float(s16);
        int status = 0;
        int c[4] = {0, 0, 0, 0};
        if (!all_finite) {
            s_bits = 0x7E00u;
            status = 5;  // RQ_ERR_NONFINITE
        } else if (s_bits == 0x7C00u) {
            status = 6;  // RQ_ERR_RANGE
        } else if (sf != 0.0f) {
            const float w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                int q = __float2int_rn(__fdiv_rn(w[i], sf));
                c[i] = max(-kQmax, min(kQmax, q));
            }
        }
        if (BITS == 4) {
            const uint16_t packed = static_cast<uint16_t>((c[0] & 0xF) | ((c[1] & 0xF) << 4) |
                                                          ((c[2] & 0xF) << 8) |
                                                          ((c[3] & 0xF) << 12));
            __stcs(reinterpret_cast<unsigned short*>(codes + gid * 32 + lane16 * 2), packed);
        } else {
            const uint32_t packed = (c[0] & 0xFF) | ((c[1] & 0xFF) << 8) | ((c[2] & 0xFF) << 16) |
                                    (static_cast<uint32_t>(c[3] & 0xFF) << 24);
            __stcs(reinterpret_cast<unsigned int*>(codes + gid * 64 + lane16 * 4), packed);
        }
        if (lane16 == 0) {
            scales[gid] = s_bits;
            // NONFINITE overrides everything; RANGE only replaces OK.
            if (dev_status != nullptr) {
                if (status == 5) atomicExch(dev_status, 5);
                else if (status == 6) atomicCAS(dev_status, 0, 6);
            }
        }
    }
}

cudaError_t launch_quantize(const float* W, int64_t n_groups, int bits, void* codes,
                            uint16_t* scales, int* dev_status, cudaStream_t s) {
    if (n_groups <= 0) return cudaSuccess;
    const int threads = 256;
    const int64_t groups_per_block = threads / 16;
    int64_t blocks = (n_groups + groups_per_block - 1) / groups_per_block;
    const int64_t cap = 148LL * 8 * 4;  // a few waves of fully resident blocks, then grid-stride
    if (blocks > cap) blocks = cap;
    if (bits == 4)
        quantize_g64_kernel<4><<<static_cast<unsigned>(blocks), threads, 0, s>>>(
            reinterpret_cast<const float4*>(W), n_groups, static_cast<uint8_t*>(codes), scales,
            dev_status);
    else
        quantize_g64_kernel<8><<<static_cast<unsigned>(blocks), threads, 0, s>>>(
            reinterpret_cast<const float4*>(W), n_groups, static_cast<uint8_t*>(codes), scales,
            dev_status);
    return cudaGetLastError();
}

}  // namespace rq
