// rq_gemv.cu -- decode product (1 <= M <= 32) on group-64 quantized weights.
//
//   y[m, n] = sum_g s16[n, g] * sum_{k in g} x[m, k] * code[n, k]
//
// The "Hakureirm/rwkv7-sglang-w4gptq-1.5b" model card credits its decode
// speed-up to a hand-written int4 GEMV / small-M kernel family streaming the
// g64 codes; the "RWKV-7 Quantization Toolkit" (rwkv-quant-nv 1.2.1) "Key
// Design" keeps weights quantized on the path and fuses R/K/V into one
// launch.  This kernel is the B200 form of that decode path.
//
// Why warp-level MMA here and not tcgen05: at decode sizes the MMA's N is the
// batch (1..32).  On B200 a tcgen05.mma with M = 128, K = 16 and N <= 64 costs
// a fixed ~47 cycles (2048 weights per instruction per SM), which caps a
// streaming int4 kernel near the HBM rate with no slack, while
// mma.sync.m16n8k16 runs at 1024 MAC/cycle/SM with an 8-token granularity:
// 128 / 64 / 32 weights per cycle per SM for M <= 8 / 16 / 32.  (Both figures
// measured on this hardware.)
//
// Data path (one CTA = 8 consumer warps + 1 TMA producer warp):
//   codes   TMA 2D tiles [ROWS rows x 128 B] (int4: 256 k, int8: 128 k per
//           stage), SWIZZLE_128B, into an SS-deep shared-memory ring;
//   x       TMA 2D tiles [8*NT tokens x 64 k] per group, SWIZZLE_128B, in the
//           same stage (rows >= M are zero-filled by the TMA);
//   scales  per thread with 8-byte loads, one stage ahead.
// A consumer warp owns 16*MT weight rows.  Thread (g = lane/4, t = lane%4)
// owns, per group of 64 k, the 16 k [16t, 16t+16) of rows g and g+8 of each
// of its m-tiles: MMA k-slot sigma of step j maps to one of those k, the same
// map on the A (weights) and B (x) side, so the sum over k is unchanged and
// every thread's codes and x are contiguous in memory.  Codes enter the MMA
// as exact biased fp16 values (code + bias placed in the mantissa of an fp16
// in [1024, 2048): Kim et al., arXiv:2211.10017); each group's fp32
// accumulation is seeded with -bias * sum_k x (an MMA against a constant
// operand), so the MMA yields sum_k x * code for the group; the group's scale
// is applied in fp32 (acc = fma(partial, s, acc)).  Nothing dequantised is
// stored.
//
// Split-K: CTAs of one cluster share a row tile and take disjoint k-stage
// ranges; partials are summed in a fixed order through distributed shared
// memory (deterministic, no atomics, no global workspace).
#include "rq_internal.h"
#include "rq_ptx.cuh"

namespace rq {

struct GvParams {
    CUtensorMap tm_x;     // x [M, K] fp16: dims {K, M}, box {64, 8*NT}, SWIZZLE_128B
    CUtensorMap tm_w[3];  // codes [N, K*bits/8] u8: box {128, ROWS}, SWIZZLE_128B
    const uint16_t* scales[3];
    float* y[3];
    int M, N, K;
    int n_tiles;          // row tiles per matrix
    int kstages;          // k stages per row (ceil(K / k-per-stage))
    int groups;           // K / 64
    int* status;
    uint64_t timeout_ns;
};

constexpr int kGvConsumers = 8;
constexpr int kGvThreads = (kGvConsumers + 1) * 32;

// BITS: 4 or 8.  NT: 8-token n-tiles (M <= 8 NT).  MT: 16-row m-tiles per
// consumer warp.  SSC: scales staged in shared memory by the producer warp (needs the
// stage's groups to be all valid or all past the end: G % groups-per-stage
// == 0); otherwise consumers load them from global memory.
template <int BITS, int NT, int MT, bool SSC>
struct GvCfg {
    static constexpr int kRows = kGvConsumers * 16 * MT;      // weight rows per CTA
    static constexpr int kKPS = BITS == 4 ? 256 : 128;        // k per stage (128 code bytes)
    static constexpr int kGPS = kKPS / 64;                    // groups per stage
    static constexpr int kTok = 8 * NT;                       // tokens per CTA
    static constexpr int kWStage = kRows * 128;
    static constexpr int kXStage = kGPS * kTok * 128;
    static constexpr int kSStage = SSC ? ((kRows * kGPS * 2 + 1023) / 1024) * 1024 : 0;
    static constexpr int kStage = kWStage + kXStage + kSStage;
    static constexpr int kBudget = (NT == 1 && MT == 1 ? 100 : 196) * 1024;   // two CTAs per SM when NT == MT == 1
    static constexpr int kSS = kBudget / kStage > 8 ? 8 : (kBudget / kStage < 2 ? 2 : kBudget / kStage);
    static constexpr int kRing = kSS * kStage;
    static constexpr int kRed = kTok * kRows * 4;
    static constexpr int kData = kRing > kRed ? kRing : kRed;
    static constexpr int kSmem = 1024 + kData + 256;
    static_assert(kWStage % 1024 == 0 && kXStage % 1024 == 0 && kSStage % 1024 == 0,
                  "stage alignment");
};

__device__ __forceinline__ uint32_t lop3_bmux(uint32_t a, uint32_t b, uint32_t c) {
    // b ? (a ^ c) : c, bitwise
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0x6a;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

__device__ __forceinline__ uint32_t h2_as_u32(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 u32_as_h2(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

// Code unpacking.  Each fp16 pair holds BIASED codes: the code plus a bias
// placed in the mantissa of an fp16 in [1024, 2048), exact, with no
// arithmetic (the bit placement of Kim et al., arXiv:2211.10017).  The bias is
// removed inside the MMA: every group's accumulation starts from
// -bias * sum_k x[k], itself computed by an MMA with a constant A operand.
//   int4: 1024 + (nibble ^ 8) = code + 1032
//   int8: 1024 + (byte ^ 0x80) = code + 1152
constexpr uint32_t kBiasI4 = 0xE408E408u;   // fp16 pair (-1032, -1032)
constexpr uint32_t kBiasI8 = 0xE480E480u;   // fp16 pair (-1152, -1152)

// int4: one 32-bit code word (positions 0..7 of one row, position 2i in the
// low nibble of byte i) -> pairs (p0,p1), (p2,p3), (p4,p5), (p6,p7).
// 9 instructions per 8 codes.
__device__ __forceinline__ void i4_word_to_pairs(uint32_t w, uint32_t (&P)[4]) {
    const uint32_t w4 = w >> 4;   // byte b of w4 holds the high nibble of byte b of w in its low bits
#pragma unroll
    for (int b = 0; b < 4; ++b) {
        const uint32_t v = __byte_perm(w, w4, static_cast<uint32_t>(b) | ((4u + b) << 8));
        P[b] = lop3_bmux(v, 0x000F000Fu, 0x64086408u);   // (nibble ^ 8) under exponent 0x64
    }
}

// int8: one 32-bit word (positions 0..3) -> pairs (p0, p1), (p2, p3).
// 3 instructions per 4 codes.
__device__ __forceinline__ void i8_word_to_pairs(uint32_t w, uint32_t (&Q)[2]) {
    w ^= 0x80808080u;
    Q[0] = __byte_perm(w, 0x64646464u, 0x5140u);
    Q[1] = __byte_perm(w, 0x64646464u, 0x5342u);
}

// Not volatile: a pure function of its operands, so the compiler may
// interleave independent accumulation chains (different groups / n-tiles).
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1, bool zero_c) {
    if (zero_c) {
        asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
            "{%8,%9}, {%10,%10,%10,%10};"
            : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.0f));
    } else {
        asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
            "{%8,%9}, {%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    }
}

// Physical row (within a 16-row m-tile) of MMA row g (0..7); MMA row g + 8 is
// that plus 8.  Chosen so that the rows read together by one shared-memory
// wavefront land on distinct 16-byte chunks of the 128-byte swizzle:
// int4 (8-byte reads, half-warps = g 0..3 / 4..7): rows 0,2,4,6 / 1,3,5,7;
// int8 (16-byte reads, quarter-warps = g pairs): rows 0,4 / 1,5 / 2,6 / 3,7.
template <int BITS>
__device__ __forceinline__ int phys_row(int g) {
    if constexpr (BITS == 4) return g < 4 ? 2 * g : 2 * (g - 4) + 1;
    else return (g >> 1) + 4 * (g & 1);
}

template <int BITS, int NT, int MT, bool SSC>
__global__ void __launch_bounds__(kGvThreads, (NT == 1 && MT == 1) ? 2 : 1)
    gemv_wq_kernel(const __grid_constant__ GvParams p) {
    using Cfg = GvCfg<BITS, NT, MT, SSC>;
    constexpr int SS = Cfg::kSS;
    constexpr int ROWS = Cfg::kRows;
    constexpr int GPS = Cfg::kGPS;
    constexpr int TOK = Cfg::kTok;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint8_t* ring = smem;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + Cfg::kData);
    uint64_t* empty = full + SS;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + SS);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int ksplit = gridDim.x;
    const int kq = blockIdx.x;
    const int mat = blockIdx.y / p.n_tiles;
    const int n0 = (blockIdx.y - mat * p.n_tiles) * ROWS;
    const int st0 = static_cast<int>((static_cast<int64_t>(kq) * p.kstages) / ksplit);
    const int st1 = static_cast<int>((static_cast<int64_t>(kq + 1) * p.kstages) / ksplit);
    const int nst = st1 - st0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < SS; ++s) {
            mbar_init(&full[s], SSC ? 1 + 32 : 1);
            mbar_init(&empty[s], kGvConsumers);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kGvConsumers && lane == 0) {
        tma_prefetch_desc(&p.tm_x);
        tma_prefetch_desc(&p.tm_w[mat]);
    }
    __syncthreads();
    pdl_launch_dependents();

    if (warp == kGvConsumers) {
        // ---------------------------------------------- producer warp --
        // lane 0 issues the TMA copies; with SSC every lane also copies the
        // stage's scales (rows lane, lane+32, ...) with cp.async completing
        // on the same barrier.
        const bool leader = lane == 0;
        const uint64_t pol_w = l2_policy_evict_first();
        const uint64_t pol_x = l2_policy_evict_last();
        const CUtensorMap* tmw = &p.tm_w[mat];
        const uint16_t* sbase = p.scales[mat];
        auto stage_scales = [&](int i, int s) {
            if constexpr (SSC) {
                uint8_t* dst = ring + s * Cfg::kStage + Cfg::kWStage + Cfg::kXStage;
                const int grp = (st0 + i) * GPS;
#pragma unroll
                for (int rr = lane; rr < ROWS; rr += 32) {
                    const int n = n0 + rr;
                    const bool ok = n < p.N && grp < p.groups;
                    const uint16_t* src = ok ? sbase + static_cast<int64_t>(n) * p.groups + grp : sbase;
                    if constexpr (GPS == 4) cp_async_8(dst + rr * 8, src, ok ? 8u : 0u);
                    else cp_async_4(dst + rr * 4, src, ok ? 4u : 0u);
                }
                cp_async_arrive_noinc(&full[s]);
            }
        };
        const int pre = nst < SS ? nst : SS;
        for (int i = 0; i < pre; ++i) {
            if (leader) {
                mbar_arrive_expect_tx(&full[i], Cfg::kWStage + Cfg::kXStage);
                tma_load_2d(ring + i * Cfg::kStage, tmw, &full[i], (st0 + i) * 128, n0, pol_w);
            }
            stage_scales(i, i);
        }
        if (leader) {
            pdl_wait();   // x may be produced by the previous kernel
            for (int i = 0; i < pre; ++i)
#pragma unroll
                for (int q = 0; q < GPS; ++q)
                    tma_load_2d(ring + i * Cfg::kStage + Cfg::kWStage + q * TOK * 128, &p.tm_x,
                                &full[i], (st0 + i) * Cfg::kKPS + q * 64, 0, pol_x);
        }
        int issued = pre;
        for (int i = SS; i < nst; ++i) {
            const int s = i % SS;
            if (!mbar_wait(&empty[s], static_cast<uint32_t>(i / SS - 1) & 1, abort_flag,
                           p.timeout_ns, p.status))
                break;
            if (leader) {
                mbar_arrive_expect_tx(&full[s], Cfg::kWStage + Cfg::kXStage);
                tma_load_2d(ring + s * Cfg::kStage, tmw, &full[s], (st0 + i) * 128, n0, pol_w);
#pragma unroll
                for (int q = 0; q < GPS; ++q)
                    tma_load_2d(ring + s * Cfg::kStage + Cfg::kWStage + q * TOK * 128, &p.tm_x,
                                &full[s], (st0 + i) * Cfg::kKPS + q * 64, 0, pol_x);
            }
            stage_scales(i, s);
            issued = i + 1;
        }
        // Wait (bounded, regardless of abort) until every copy this warp
        // issued has landed, so none is in flight when the CTA exits.
        int dummy_abort = 0;
        const int first = issued > SS ? issued - SS : 0;
        for (int i = first; i < issued; ++i)
            mbar_wait(&full[i % SS], static_cast<uint32_t>(i / SS) & 1, &dummy_abort,
                      p.timeout_ns, p.status);
        __syncwarp();
    }

    float acc[MT][NT][4];
#pragma unroll
    for (int i = 0; i < MT; ++i)
#pragma unroll
        for (int j = 0; j < NT; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[i][j][e] = 0.0f;

    const int g = lane >> 2;
    const int t = lane & 3;
    const int rbase = warp * 16 * MT;           // this warp's first row in the tile
    if (warp < kGvConsumers) {
        // ---------------------------------------------------- consumers --
        int rloc[MT][2];                        // physical rows (within the tile)
#pragma unroll
        for (int i = 0; i < MT; ++i)
#pragma unroll
            for (int h = 0; h < 2; ++h) rloc[i][h] = rbase + 16 * i + phys_row<BITS>(g) + 8 * h;
        // global scale pointers, only for the path without shared-memory scales
        const uint16_t* srow[MT][2];
        bool rok[MT][2];
#pragma unroll
        for (int i = 0; i < MT; ++i)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int n = n0 + rloc[i][h];
                rok[i][h] = n < p.N;
                srow[i][h] = p.scales[mat] + static_cast<int64_t>(rok[i][h] ? n : 0) * p.groups;
            }

        for (int i = 0; i < nst; ++i) {
            const int s = i % SS;
            if (!mbar_wait(&full[s], static_cast<uint32_t>(i / SS) & 1, abort_flag, p.timeout_ns,
                           p.status))
                break;
            const uint8_t* wt = ring + s * Cfg::kStage;
            const uint8_t* xt = wt + Cfg::kWStage;
            // scales of this stage for the thread's rows: [m-tile][half][group]
            float sv[MT][2][GPS];
#pragma unroll
            for (int a = 0; a < MT; ++a)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    if constexpr (SSC) {
                        const uint8_t* sp = xt + Cfg::kXStage + rloc[a][h] * GPS * 2;
                        if constexpr (GPS == 4) {
                            const uint2 u = *reinterpret_cast<const uint2*>(sp);
                            const float2 f0 = __half22float2(u32_as_h2(u.x));
                            const float2 f1 = __half22float2(u32_as_h2(u.y));
                            sv[a][h][0] = f0.x; sv[a][h][1] = f0.y;
                            sv[a][h][2] = f1.x; sv[a][h][3] = f1.y;
                        } else {
                            const float2 f0 = __half22float2(u32_as_h2(*reinterpret_cast<const uint32_t*>(sp)));
                            sv[a][h][0] = f0.x; sv[a][h][1] = f0.y;
                        }
                    } else {
#pragma unroll
                        for (int q = 0; q < GPS; ++q) {
                            const int grp = (st0 + i) * GPS + q;
                            sv[a][h][q] = (rok[a][h] && grp < p.groups)
                                              ? __half2float(__ushort_as_half(__ldg(srow[a][h] + grp)))
                                              : 0.0f;
                        }
                    }
                }
#pragma unroll
            for (int q = 0; q < GPS; ++q) {
                // ---- x fragments of this group: B registers per n-tile and step
                // (thread (g, t): token g of the n-tile, positions 16t .. 16t+15
                // of the group; step j covers positions 4j .. 4j+3)
                uint32_t b[NT][4][2];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const int tok = nt * 8 + g;
                    const uint8_t* xrow = xt + q * TOK * 128 + tok * 128;
                    const int sw = tok & 7;
                    const uint4 x0 = *reinterpret_cast<const uint4*>(xrow + (((2 * t) ^ sw) << 4));
                    const uint4 x1 = *reinterpret_cast<const uint4*>(xrow + (((2 * t + 1) ^ sw) << 4));
                    b[nt][0][0] = x0.x; b[nt][0][1] = x0.y;
                    b[nt][1][0] = x0.z; b[nt][1][1] = x0.w;
                    b[nt][2][0] = x1.x; b[nt][2][1] = x1.y;
                    b[nt][3][0] = x1.z; b[nt][3][1] = x1.w;
                }
                // ---- bias term of the group: -bias * sum_k x[tok, k], the same
                // for every row; it seeds each m-tile's accumulation
                float corr[NT][4];
                {
                    const uint32_t cb = BITS == 4 ? kBiasI4 : kBiasI8;
                    const uint32_t Ac[4] = {cb, cb, cb, cb};
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            mma16816(corr[nt], Ac, b[nt][j][0], b[nt][j][1], j == 0);
                }
                // ---- per m-tile: codes -> A registers, 4 MMA steps, scale
#pragma unroll
                for (int mi = 0; mi < MT; ++mi) {
                    uint32_t A[4][4];   // [step][a-reg]
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int r = rloc[mi][h];
                        const uint8_t* crow = wt + r * 128;
                        const int sw = r & 7;
                        if constexpr (BITS == 4) {
                            // bytes [32q + 8t, +8): chunk 2q + t/2, offset (t&1)*8
                            const uint2 cw = *reinterpret_cast<const uint2*>(
                                crow + (((2 * q + (t >> 1)) ^ sw) << 4) + ((t & 1) << 3));
                            uint32_t P0[4], P1[4];
                            i4_word_to_pairs(cw.x, P0);
                            i4_word_to_pairs(cw.y, P1);
                            // step j: a0a1 (h = 0) / a2a3 (h = 1) = positions 4j, 4j+1;
                            //         a4a5 / a6a7 = positions 4j+2, 4j+3
                            A[0][h] = P0[0]; A[0][h + 2] = P0[1];
                            A[1][h] = P0[2]; A[1][h + 2] = P0[3];
                            A[2][h] = P1[0]; A[2][h + 2] = P1[1];
                            A[3][h] = P1[2]; A[3][h + 2] = P1[3];
                        } else {
                            // bytes [64q + 16t, +16): chunk 4q + t
                            const uint4 cw = *reinterpret_cast<const uint4*>(
                                crow + (((4 * q + t) ^ sw) << 4));
                            const uint32_t wv[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                uint32_t Q[2];
                                i8_word_to_pairs(wv[j], Q);
                                A[j][h] = Q[0];
                                A[j][h + 2] = Q[1];
                            }
                        }
                    }
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        // the bias chain runs beside this one (no dependency); it is
                        // added to the group's partial before scaling
                        float part[4];
#pragma unroll
                        for (int j = 0; j < 4; ++j) mma16816(part, A[j], b[nt][j][0], b[nt][j][1], j == 0);
                        acc[mi][nt][0] = fmaf(part[0] + corr[nt][0], sv[mi][0][q], acc[mi][nt][0]);
                        acc[mi][nt][1] = fmaf(part[1] + corr[nt][1], sv[mi][0][q], acc[mi][nt][1]);
                        acc[mi][nt][2] = fmaf(part[2] + corr[nt][2], sv[mi][1][q], acc[mi][nt][2]);
                        acc[mi][nt][3] = fmaf(part[3] + corr[nt][3], sv[mi][1][q], acc[mi][nt][3]);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
        }
    }

    __syncthreads();   // every stage consumed: the ring is free for the partials

    float* y = p.y[mat];
    if (warp < kGvConsumers && !*abort_flag) {
        float* red = reinterpret_cast<float*>(ring);
#pragma unroll
        for (int mi = 0; mi < MT; ++mi)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int r = rbase + 16 * mi + phys_row<BITS>(g) + ((e >> 1) << 3);
                    const int tok = nt * 8 + 2 * t + (e & 1);
                    if (ksplit == 1) {
                        const int n = n0 + r;
                        if (n < p.N && tok < p.M) y[static_cast<int64_t>(tok) * p.N + n] = acc[mi][nt][e];
                    } else {
                        red[tok * ROWS + r] = acc[mi][nt][e];
                    }
                }
    }

    if (ksplit > 1) {
        __syncthreads();
        cluster_sync();
        if (!*abort_flag) {
            constexpr int E4 = TOK * ROWS / 4;
            const int e0 = static_cast<int>((static_cast<int64_t>(kq) * E4) / ksplit);
            const int e1 = static_cast<int>((static_cast<int64_t>(kq + 1) * E4) / ksplit);
            const uint32_t red_local = smem_u32(ring);
            for (int e = e0 + static_cast<int>(threadIdx.x); e < e1; e += kGvThreads) {
                float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
                for (int src = 0; src < ksplit; ++src) {
                    const float4 v = ld_dsmem_f32x4(map_to_rank(red_local + e * 16, src));
                    sum.x += v.x; sum.y += v.y; sum.z += v.z; sum.w += v.w;
                }
                const int tok = (e * 4) / ROWS;
                const int r = (e * 4) % ROWS;
                if (tok < p.M) {
                    const float out[4] = {sum.x, sum.y, sum.z, sum.w};
                    float* yrow = y + static_cast<int64_t>(tok) * p.N;
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        if (n0 + r + u < p.N) yrow[n0 + r + u] = out[u];
                }
            }
        }
        cluster_sync();
    }
}

// ------------------------------------------------------------- launcher --

static int gv_num_sms() {
    static int sms = 0;
    if (sms == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (sms <= 0) sms = 148;
    }
    return sms;
}

template <int BITS, int NT, int MT, bool SSC>
static cudaError_t gv_launch(GvParams& prm, const void* x, const void* const* codes, int nmat,
                             cudaStream_t s) {
    using Cfg = GvCfg<BITS, NT, MT, SSC>;
    auto kern = gemv_wq_kernel<BITS, NT, MT, SSC>;
    static int resident[64] = {};   // CTAs per SM, per device (0 = not yet set up)
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (resident[dev] == 0) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmem);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
        int occ = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kGvThreads, Cfg::kSmem);
        if (e != cudaSuccess) return e;
        resident[dev] = occ > 0 ? occ : 1;
    }
    prm.n_tiles = (prm.N + Cfg::kRows - 1) / Cfg::kRows;
    prm.kstages = (prm.K + Cfg::kKPS - 1) / Cfg::kKPS;
    const int64_t tiles = static_cast<int64_t>(nmat) * prm.n_tiles;
    const int64_t slots = static_cast<int64_t>(resident[dev]) * gv_num_sms();
    int ks = 1;
    while (ks < 8 && tiles * (ks + 1) <= slots && prm.kstages / (ks + 1) >= 2) ++ks;

    // codes tensor maps (box rows = ROWS) and x map (box rows = 8*NT)
    const uint64_t row_bytes = static_cast<uint64_t>(prm.K) * BITS / 8;
    for (int i = 0; i < nmat; ++i) {
        if (!make_tmap_2d(&prm.tm_w[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, codes[i], row_bytes,
                          static_cast<uint64_t>(prm.N), row_bytes, 128, Cfg::kRows,
                          CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
    }
    if (!make_tmap_2d(&prm.tm_x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, x,
                      static_cast<uint64_t>(prm.K), static_cast<uint64_t>(prm.M),
                      static_cast<uint64_t>(prm.K) * 2, 64, Cfg::kTok, CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(ks), static_cast<unsigned>(tiles), 1);
    cfg.blockDim = dim3(kGvThreads, 1, 1);
    cfg.dynamicSmemBytes = static_cast<size_t>(Cfg::kSmem);
    cfg.stream = s;
    cudaLaunchAttribute attrs[2];
    int na = 0;
    attrs[na].id = cudaLaunchAttributeClusterDimension;
    attrs[na].val.clusterDim.x = static_cast<unsigned>(ks);
    attrs[na].val.clusterDim.y = 1;
    attrs[na].val.clusterDim.z = 1;
    ++na;
    if (pdl_enabled()) {
        attrs[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attrs[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    cfg.attrs = attrs;
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<const GvParams&>(prm));
}

template <int BITS, bool SSC>
static cudaError_t gv_dispatch_ssc(GvParams& prm, const void* x, const void* const* codes, int nmat,
                                   cudaStream_t s) {
    // 8 tokens per n-tile; two m-tiles per warp (x fragments and the bias
    // term reused twice) when N leaves enough row tiles for the SMs.
    const bool wide = static_cast<int64_t>(nmat) * prm.N >= 8192;
    if (prm.M <= 8) {
        if (wide) return gv_launch<BITS, 1, 2, SSC>(prm, x, codes, nmat, s);
        return gv_launch<BITS, 1, 1, SSC>(prm, x, codes, nmat, s);
    }
    if (prm.M <= 16) {
        if (wide) return gv_launch<BITS, 2, 2, SSC>(prm, x, codes, nmat, s);
        return gv_launch<BITS, 2, 1, SSC>(prm, x, codes, nmat, s);
    }
    if (prm.M <= 24) {
        if (wide) return gv_launch<BITS, 3, 2, SSC>(prm, x, codes, nmat, s);
        return gv_launch<BITS, 3, 1, SSC>(prm, x, codes, nmat, s);
    }
    if (wide) return gv_launch<BITS, 4, 2, SSC>(prm, x, codes, nmat, s);
    return gv_launch<BITS, 4, 1, SSC>(prm, x, codes, nmat, s);
}

template <int BITS>
static cudaError_t gv_dispatch(GvParams& prm, const void* x, const void* const* codes, int nmat,
                               cudaStream_t s) {
    constexpr int gps = BITS == 4 ? 4 : 2;
    if (prm.groups % gps == 0) return gv_dispatch_ssc<BITS, true>(prm, x, codes, nmat, s);
    return gv_dispatch_ssc<BITS, false>(prm, x, codes, nmat, s);
}

cudaError_t launch_gemv_product(const uint16_t* x, int64_t M, int64_t K, int64_t N, int bits,
                                const WOperand* w, int nmat, cudaStream_t s) {
    GvParams prm;
    memset(&prm, 0, sizeof(prm));
    prm.M = static_cast<int>(M);
    prm.N = static_cast<int>(N);
    prm.K = static_cast<int>(K);
    prm.groups = static_cast<int>(K / kGroup);
    prm.status = device_status_ptr();
    prm.timeout_ns = wait_limit_ns();
    const void* codes[3] = {nullptr, nullptr, nullptr};
    for (int i = 0; i < nmat; ++i) {
        codes[i] = w[i].codes;
        prm.scales[i] = w[i].scales;
        prm.y[i] = w[i].y;
    }
    return bits == 4 ? gv_dispatch<4>(prm, x, codes, nmat, s) : gv_dispatch<8>(prm, x, codes, nmat, s);
}

}  // namespace rq
