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
// every thread's codes and x are contiguous in memory.  Codes become exact
// fp16 values in registers (bit placement plus one exact fp16 operation:
// Kim et al., arXiv:2211.10017); the MMA sums x * code for one group in fp32
// registers; the group's scale is applied in fp32 (acc = fma(partial, s,
// acc)).  Nothing dequantised is stored.
//
// Work split (stream-K): the work is a list of units (one 128-row tile x one
// k-stage, tile-major) cut into equal contiguous runs, one per resident CTA,
// so every SM streams the same number of bytes whatever the shape.  A CTA
// stores a tile it covers whole directly; a tile shared by several CTAs is
// stored as pieces in a global workspace and summed, in a fixed CTA order, by
// whichever contributor arrives last (an atomic counter per tile), so results
// are deterministic.
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
    int kstages;          // k stages per row tile (ceil(K / k-per-stage))
    int groups;           // K / 64
    int units;            // work units: nmat * n_tiles * kstages (one tile x one stage each)
    int uq, ur;           // units / gridDim.x and units % gridDim.x: CTA c owns
                          // [c*uq + min(c, ur), (c+1)*uq + min(c+1, ur))
    float* ws;            // partial-tile slots: [2 * gridDim.x][8*NT tokens * ROWS rows] fp32
    int* cnt;             // per-tile arrival counters, zero between launches
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

// Code unpacking to EXACT fp16 codes, without integer->float conversions:
// the biased code is placed in the mantissa of an fp16 in [1024, 2048) and
// the bias is removed with one exact fp16 operation (the bit placement of
// Kim et al., "Who Says Elephants Can't Run?", arXiv:2211.10017).

// int4, permuted order: one code word (positions 0..7 of a row, position 2i
// in the low nibble of byte i) -> pairs (p0,p4), (p1,p5), (p2,p6), (p3,p7).
// 9 instructions per 8 codes; x is permuted to the same order.
__device__ __forceinline__ void i4_word_to_pairs_perm(uint32_t w, uint32_t (&P)[4]) {
    const __half2 bias_lo = u32_as_h2(0x64086408u);                      // 1032, 1032
    const __half2 inv16 = u32_as_h2(0x2C002C00u);                        // 1/16
    const __half2 bias_hi = u32_as_h2(0xD480D480u);                      // -72
    const uint32_t w8 = w >> 8;
    // low nibbles of bytes 0 and 2 -> 1024 + (nibble ^ 8); high nibbles -> 1024 + 16*(nibble ^ 8)
    P[0] = h2_as_u32(__hsub2(u32_as_h2(lop3_bmux(w, 0x000F000Fu, 0x64086408u)), bias_lo));
    P[1] = h2_as_u32(__hfma2(u32_as_h2(lop3_bmux(w, 0x00F000F0u, 0x64806480u)), inv16, bias_hi));
    P[2] = h2_as_u32(__hsub2(u32_as_h2(lop3_bmux(w8, 0x000F000Fu, 0x64086408u)), bias_lo));
    P[3] = h2_as_u32(__hfma2(u32_as_h2(lop3_bmux(w8, 0x00F000F0u, 0x64806480u)), inv16, bias_hi));
}

// int4, natural order: one code word -> pairs (p0,p1), (p2,p3), (p4,p5), (p6,p7)
// (the two nibbles of each byte).  13 instructions per 8 codes; x is used as is.
__device__ __forceinline__ void i4_word_to_pairs_nat(uint32_t w, uint32_t (&P)[4]) {
    const __half2 bias = u32_as_h2(0x64086408u);                         // 1032, 1032
    const uint32_t w4 = w >> 4;   // byte b of w4 holds the high nibble of byte b of w in its low bits
#pragma unroll
    for (int b = 0; b < 4; ++b) {
        const uint32_t v = __byte_perm(w, w4, static_cast<uint32_t>(b) | ((4u + b) << 8));
        P[b] = h2_as_u32(__hsub2(u32_as_h2(lop3_bmux(v, 0x000F000Fu, 0x64086408u)), bias));
    }
}

// int8: one 32-bit word (positions 0..3) -> exact pairs (p0, p1), (p2, p3).
__device__ __forceinline__ void i8_word_to_pairs(uint32_t w, uint32_t (&Q)[2]) {
    const __half2 bias = u32_as_h2(0x64806480u);                         // 1152 = 1024 + 128
    w ^= 0x80808080u;
    Q[0] = h2_as_u32(__hsub2(u32_as_h2(__byte_perm(w, 0x64646464u, 0x5140u)), bias));
    Q[1] = h2_as_u32(__hsub2(u32_as_h2(__byte_perm(w, 0x64646464u, 0x5342u)), bias));
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

// First work unit of CTA c: the first ur CTAs take uq + 1 units, the rest uq.
__device__ __forceinline__ int range_begin(int c, int uq, int ur) {
    return c * uq + (c < ur ? c : ur);
}

// The CTA whose unit range holds unit u.
__device__ __forceinline__ int range_owner(int u, int uq, int ur) {
    const int big = ur * (uq + 1);
    return u < big ? u / (uq + 1) : ur + (u - big) / uq;
}

// Named barrier over the eight consumer warps (the producer warp is not in it).
__device__ __forceinline__ void consumers_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(kGvConsumers * 32) : "memory");
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
    volatile int* last_flag = abort_flag + 1;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int G = static_cast<int>(gridDim.x);
    const int cta = static_cast<int>(blockIdx.x);
    const int S = p.kstages;
    const int u0 = range_begin(cta, p.uq, p.ur);
    const int nu = p.uq + (cta < p.ur ? 1 : 0);
    // position of the first unit: tile (matrix, row tile) and k-stage
    const int tile0 = u0 / S;
    const int st0 = u0 - tile0 * S;

    if (threadIdx.x == 0) {
        for (int s = 0; s < SS; ++s) {
            mbar_init(&full[s], SSC ? 1 + 32 : 1);
            mbar_init(&empty[s], kGvConsumers);
        }
        *abort_flag = 0;
        *last_flag = 0;
        fence_mbar_init();
    }
    if (warp == kGvConsumers && lane == 0) {
        tma_prefetch_desc(&p.tm_x);
        for (int m = 0; m < 3; ++m)
            if (p.y[m] != nullptr) tma_prefetch_desc(&p.tm_w[m]);
    }
    __syncthreads();
    pdl_launch_dependents();

    if (warp == kGvConsumers) {
        // ---------------------------------------------- producer warp --
        // lane 0 issues the TMA copies; with SSC every lane also copies the
        // unit's scales (rows lane, lane+32, ...) with cp.async completing on
        // the same barrier.
        const bool leader = lane == 0;
        const uint64_t pol_w = l2_policy_evict_first();
        const uint64_t pol_x = l2_policy_evict_last();
        // position of the next unit to issue, advanced one unit at a time
        int c_st = st0, c_tm = tile0 % p.n_tiles, c_mat = tile0 / p.n_tiles;
        auto unit_codes = [&](int s) {
            const int st = c_st;
            const int mat = c_mat;
            const int n0 = c_tm * ROWS;
            if (leader) {
                mbar_arrive_expect_tx(&full[s], Cfg::kWStage + Cfg::kXStage);
                tma_load_2d(ring + s * Cfg::kStage, &p.tm_w[mat], &full[s], st * 128, n0, pol_w);
            }
            if constexpr (SSC) {
                uint8_t* dst = ring + s * Cfg::kStage + Cfg::kWStage + Cfg::kXStage;
                const int grp = st * GPS;
                const uint16_t* sbase = p.scales[mat];
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
        auto advance = [&]() {
            if (++c_st == S) {
                c_st = 0;
                if (++c_tm == p.n_tiles) {
                    c_tm = 0;
                    ++c_mat;
                }
            }
        };
        auto unit_x = [&](int st, int s) {
#pragma unroll
            for (int q = 0; q < GPS; ++q)
                tma_load_2d(ring + s * Cfg::kStage + Cfg::kWStage + q * TOK * 128, &p.tm_x,
                            &full[s], st * Cfg::kKPS + q * 64, 0, pol_x);
        };
        const int pre = nu < SS ? nu : SS;
        // Weights do not depend on the previous kernel: fetch them first.
        for (int i = 0; i < pre; ++i) {
            unit_codes(i);
            advance();
        }
        if (leader) {
            pdl_wait();   // x may be produced by the previous kernel
            int st = st0;
            for (int i = 0; i < pre; ++i) {
                unit_x(st, i);
                if (++st == S) st = 0;
            }
        }
        int issued = pre;
        for (int i = SS; i < nu; ++i) {
            const int s = i % SS;
            if (!mbar_wait(&empty[s], static_cast<uint32_t>(i / SS - 1) & 1, abort_flag,
                           p.timeout_ns, p.status))
                break;
            const int st = c_st;
            unit_codes(s);
            if (leader) unit_x(st, s);
            advance();
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
    } else {
        // ---------------------------------------------------- consumers --
        const int g = lane >> 2;
        const int t = lane & 3;
        const int rbase = warp * 16 * MT;       // this warp's first row in a tile
        int rloc[MT][2];                        // physical rows (within the tile)
#pragma unroll
        for (int i = 0; i < MT; ++i)
#pragma unroll
            for (int h = 0; h < 2; ++h) rloc[i][h] = rbase + 16 * i + phys_row<BITS>(g) + 8 * h;

        float acc[MT][NT][4];
        int seg_first_i = 0;                    // unit index where the current segment began
        // After a timeout a warp keeps walking the units without working, so
        // every consumer warp reaches the same named barriers: none can wait
        // at one that another warp has left.
        bool dead = false;
        int st = st0, tile = tile0, tm = tile0 % p.n_tiles, mat = tile0 / p.n_tiles;
        for (int i = 0; i < nu; ++i) {
            if (i > 0 && ++st == S) {     // next unit: next stage, or next row tile
                st = 0;
                ++tile;
                if (++tm == p.n_tiles) {
                    tm = 0;
                    ++mat;
                }
            }
            const int n0 = tm * ROWS;
            if (i == 0 || st == 0) {
                seg_first_i = i;
#pragma unroll
                for (int a = 0; a < MT; ++a)
#pragma unroll
                    for (int j = 0; j < NT; ++j)
#pragma unroll
                        for (int e = 0; e < 4; ++e) acc[a][j][e] = 0.0f;
            }
            const int s = i % SS;
            if (!dead && !mbar_wait(&full[s], static_cast<uint32_t>(i / SS) & 1, abort_flag,
                                    p.timeout_ns, p.status))
                dead = true;
            if (!dead) {
            const uint8_t* wt = ring + s * Cfg::kStage;
            const uint8_t* xt = wt + Cfg::kWStage;
            // int4 with one n-tile uses the permuted pair order (cheapest
            // unpacking; x permuted once per group and n-tile)
            constexpr bool PERM = BITS == 4 && NT == 1;
            constexpr int CW = BITS == 4 ? 2 : 4;            // code words per row and group
            // ---- the unit's shared-memory operands, all loaded up front
            float sv[MT][2][GPS];                             // scales [m-tile][half][group]
            uint32_t cw[GPS][MT][2][CW];                      // code words
#pragma unroll
            for (int a = 0; a < MT; ++a)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int r = rloc[a][h];
                    const uint8_t* crow = wt + r * 128;
                    const int sw = r & 7;
#pragma unroll
                    for (int q = 0; q < GPS; ++q) {
                        if constexpr (BITS == 4) {
                            // bytes [32q + 8t, +8): chunk 2q + t/2, offset (t&1)*8
                            const uint2 v = *reinterpret_cast<const uint2*>(
                                crow + (((2 * q + (t >> 1)) ^ sw) << 4) + ((t & 1) << 3));
                            cw[q][a][h][0] = v.x;
                            cw[q][a][h][1] = v.y;
                        } else {
                            // bytes [64q + 16t, +16): chunk 4q + t
                            const uint4 v = *reinterpret_cast<const uint4*>(
                                crow + (((4 * q + t) ^ sw) << 4));
                            cw[q][a][h][0] = v.x; cw[q][a][h][1] = v.y;
                            cw[q][a][h][2] = v.z; cw[q][a][h][3] = v.w;
                        }
                    }
                    if constexpr (SSC) {
                        const uint8_t* sp = xt + Cfg::kXStage + r * GPS * 2;
                        if constexpr (GPS == 4) {
                            const uint2 uu = *reinterpret_cast<const uint2*>(sp);
                            const float2 f0 = __half22float2(u32_as_h2(uu.x));
                            const float2 f1 = __half22float2(u32_as_h2(uu.y));
                            sv[a][h][0] = f0.x; sv[a][h][1] = f0.y;
                            sv[a][h][2] = f1.x; sv[a][h][3] = f1.y;
                        } else {
                            const float2 f0 = __half22float2(u32_as_h2(*reinterpret_cast<const uint32_t*>(sp)));
                            sv[a][h][0] = f0.x; sv[a][h][1] = f0.y;
                        }
                    } else {
                        const int n = n0 + r;
                        const uint16_t* srow = p.scales[mat] + static_cast<int64_t>(n < p.N ? n : 0) * p.groups;
#pragma unroll
                        for (int q = 0; q < GPS; ++q) {
                            const int grp = st * GPS + q;
                            sv[a][h][q] = (n < p.N && grp < p.groups)
                                              ? __half2float(__ushort_as_half(__ldg(srow + grp)))
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
                    const uint32_t X[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        if constexpr (PERM) {
                            // step j pairs (p0,p4),(p1,p5) or (p2,p6),(p3,p7) of word j/2
                            const int wb = (j >> 1) * 4 + (j & 1);
                            b[nt][j][0] = __byte_perm(X[wb], X[wb + 2], 0x5410);
                            b[nt][j][1] = __byte_perm(X[wb], X[wb + 2], 0x7632);
                        } else {
                            b[nt][j][0] = X[2 * j];
                            b[nt][j][1] = X[2 * j + 1];
                        }
                    }
                }
                // ---- per m-tile: exact fp16 codes -> A registers, 4 MMA steps,
                // the group's scale in fp32
#pragma unroll
                for (int mi = 0; mi < MT; ++mi) {
                    uint32_t A[4][4];   // [step][a-reg]
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        if constexpr (BITS == 4) {
                            uint32_t P0[4], P1[4];
                            if constexpr (PERM) {
                                i4_word_to_pairs_perm(cw[q][mi][h][0], P0);
                                i4_word_to_pairs_perm(cw[q][mi][h][1], P1);
                            } else {
                                i4_word_to_pairs_nat(cw[q][mi][h][0], P0);
                                i4_word_to_pairs_nat(cw[q][mi][h][1], P1);
                            }
                            // step j: a0a1 (h = 0) / a2a3 (h = 1), and a4a5 / a6a7
                            A[0][h] = P0[0]; A[0][h + 2] = P0[1];
                            A[1][h] = P0[2]; A[1][h + 2] = P0[3];
                            A[2][h] = P1[0]; A[2][h + 2] = P1[1];
                            A[3][h] = P1[2]; A[3][h + 2] = P1[3];
                        } else {
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                uint32_t Q[2];
                                i8_word_to_pairs(cw[q][mi][h][j], Q);
                                A[j][h] = Q[0];
                                A[j][h + 2] = Q[1];
                            }
                        }
                    }
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        float part[4];
#pragma unroll
                        for (int j = 0; j < 4; ++j) mma16816(part, A[j], b[nt][j][0], b[nt][j][1], j == 0);
                        acc[mi][nt][0] = fmaf(part[0], sv[mi][0][q], acc[mi][nt][0]);
                        acc[mi][nt][1] = fmaf(part[1], sv[mi][0][q], acc[mi][nt][1]);
                        acc[mi][nt][2] = fmaf(part[2], sv[mi][1][q], acc[mi][nt][2]);
                        acc[mi][nt][3] = fmaf(part[3], sv[mi][1][q], acc[mi][nt][3]);
                    }
                }
            }
            }   // !dead
            __syncwarp();
            if (lane == 0 && !dead) mbar_arrive(&empty[s]);

            // ---- end of a tile segment: store it, or combine partial tiles
            if (st == S - 1 || i == nu - 1) {
                float* y = p.y[mat];
                const bool whole = (i - seg_first_i) == st && st == S - 1;   // began at stage 0
                if (whole && !dead) {
#pragma unroll
                    for (int mi = 0; mi < MT; ++mi)
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int n = n0 + rloc[mi][e >> 1];
                                const int tok = nt * 8 + 2 * t + (e & 1);
                                if (n < p.N && tok < p.M)
                                    y[static_cast<int64_t>(tok) * p.N + n] = acc[mi][nt][e];
                            }
                } else if (!whole) {
                    // This CTA's piece of a tile that several CTAs share: slot 2c
                    // for the CTA's first segment, 2c+1 for its last one.
                    const int slot = 2 * cta + (seg_first_i == 0 ? 0 : 1);
                    float* wsl = p.ws + static_cast<int64_t>(slot) * (TOK * ROWS);
                    if (!dead)
#pragma unroll
                    for (int mi = 0; mi < MT; ++mi)
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                wsl[(nt * 8 + 2 * t + (e & 1)) * ROWS + rloc[mi][e >> 1]] = acc[mi][nt][e];
                    const int tb = tile * S;
                    const int c_first = range_owner(tb, p.uq, p.ur);
                    const int c_last = range_owner(tb + S - 1, p.uq, p.ur);
                    consumers_sync();
                    if (threadIdx.x == 0) {
                        if (*abort_flag) {
                            *last_flag = 0;
                        } else {
                            __threadfence();
                            const int arrived = atomicAdd(&p.cnt[tile], 1);
                            *last_flag = arrived == c_last - c_first;
                        }
                    }
                    consumers_sync();
                    if (*last_flag) {
                        // Last arrival: sum every contributor's piece in CTA
                        // order (deterministic) and write the tile.
                        __threadfence();
                        float sum[MT][NT][4];
#pragma unroll
                        for (int mi = 0; mi < MT; ++mi)
#pragma unroll
                            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                                for (int e = 0; e < 4; ++e) sum[mi][nt][e] = 0.0f;
                        for (int c = c_first; c <= c_last; ++c) {
                            const int sl = 2 * c + (range_begin(c, p.uq, p.ur) < tb ? 1 : 0);
                            const float* src = p.ws + static_cast<int64_t>(sl) * (TOK * ROWS);
#pragma unroll
                            for (int mi = 0; mi < MT; ++mi)
#pragma unroll
                                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                                    for (int e = 0; e < 4; ++e)
                                        sum[mi][nt][e] += __ldcg(src + (nt * 8 + 2 * t + (e & 1)) * ROWS +
                                                                 rloc[mi][e >> 1]);
                        }
#pragma unroll
                        for (int mi = 0; mi < MT; ++mi)
#pragma unroll
                            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    const int n = n0 + rloc[mi][e >> 1];
                                    const int tok = nt * 8 + 2 * t + (e & 1);
                                    if (n < p.N && tok < p.M)
                                        y[static_cast<int64_t>(tok) * p.N + n] = sum[mi][nt][e];
                                }
                        if (threadIdx.x == 0) p.cnt[tile] = 0;   // ready for the next launch
                    }
                    consumers_sync();
                }
            }
        }
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
                             cudaStream_t s, const GemvScratch* scratch) {
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
        int occ = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kGvThreads, Cfg::kSmem);
        if (e != cudaSuccess) return e;
        resident[dev] = occ > 0 ? occ : 1;
    }
    prm.n_tiles = (prm.N + Cfg::kRows - 1) / Cfg::kRows;
    prm.kstages = (prm.K + Cfg::kKPS - 1) / Cfg::kKPS;
    const int64_t tiles = static_cast<int64_t>(nmat) * prm.n_tiles;
    const int64_t units = tiles * prm.kstages;
    if (units >= (int64_t{1} << 31)) return cudaErrorInvalidValue;
    prm.units = static_cast<int>(units);
    // One wave of resident CTAs, each taking an equal run of units.
    const int64_t slots = static_cast<int64_t>(resident[dev]) * gv_num_sms();
    const int grid = static_cast<int>(units < slots ? units : slots);
    prm.uq = prm.units / grid;
    prm.ur = prm.units % grid;

    const size_t ws_bytes = static_cast<size_t>(2) * grid * Cfg::kTok * Cfg::kRows * sizeof(float);
    if (scratch == nullptr) {
        e = workspace_get(ws_bytes, static_cast<size_t>(tiles), &prm.ws, &prm.cnt);
        if (e != cudaSuccess) return e;
    } else {
        if (ws_bytes > scratch->ws_bytes || static_cast<size_t>(tiles) > scratch->n_cnt) {
            if (scratch->too_large) *scratch->too_large = true;
            return cudaErrorInvalidValue;
        }
        prm.ws = scratch->ws;
        prm.cnt = scratch->cnt;
    }

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
    cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
    cfg.blockDim = dim3(kGvThreads, 1, 1);
    cfg.dynamicSmemBytes = static_cast<size_t>(Cfg::kSmem);
    cfg.stream = s;
    cudaLaunchAttribute attrs[1];
    int na = 0;
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
                                   cudaStream_t s, const GemvScratch* sc) {
    // 8 tokens per n-tile
    if (prm.M <= 8) return gv_launch<BITS, 1, 1, SSC>(prm, x, codes, nmat, s, sc);
    if (prm.M <= 16) return gv_launch<BITS, 2, 1, SSC>(prm, x, codes, nmat, s, sc);
    if (prm.M <= 24) return gv_launch<BITS, 3, 1, SSC>(prm, x, codes, nmat, s, sc);
    return gv_launch<BITS, 4, 1, SSC>(prm, x, codes, nmat, s, sc);
}

template <int BITS>
static cudaError_t gv_dispatch(GvParams& prm, const void* x, const void* const* codes, int nmat,
                               cudaStream_t s, const GemvScratch* sc) {
    constexpr int gps = BITS == 4 ? 4 : 2;
    if (prm.groups % gps == 0) return gv_dispatch_ssc<BITS, true>(prm, x, codes, nmat, s, sc);
    return gv_dispatch_ssc<BITS, false>(prm, x, codes, nmat, s, sc);
}

static cudaError_t gemv_product(const uint16_t* x, int64_t M, int64_t K, int64_t N, int bits,
                                const WOperand* w, int nmat, cudaStream_t s, const GemvScratch* sc) {
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
    return bits == 4 ? gv_dispatch<4>(prm, x, codes, nmat, s, sc)
                     : gv_dispatch<8>(prm, x, codes, nmat, s, sc);
}

cudaError_t launch_gemv_product(const uint16_t* x, int64_t M, int64_t K, int64_t N, int bits,
                                const WOperand* w, int nmat, cudaStream_t s) {
    return gemv_product(x, M, K, N, bits, w, nmat, s, nullptr);
}

cudaError_t launch_gemv_product_scratch(const uint16_t* x, int64_t M, int64_t K, int64_t N,
                                        int bits, const WOperand* w, int nmat, cudaStream_t s,
                                        const GemvScratch* scratch) {
    return gemv_product(x, M, K, N, bits, w, nmat, s, scratch);
}

}  // namespace rq
