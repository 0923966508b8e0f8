// rq_tcs.cu -- streaming tensor-core product for small batches (1 <= M <= 64)
// on group-64 quantized weights (sm_100a).
//
//   y[m, n] = sum_g s16[n, g] * sum_{k in g} x[m, k] * code[n, k]
//
// The "Hakureirm/rwkv7-sglang-w4gptq-1.5b" model card (opening summary) pairs
// its int4 GEMV with a small-M GEMM over the same g64 format.  At a decode
// batch of 16..64 tokens the warp-level MMA (mma.sync) of the decode kernels
// becomes the bottleneck on B200 (it runs far below the fifth-generation
// tensor cores), so this kernel moves the contraction to tcgen05 while
// keeping the streaming shape of a decode kernel:
//
// Work.  A CTA owns one 256-row block of one matrix and a contiguous range
// of its stages (4 k groups of int4, 2 of int8): the ks CTAs of a
// thread-block cluster split the block's K range (ks chosen from the
// cluster occupancy so that the blocks run in as few waves as possible).
// Their fp32 partial sums meet in shared memory and are added across the
// cluster through distributed shared memory in rank order -- deterministic,
// no workspace, no atomics.
//
// Roles (704 threads):
//   warp 0      TMA producer: per unit the codes of 256 rows x 64 k (one box)
//               and the x tile [BNT tokens x 64 k] (128-byte swizzle, the
//               K-major B operand) into an SS-deep shared-memory ring.
//   warp 1      TMEM allocator and MMA issuer: per unit two 128-row MMAs
//               (tcgen05.mma kind::f16, M = 128, N = BNT, 4 steps of K = 16)
//               accumulating in TMEM.
//   warps 2-5   (int4) while the accumulators fill, put each stage's x
//               tiles into the pair order of the unpacking; then the
//               epilogue: tcgen05.ld of the accumulators, then y (or the
//               partial sums into shared memory for the cluster sum, which
//               all threads then share).
//   warps 6-21  four dequantiser groups of four warps; group g takes units
//               g, g+4, ...  Thread = rows r and r + 128 of the block (its
//               TMEM lane): it reads the rows' codes from shared memory,
//               forms fp16(code * s16) and tcgen05.st's them into the
//               group's A stage in tensor memory.
//
// int4 unpacking.  A code word (positions 0..7 of a row) becomes the pairs
// (p0,p4), (p1,p5), (p2,p6), (p3,p7) with one lop3 each (bit placement of Kim
// et al., arXiv:2211.10017: low nibbles as 1024 + c + 8, high nibbles as
// 64 + c + 8), an exact fp16 subtraction and the fp16 scale product.  That
// pair order is a permutation of k inside each 8-k chunk; the epilogue warps
// apply the same permutation to each stage's x tiles in shared memory (each
// 16-byte chunk in place, which the swizzle leaves intact) before the MMAs
// read them, so the sum over k is unchanged.
//
// Numerics: A = fp16(code * s16) (one rounding), fp32 accumulation in the
// tensor core, partial sums added in fp32 in k order.
//
// Every wait is bounded (rq_ptx.cuh); a timeout raises RQ_ERR_TIMEOUT in the
// device status word, the CTA winds down, waits for its own TMA copies, frees
// its TMEM and exits.
#include <cuda_fp16.h>

#include <cstring>

#include "rq_internal.h"
#include "rq_ptx.cuh"

namespace rq {

struct TcsParams {
    CUtensorMap tm_x[3];   // x of each input [M, K] fp16: box {64, BNT}, SWIZZLE_128B
    CUtensorMap tm_w[3];   // codes [N, K*bits/8] u8: box {64*bits/8, 256}, SWIZZLE_32B / 64B
    const uint16_t* scales[3];
    void* y[3];            // fp32 (or fp16 when yh) [M, N]
    int M, N, K;
    int nrb;               // 256-row blocks per matrix
    int kblocks;           // K / 64
    int nx;                // distinct inputs (1 shared, or one per matrix)
    int yh, epi;           // fp16 output; epilogue 1 = relu(y)^2
    int* status;
    uint64_t timeout_ns;
};

constexpr int kTcsRows = 256;          // rows per block (two 128-row MMA tiles)
constexpr int kTcsG = 4;               // dequantiser groups
constexpr int kTcsThreads = 32 * (2 + 4 + 4 * kTcsG);
constexpr int kTcsSmemBudget = 220 * 1024;

template <int BITS, int BNT>
struct TcsCfg {
    // A stage is KS k groups: 128 bytes of codes per row (one box of 256 rows
    // x 128 B, 128-byte swizzle) and the KS x tiles [BNT tokens x 64 k].
    static constexpr int KS = BITS == 4 ? 4 : 2;                  // k groups per stage
    static constexpr int kCodeBytes = 64 * BITS / 8;              // per row per k group
    static constexpr int kXTile = BNT * 128;                      // x of one k group
    static constexpr int kXStage = KS * kXTile;
    static constexpr int kWStage = kTcsRows * 128;
    static constexpr int kStage = kXStage + kWStage;
    // ring depth: as many stages as fit, a multiple of G / KS so that every
    // stage is always read by the same dequantiser groups (a group must never
    // see a stage's barrier two rounds ahead of it)
    static constexpr int kSSmul = kTcsG / KS;
    static constexpr int kSSraw = kTcsSmemBudget / kStage;
    static constexpr int kSS = kSSraw / kSSmul * kSSmul;
    static constexpr int kRing = kSS * kStage;
    // TMEM: the accumulators (2 tiles x BNT columns), then as many A stages
    // (2 tiles x 32 columns each) as fit in the 512 columns.  A group writes
    // k group i into A stage i % SA once the MMAs of k group i - SA are done;
    // with SA above the group count that wait is over long before.
    static constexpr int kAccCols = 2 * BNT;
    static constexpr int kACol0 = kAccCols;
    static constexpr int kSA = (512 - kAccCols) / 64;
    static constexpr int kColsNeeded = kACol0 + kSA * 64;
    static constexpr int kTmemCols = 512;
    static constexpr int kChunks = kCodeBytes / 16;               // 16-byte code chunks per group
    static constexpr int kBars = 3 * kSS + 2 * kSA + 1;
    static constexpr int kSmem = 1024 + kRing + kBars * 8 + 64;
    static_assert(kSS >= 2, "ring too shallow");
    static_assert(kColsNeeded <= 512 && kSA > kTcsG, "TMEM layout");
    static_assert(kXTile % 1024 == 0 && kWStage % 1024 == 0, "stage alignment");
    static_assert(kSmem <= 227 * 1024, "shared memory");
    // partial sums of a split K: [256 rows][kRedStride] fp32 in the ring, a
    // row's tokens contiguous (16-byte stores and loads); the 4-float pad
    // spreads consecutive rows over the banks
    static constexpr int kRedStride = BNT + 4;
    static_assert(kRing >= kTcsRows * kRedStride * 4, "the partial sums reuse the ring");
};

// 16-byte chunk c of row r of the codes box (128-byte rows, 128-byte swizzle:
// chunk index ^= row % 8, so the rows a warp reads hit distinct banks).
__device__ __forceinline__ uint4 tcs_code_chunk(const uint8_t* tile, int r, int c) {
    return *reinterpret_cast<const uint4*>(tile + r * 128 + ((c ^ (r & 7)) << 4));
}

__device__ __forceinline__ uint32_t tcs_lop3_6a(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0x6a;" : "=r"(d) : "r"(a), "r"(b), "r"(c));   // (a & b) ^ c
    return d;
}

__device__ __forceinline__ uint32_t h2u(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 u2h(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

// One row's 64 codes -> 32 TMEM columns of fp16(code * s) pairs.
//   int4: column 4w + j of word w holds (p_j, p_{j+4}) (the permuted order);
//   int8: column 2w + j holds (k 4w + 2j, 4w + 2j + 1).
template <int BITS>
__device__ __forceinline__ void tcs_dequant_row(const uint4 (&v)[BITS == 4 ? 2 : 4], __half2 s2,
                                                uint32_t (&a)[32]) {
    if constexpr (BITS == 4) {
        const __half2 b_lo = u2h(0x64086408u);    // 1032: (1024 + c + 8) - 1032 = c
        const __half2 b_hi = u2h(0x54805480u);    // 72:   (64 + c + 8) - 72 = c
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const uint32_t wv[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const uint32_t w8 = wv[w] >> 8;
                const uint32_t p0 = tcs_lop3_6a(wv[w], 0x000F000Fu, 0x64086408u);
                const uint32_t p1 = tcs_lop3_6a(wv[w], 0x00F000F0u, 0x54805480u);
                const uint32_t p2 = tcs_lop3_6a(w8, 0x000F000Fu, 0x64086408u);
                const uint32_t p3 = tcs_lop3_6a(w8, 0x00F000F0u, 0x54805480u);
                const int o = (c * 4 + w) * 4;
                a[o + 0] = h2u(__hmul2(__hsub2(u2h(p0), b_lo), s2));
                a[o + 1] = h2u(__hmul2(__hsub2(u2h(p1), b_hi), s2));
                a[o + 2] = h2u(__hmul2(__hsub2(u2h(p2), b_lo), s2));
                a[o + 3] = h2u(__hmul2(__hsub2(u2h(p3), b_hi), s2));
            }
        }
    } else {
        const __half2 bias = u2h(0x64806480u);    // 1152: 1024 + (c + 128) - 1152 = c
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const uint32_t wv[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const uint32_t u = wv[w] ^ 0x80808080u;
                const uint32_t q0 = __byte_perm(u, 0x64646464u, 0x5140u);
                const uint32_t q1 = __byte_perm(u, 0x64646464u, 0x5342u);
                const int o = (c * 4 + w) * 2;
                a[o + 0] = h2u(__hmul2(__hsub2(u2h(q0), bias), s2));
                a[o + 1] = h2u(__hmul2(__hsub2(u2h(q1), bias), s2));
            }
        }
    }
}

template <int BITS, int BNT>
__global__ void __launch_bounds__(kTcsThreads, 1) tcs_kernel(const __grid_constant__ TcsParams p) {
    using Cfg = TcsCfg<BITS, BNT>;
    constexpr int SS = Cfg::kSS;
    constexpr int SA = Cfg::kSA;
    constexpr int G = kTcsG;
    constexpr int KS = Cfg::KS;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    const uint32_t s0 = static_cast<uint32_t>(__cvta_generic_to_shared(smem_raw));
    uint8_t* smem = smem_raw + ((1024u - (s0 & 1023u)) & 1023u);
    uint8_t* ring = smem;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kRing);
    uint64_t* full = bars;                   // [SS] TMA landed (x + codes)
    uint64_t* empty = bars + SS;             // [SS] codes read, x fixed and MMAs done
    uint64_t* afull = bars + 2 * SS;         // [SA] A stage written
    uint64_t* aempty = bars + 2 * SS + SA;   // [SA] MMAs reading the A stage done
    uint64_t* accfull = bars + 2 * SS + 2 * SA;      // accumulators complete
    uint64_t* xready = accfull + 1;                   // [SS] (int4) x tiles put in pair order
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(xready + SS);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int ks = gridDim.x;                         // cluster size along K
    const int kq = blockIdx.x;                        // rank in the cluster
    const int blk = blockIdx.y;
    const int mat = blk / p.nrb;
    const int rb = blk - mat * p.nrb;
    const int KB = p.kblocks;
    const int nst = (KB + KS - 1) / KS;               // stages of a row
    const int st0 = static_cast<int>((static_cast<int64_t>(kq) * nst) / ks);
    const int st1 = static_cast<int>((static_cast<int64_t>(kq + 1) * nst) / ks);
    const int n_stages = st1 - st0;
    // k groups of this CTA: units 0 .. n_units-1 are k groups st0*KS + i
    // (those at or past KB, in the row's last stage, are zero-filled)
    const int n_units = n_stages * KS;
    const int kb0 = st0 * KS;
    const CUtensorMap* tmx = &p.tm_x[p.nx > 1 ? mat : 0];

    const int pre = n_stages < SS ? n_stages : SS;
    if (threadIdx.x == 0) {
        for (int s = 0; s < SS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 4 * KS + 1);
        }
        for (int a = 0; a < SA; ++a) {
            mbar_init(&afull[a], 4);
            mbar_init(&aempty[a], 1);
        }
        mbar_init(accfull, 1);
        for (int s = 0; s < SS; ++s) mbar_init(&xready[s], 4);
        *abort_flag = 0;
        fence_mbar_init();
        // codes never depend on the previous kernel: the first stages' go out
        // at once, while the rest of the CTA sets up
        tma_prefetch_desc(&p.tm_w[mat]);
        tma_prefetch_desc(tmx);
        const uint64_t pol_w = l2_policy_evict_first();
        for (int j = 0; j < pre; ++j) {
            mbar_arrive_expect_tx(&full[j], Cfg::kStage);
            tma_load_2d(ring + j * Cfg::kStage + Cfg::kXStage, &p.tm_w[mat], &full[j],
                        (st0 + j) * 128, rb * kTcsRows, pol_w);
        }
    }
    // dequantisers: their rows' scales, and the first unit's, also early
    const int dw = warp - 6;
    const int grp = dw >> 2;                        // k groups grp, grp + G, ...
    const uint16_t* srow[2] = {nullptr, nullptr};
    bool row_ok[2] = {false, false};
    uint16_t sc_next[2] = {0, 0};
    if (warp >= 6) {
#pragma unroll
        for (int tt = 0; tt < 2; ++tt) {
            const int n = rb * kTcsRows + tt * 128 + (warp & 3) * 32 + lane;
            row_ok[tt] = n < p.N;
            srow[tt] = p.scales[mat] + static_cast<int64_t>(row_ok[tt] ? n : 0) * KB;
            sc_next[tt] = (row_ok[tt] && grp < n_units && kb0 + grp < KB) ? __ldg(srow[tt] + kb0 + grp) : 0;
        }
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, Cfg::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    pdl_launch_dependents();

    if (warp == 0) {
        // ------------------------------------------------ TMA producer --
        if (threadIdx.x == 0) {
            const uint64_t pol_w = l2_policy_evict_first();   // codes: read once
            const uint64_t pol_x = l2_policy_evict_last();    // x: read by every block
            pdl_wait();
            for (int j = 0; j < pre; ++j)
                tma_load_3d(ring + j * Cfg::kStage, tmx, &full[j], 0, 0, (st0 + j) * KS, pol_x);
            int issued = pre;
            int s = 0;
            uint32_t ph = 0;            // parity of the round stage s is in
            for (int j = SS; j < n_stages; ++j) {
                if (!mbar_wait(&empty[s], ph, abort_flag, p.timeout_ns, p.status)) break;
                mbar_arrive_expect_tx(&full[s], Cfg::kStage);
                tma_load_2d(ring + s * Cfg::kStage + Cfg::kXStage, &p.tm_w[mat], &full[s],
                            (st0 + j) * 128, rb * kTcsRows, pol_w);
                tma_load_3d(ring + s * Cfg::kStage, tmx, &full[s], 0, 0, (st0 + j) * KS, pol_x);
                issued = j + 1;
                if (++s == SS) {
                    s = 0;
                    ph ^= 1u;
                }
            }
            // wait (bounded, even after an abort) for the copies issued last
            // into every stage, so none is in flight when the CTA exits
            int dummy_abort = 0;
            const int first = issued > SS ? issued - SS : 0;
            for (int j = first; j < issued; ++j)
                mbar_wait(&full[j % SS], static_cast<uint32_t>(j / SS) & 1u, &dummy_abort,
                          p.timeout_ns, p.status);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------- MMA issuer --
        if (elect_one()) {
            constexpr uint32_t idesc = idesc_f16_f32(128, BNT);
            for (int i = 0; i < n_units; ++i) {
                const int j = i / KS;                 // stage index within the CTA
                const int s = j % SS;
                const int a = i % SA;
                if (i % KS == 0 && !mbar_wait(&full[s], static_cast<uint32_t>(j / SS) & 1u, abort_flag,
                                              p.timeout_ns, p.status))
                    break;
                if (BITS == 4 && i % KS == 0 &&
                    !mbar_wait(&xready[s], static_cast<uint32_t>(j / SS) & 1u, abort_flag,
                               p.timeout_ns, p.status))
                    break;
                if (!mbar_wait(&afull[a], static_cast<uint32_t>(i / SA) & 1u, abort_flag,
                               p.timeout_ns, p.status))
                    break;
                tc_fence_after();
                const uint32_t xs = smem_u32(ring + s * Cfg::kStage + (i % KS) * Cfg::kXTile);
                const uint32_t acol = tmem_base + Cfg::kACol0 + a * 64;
#pragma unroll
                for (int tt = 0; tt < 2; ++tt)
#pragma unroll
                    for (int t = 0; t < 4; ++t)
                        tc_mma_ts(tmem_base + tt * BNT, acol + tt * 32 + t * 8,
                                  smem_desc_k_sw128(xs + t * 32), idesc, (i == 0 && t == 0) ? 0u : 1u);
                tc_commit(&aempty[a]);
                if (i % KS == KS - 1) tc_commit(&empty[s]);
            }
            tc_commit(accfull);
        }
        __syncwarp();
    } else if (warp < 6) {
        // --------------------------------------------------- epilogue --
        const int q = warp & 3;                     // TMEM lane quarter
        const int r0 = q * 32 + lane;               // row of tile 0; tile 1: + 128
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
        pdl_wait();                                 // y: after the previous grid
        if constexpr (BITS == 4) {
            // While the accumulators fill, these warps put every stage's x
            // tiles into the pair order of the int4 unpacking (each 16-byte
            // chunk in place; the swizzle moves whole chunks), off the
            // dequantisers' path; the MMAs wait for it per stage.
            const int et = threadIdx.x - 64;        // 0 .. 127
            for (int j = 0; j < n_stages; ++j) {
                const int s = j % SS;
                if (!mbar_wait(&full[s], static_cast<uint32_t>(j / SS) & 1u, abort_flag, p.timeout_ns,
                               p.status))
                    break;
                uint8_t* xs = ring + s * Cfg::kStage;
                for (int ch = et; ch < KS * BNT * 8; ch += 128) {
                    uint4* xp = reinterpret_cast<uint4*>(xs + ch * 16);
                    const uint4 xv = *xp;
                    uint4 o;
                    o.x = __byte_perm(xv.x, xv.z, 0x5410);
                    o.y = __byte_perm(xv.x, xv.z, 0x7632);
                    o.z = __byte_perm(xv.y, xv.w, 0x5410);
                    o.w = __byte_perm(xv.y, xv.w, 0x7632);
                    *xp = o;
                }
                // the MMAs read x through the async proxy
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
                if (lane == 0) mbar_arrive(&xready[s]);
            }
        }
        // (suspending between checks: these warps wait for most of the kernel)
        const bool ok = mbar_wait_suspend(accfull, 0, abort_flag, p.timeout_ns, p.status);
        tc_fence_after();
        if (ok && !*abort_flag) {
            float* red = reinterpret_cast<float*>(ring);     // [256][kRedStride] when ks > 1
#pragma unroll 1
            for (int tt = 0; tt < 2; ++tt) {
                const int r = tt * 128 + r0;
                const int n = rb * kTcsRows + r;
#pragma unroll 1
                for (int j0 = 0; j0 < BNT && j0 < p.M; j0 += 16) {
                    uint32_t v[16];
                    tmem_ld_32x32b_x16(lane_base + tt * BNT + j0, v);
                    tc_wait_ld();
                    if (ks > 1) {
                        // the row's 16 token sums (those past M are never read)
                        float4* dst = reinterpret_cast<float4*>(red + r * Cfg::kRedStride + j0);
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            dst[u] = make_float4(__uint_as_float(v[4 * u]), __uint_as_float(v[4 * u + 1]),
                                                 __uint_as_float(v[4 * u + 2]), __uint_as_float(v[4 * u + 3]));
                        continue;
                    }
#pragma unroll
                    for (int jj = 0; jj < 16; ++jj) {
                        const int m = j0 + jj;
                        if (m >= p.M) break;
                        float val = __uint_as_float(v[jj]);
                        if (n < p.N) {
                            if (p.epi == 1) {
                                val = fmaxf(val, 0.0f);
                                val = val * val;
                            }
                            const int64_t at = static_cast<int64_t>(m) * p.N + n;
                            if (p.yh)
                                static_cast<__half*>(p.y[mat])[at] = __float2half_rn(val);
                            else
                                static_cast<float*>(p.y[mat])[at] = val;
                        }
                    }
                }
            }
        }
    } else {
        // ---------------------------------------- dequantise into TMEM --
        const int q = warp & 3;                     // TMEM lane quarter
        const int r0 = q * 32 + lane;
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
        // scales of this thread's rows for unit i (0 outside the matrix and
        // past the row's last k group)
        auto scales_of = [&](int i, uint16_t (&sc)[2]) {
            const int kb = kb0 + i;
#pragma unroll
            for (int tt = 0; tt < 2; ++tt)
                sc[tt] = (row_ok[tt] && i < n_units && kb < KB) ? __ldg(srow[tt] + kb) : 0;
        };
        for (int i = grp; i < n_units; i += G) {
            const int j = i / KS;
            const int s = j % SS;
            const int a = i % SA;
            const int kj = i % KS;                      // k group within the stage
            uint16_t sc[2] = {sc_next[0], sc_next[1]};
            scales_of(i + G, sc_next);
            if (!mbar_wait(&full[s], static_cast<uint32_t>(j / SS) & 1u, abort_flag, p.timeout_ns,
                           p.status))
                break;
            uint8_t* st = ring + s * Cfg::kStage;
            const uint8_t* wt = st + Cfg::kXStage;
            uint4 v[2][Cfg::kChunks];
#pragma unroll
            for (int tt = 0; tt < 2; ++tt)
#pragma unroll
                for (int c = 0; c < Cfg::kChunks; ++c)
                    v[tt][c] = tcs_code_chunk(wt, tt * 128 + r0, kj * Cfg::kChunks + c);
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            if (i >= SA && !mbar_wait(&aempty[a], static_cast<uint32_t>(i / SA - 1) & 1u, abort_flag,
                                      p.timeout_ns, p.status))
                break;
            tc_fence_after();
#pragma unroll
            for (int tt = 0; tt < 2; ++tt) {
                const __half2 s2 = __halves2half2(__ushort_as_half(sc[tt]), __ushort_as_half(sc[tt]));
                uint32_t regs[32];
                tcs_dequant_row<BITS>(v[tt], s2, regs);
                tmem_st_32x32b_x32(lane_base + Cfg::kACol0 + a * 64 + tt * 32, regs);
            }
            tc_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&afull[a]);
        }
    }

    tc_fence_before();
    __syncthreads();

    if (ks > 1) {
        // Fixed-order sum of the cluster's partials through distributed shared
        // memory, every thread of the CTA taking part.  Every CTA reaches both
        // cluster barriers on every path.
        cluster_sync();
        if (!*abort_flag) {
            // element e: rows fastest (so a warp's y stores are 32
            // consecutive n), then groups of 4 tokens
            const int MQ = (p.M + 3) / 4;
            const int E4 = MQ * kTcsRows;
            const int e0 = static_cast<int>((static_cast<int64_t>(kq) * E4) / ks);
            const int e1 = static_cast<int>((static_cast<int64_t>(kq + 1) * E4) / ks);
            const uint32_t red_local = smem_u32(ring);
            for (int e = e0 + static_cast<int>(threadIdx.x); e < e1; e += kTcsThreads) {
                const int m4 = e / kTcsRows;
                const int r = e - m4 * kTcsRows;
                const uint32_t off = static_cast<uint32_t>(r * Cfg::kRedStride + 4 * m4) * 4u;
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
                for (int src0 = 0; src0 < ks; src0 += 4) {
                    // four ranks' loads in flight at once, added in rank order
                    float4 v[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        if (src0 + u < ks) v[u] = ld_dsmem_f32x4(map_to_rank(red_local + off, src0 + u));
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        if (src0 + u < ks) {
                            acc.x += v[u].x;
                            acc.y += v[u].y;
                            acc.z += v[u].z;
                            acc.w += v[u].w;
                        }
                }
                const int n = rb * kTcsRows + r;
                if (n >= p.N) continue;
                const float out[4] = {acc.x, acc.y, acc.z, acc.w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int m = 4 * m4 + u;
                    if (m >= p.M) break;
                    float val = out[u];
                    if (p.epi == 1) {
                        val = fmaxf(val, 0.0f);
                        val = val * val;
                    }
                    const int64_t at = static_cast<int64_t>(m) * p.N + n;
                    if (p.yh)
                        static_cast<__half*>(p.y[mat])[at] = __float2half_rn(val);
                    else
                        static_cast<float*>(p.y[mat])[at] = val;
                }
            }
        }
        cluster_sync();
    }

    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, Cfg::kTmemCols);
    }
}

// ------------------------------------------------------------- launcher --

static int tcs_bnt(int64_t M) { return M <= 16 ? 16 : M <= 32 ? 32 : 64; }

bool tcs_fits(int64_t M, int64_t K, int64_t N, int bits) {
    (void)K;
    (void)N;
    return M >= 1 && M <= 64 && (bits == 4 || bits == 8);
}

// K split (cluster size): as many CTAs per block as keep blocks x ks within
// the SMs, at most 16 and at most one per stage of k groups.
int tcs_ksplit(int64_t K, int64_t N, int nmat, int bits) {
    const int64_t blocks = static_cast<int64_t>(nmat) * ((N + kTcsRows - 1) / kTcsRows);
    int64_t ks = num_sms() / blocks;
    const int64_t kb = (K / kGroup + (bits == 4 ? 3 : 1)) / (bits == 4 ? 4 : 2);   // stages
    if (ks > 16) ks = 16;
    if (ks > kb) ks = kb;
    if (ks < 1) ks = 1;
    return static_cast<int>(ks);
}

// How many clusters of `ks` CTAs of this kernel the device can hold at once
// (cached per device and size; 0: such a cluster cannot be scheduled).
template <int BITS, int BNT>
static int tcs_active_clusters(int dev, int ks) {
    using Cfg = TcsCfg<BITS, BNT>;
    static int cache[64][17] = {};                 // value + 1; 0 = not asked yet
    if (cache[dev][ks] == 0) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(ks), 1, 1);
        cfg.blockDim = dim3(kTcsThreads, 1, 1);
        cfg.dynamicSmemBytes = static_cast<size_t>(Cfg::kSmem);
        cudaLaunchAttribute attr;
        attr.id = cudaLaunchAttributeClusterDimension;
        attr.val.clusterDim.x = static_cast<unsigned>(ks);
        attr.val.clusterDim.y = 1;
        attr.val.clusterDim.z = 1;
        cfg.attrs = &attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, tcs_kernel<BITS, BNT>, &cfg) != cudaSuccess) {
            cudaGetLastError();
            n = 0;
        }
        cache[dev][ks] = n + 1;
    }
    return cache[dev][ks] - 1;
}

template <int BITS, int BNT>
static cudaError_t tcs_launch_cfg(const TcsParams& prm, int ks_want, int blocks, cudaStream_t s) {
    using Cfg = TcsCfg<BITS, BNT>;
    auto kern = tcs_kernel<BITS, BNT>;
    static bool attr_set[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!attr_set[dev]) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmem);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    // the cluster size with the least time per block: a block's work shrinks
    // as 1/ks, but clusters must fit in a GPC, so large ones may not all be
    // resident at once and then run in waves (ks / waves is the figure of merit)
    int ks = 1;
    double best = -1.0;
    for (int c = ks_want; c >= 1; --c) {
        const int act = tcs_active_clusters<BITS, BNT>(dev, c);
        if (act <= 0) continue;
        const int waves = (blocks + act - 1) / act;
        const double merit = static_cast<double>(c) / waves;
        if (merit > best) {
            best = merit;
            ks = c;
        }
    }
    if (best < 0) return cudaErrorInvalidConfiguration;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(ks), static_cast<unsigned>(blocks), 1);
    cfg.blockDim = dim3(kTcsThreads, 1, 1);
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
    return cudaLaunchKernelEx(&cfg, kern, prm);
}

cudaError_t launch_tcs(const uint16_t* const* xs, int nx, int64_t M, int64_t K, int64_t N,
                       int bits, const WOperand* w, int nmat, bool y_half, int epilogue,
                       cudaStream_t s) {
    if (!tcs_fits(M, K, N, bits)) return cudaErrorInvalidValue;
    const int bnt = tcs_bnt(M);
    TcsParams prm;
    memset(&prm, 0, sizeof(prm));
    prm.M = static_cast<int>(M);
    prm.N = static_cast<int>(N);
    prm.K = static_cast<int>(K);
    prm.nrb = static_cast<int>((N + kTcsRows - 1) / kTcsRows);
    prm.kblocks = static_cast<int>(K / kGroup);
    prm.nx = nx;
    prm.yh = y_half ? 1 : 0;
    prm.epi = epilogue;
    prm.status = device_status_ptr();
    prm.timeout_ns = wait_limit_ns();
    const int ks = tcs_ksplit(K, N, nmat, bits);
    const int blocks = nmat * prm.nrb;
    const uint64_t row_bytes = static_cast<uint64_t>(K) * bits / 8;
    for (int i = 0; i < nmat; ++i) {
        if (!make_tmap_2d(&prm.tm_w[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, w[i].codes, row_bytes,
                          static_cast<uint64_t>(N), row_bytes, 128, kTcsRows,
                          CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
        prm.scales[i] = w[i].scales;
        prm.y[i] = w[i].y;
    }
    // x as {64 k, M tokens, K/64 groups}: one box per stage = KS x tiles
    const uint32_t kstage = bits == 4 ? 4 : 2;
    for (int i = 0; i < nx; ++i)
        if (!make_tmap_3d(&prm.tm_x[i], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, xs[i], 64,
                          static_cast<uint64_t>(M), static_cast<uint64_t>(K / kGroup),
                          static_cast<uint64_t>(K) * 2, 128, 64, static_cast<uint32_t>(bnt), kstage,
                          CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;
    if (bits == 4)
        return bnt == 16 ? tcs_launch_cfg<4, 16>(prm, ks, blocks, s)
               : bnt == 32 ? tcs_launch_cfg<4, 32>(prm, ks, blocks, s)
                           : tcs_launch_cfg<4, 64>(prm, ks, blocks, s);
    return bnt == 16 ? tcs_launch_cfg<8, 16>(prm, ks, blocks, s)
           : bnt == 32 ? tcs_launch_cfg<8, 32>(prm, ks, blocks, s)
                       : tcs_launch_cfg<8, 64>(prm, ks, blocks, s);
}

}  // namespace rq
