// rq_tc.cu -- tensor-core product on group-64 quantized weights (sm_100a).
//
//   y[m, n] = sum_k x[m, k] * code[n, k] * s16[n, k/64]
//
// The "RWKV-7 Quantization Toolkit" (rwkv-quant-nv 1.2.1) "Key Design" list
// keeps the weights quantized on the inference path and computes R/K/V in one
// launch; the "Hakureirm/rwkv7-sglang-w4gptq-1.5b" model card names a
// small-M GEMM and a tensor-core GEMM over the same int4 g64 format.  This
// kernel is the B200 form of both: the weight tile is dequantised straight
// into TENSOR MEMORY and used there as the A operand of tcgen05.mma, so no
// dequantised weight ever touches HBM or shared memory.
//
// Roles (64 + 128*G threads):
//   warp 0     TMA producer: codes tile [128 rows x 64 k] and x tile
//              [BNT tokens x 64 k] per k-block into an SS-deep shared-memory
//              ring (deep, to keep enough bytes in flight for HBM).
//   warp 1     TMEM allocator + MMA issuer: 4 x tcgen05.mma (M=128, N=BNT,
//              K=16) per k-block, D[n, token] accumulates in TMEM (fp32).
//   warps 2..  G dequantiser groups of 4 warps (one warp per TMEM lane
//              quarter); group g takes k-blocks g, g+G, g+2G, ... so G
//              k-blocks are in flight at once.  Thread = one weight row n (its
//              TMEM lane): it reads the row's 64 codes from shared memory,
//              releases the shared-memory stage, forms fp16(code * s16) and
//              tcgen05.st's them into one of SA = 2G tensor-memory A stages.
//              After the K loop group 0 is the epilogue (tcgen05.ld -> y, or
//              -> shared memory for the split-K sum).
//
// Split-K: the CTAs of one thread-block cluster (gridDim.x = cluster size)
// share one (matrix, 128-row tile, token tile) and take disjoint k-block
// ranges; their fp32 partials are summed in a fixed order through distributed
// shared memory -- deterministic, no atomics, no global workspace.
//
// Operand layouts:
//   A (TMEM): lane = weight row, 32-bit column j of a stage = fp16 pair
//             (k = 2j, 2j+1) of that row's k-block (64 k = 32 columns).
//   B (smem): x tile, K-major, 128-byte swizzle (TMA SWIZZLE_128B).
//   codes (smem): 128 rows x 32 B (int4, TMA SWIZZLE_32B) or x 64 B (int8,
//             SWIZZLE_64B): the swizzle makes the row-per-thread reads free
//             of bank conflicts.
//
// Every mbarrier wait is bounded (see rq_ptx.cuh); a timeout sets the
// device status word to RQ_ERR_TIMEOUT and the CTA winds down, waits for its
// own TMA copies, frees its TMEM and exits.
#include "rq_internal.h"
#include "rq_ptx.cuh"

namespace rq {

struct TcParams {
    CUtensorMap tm_x;     // x [M, K] fp16: dims {K, M}, box {64, BNT}, SWIZZLE_128B
    CUtensorMap tm_w[3];  // codes [N, K*bits/8] u8: box {64*bits/8, 128}, SWIZZLE_32B/64B
    const uint16_t* scales[3];
    float* y[3];
    int M, N, K;
    int n_tiles;          // ceil(N / 128): row tiles per matrix
    int kblocks;          // K / 64
    int* status;          // device status word
    uint64_t timeout_ns;
};

constexpr int kRows = 128;   // weight rows per CTA (MMA M)
constexpr int kKB = 64;      // k per pipeline stage (one group)

template <int BITS, int BNT, int SS, int G>
struct TcCfg {
    static constexpr int kSA = 2 * G;                             // tensor-memory A stages
    static constexpr int kThreads = 64 + 128 * G;
    static constexpr int kCodeBytes = kKB * BITS / 8;             // per row per stage
    static constexpr int kXStage = BNT * 128;                     // bytes
    static constexpr int kWStage = kRows * kCodeBytes;            // bytes
    static constexpr int kStage = kXStage + kWStage;
    static constexpr int kRing = SS * kStage;
    static constexpr int kRed = kRows * BNT * 4;                  // split-K partial (fp32)
    static constexpr int kData = kRing > kRed ? kRing : kRed;
    static constexpr int kBars = (2 * SS + 2 * kSA + 1) * 8 + 16;
    static constexpr int kSmem = 1024 /*align slack*/ + kData + ((kBars + 127) / 128) * 128;
    // Independent accumulators: consecutive MMAs rotate over them so that
    // small-N MMAs do not wait on each other's accumulation.
    static constexpr int kNAcc = BNT >= 256 ? 1 : (256 / BNT > 8 ? 8 : 256 / BNT);
    static constexpr int kAccCols = kNAcc * BNT;
    static constexpr int kAStageCols = kKB / 2;                    // 32 columns
    static constexpr int kColsNeeded = kAccCols + kSA * kAStageCols;
    static constexpr int kTmemCols = kColsNeeded <= 32    ? 32
                                     : kColsNeeded <= 64  ? 64
                                     : kColsNeeded <= 128 ? 128
                                     : kColsNeeded <= 256 ? 256
                                                          : 512;
    static constexpr int kChunks = kCodeBytes / 16;               // 16-byte code chunks per row
    static_assert(kColsNeeded <= 512, "TMEM overflow");
    static_assert(kXStage % 1024 == 0 && kWStage % 1024 == 0, "stage alignment");
    static_assert(SS % G == 0, "each ring stage must belong to one dequantiser group");
};

// Read one 16-byte chunk `c` of row `r` from a swizzled codes tile.
template <int BITS>
__device__ __forceinline__ uint4 load_code_chunk(const uint8_t* tile, int r, int c) {
    if constexpr (BITS == 4) {
        // 32-byte rows, SWIZZLE_32B: chunk bit 0 ^= address bit 7 (row bit 2)
        const int pc = c ^ ((r >> 2) & 1);
        return *reinterpret_cast<const uint4*>(tile + r * 32 + pc * 16);
    } else {
        // 64-byte rows, SWIZZLE_64B: chunk bits 0..1 ^= address bits 7..8 (row bits 1..2)
        const int pc = c ^ ((r >> 1) & 3);
        return *reinterpret_cast<const uint4*>(tile + r * 64 + pc * 16);
    }
}

// Dequantise one row's k-block (64 codes) into 32 packed fp16-pair registers.
template <int BITS>
__device__ __forceinline__ void dequant_row(const uint4 (&v)[BITS == 4 ? 2 : 4], __half2 s2,
                                            uint32_t (&a)[32]) {
    constexpr int NCH = BITS == 4 ? 2 : 4;
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
        const uint32_t wv[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
        if constexpr (BITS == 4) {
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                uint32_t o[4];
                dequant8_i4(wv[w], s2, o);
#pragma unroll
                for (int j = 0; j < 4; ++j) a[c * 16 + w * 4 + j] = o[j];
            }
        } else {
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                uint32_t o[2];
                dequant4_i8(wv[w], s2, o);
                a[c * 8 + w * 2 + 0] = o[0];
                a[c * 8 + w * 2 + 1] = o[1];
            }
        }
    }
}

template <int BITS, int BNT, int SS, int G>
__global__ void __launch_bounds__(TcCfg<BITS, BNT, SS, G>::kThreads, 1)
    tc_wq_kernel(const __grid_constant__ TcParams p) {
    using Cfg = TcCfg<BITS, BNT, SS, G>;
    constexpr int SA = Cfg::kSA;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint8_t* ring = smem;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kData);
    uint64_t* full = bars;                    // [SS] TMA landed (x + codes)
    uint64_t* empty = bars + SS;              // [SS] codes read by dequant + x read by MMA
    uint64_t* afull = bars + 2 * SS;          // [SA] A stage written to TMEM
    uint64_t* aempty = bars + 2 * SS + SA;    // [SA] MMAs reading the A stage complete
    uint64_t* accf = bars + 2 * SS + 2 * SA;  // accumulator complete
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(accf + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int ksplit = gridDim.x;
    const int kq = blockIdx.x;                        // rank in the cluster
    const int mat = blockIdx.y / p.n_tiles;
    const int n0 = (blockIdx.y - mat * p.n_tiles) * kRows;
    const int m0 = blockIdx.z * BNT;
    const int kb0 = static_cast<int>((static_cast<int64_t>(kq) * p.kblocks) / ksplit);
    const int kb1 = static_cast<int>((static_cast<int64_t>(kq + 1) * p.kblocks) / ksplit);
    const int nkb = kb1 - kb0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < SS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 4 + 1);
        }
        for (int a = 0; a < SA; ++a) {
            mbar_init(&afull[a], 4);
            mbar_init(&aempty[a], 1);
        }
        mbar_init(accf, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&p.tm_x);
        tma_prefetch_desc(&p.tm_w[mat]);
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, Cfg::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;
    const uint32_t acc_col = 0;
    const uint32_t a_col0 = Cfg::kAccCols;

    // Let the next kernel in the stream start its prologue (weight prefetch)
    // while this one runs; it still waits for our results before reading x.
    pdl_launch_dependents();

    if (warp == 0) {
        // ------------------------------------------------ TMA producer --
        if (elect_one()) {
            const uint64_t pol_w = l2_policy_evict_first();   // codes: streamed once
            const uint64_t pol_x = l2_policy_evict_last();    // x: re-read by every row tile
            const CUtensorMap* tmw = &p.tm_w[mat];
            int issued = 0;
            const int pre = nkb < SS ? nkb : SS;
            // Weights do not depend on the previous kernel: fetch the first
            // stages' codes before waiting for it.
            for (int i = 0; i < pre; ++i) {
                mbar_arrive_expect_tx(&full[i], Cfg::kStage);
                tma_load_2d(ring + i * Cfg::kStage + Cfg::kXStage, tmw, &full[i],
                            (kb0 + i) * Cfg::kCodeBytes, n0, pol_w);
            }
            pdl_wait();
            for (int i = 0; i < pre; ++i)
                tma_load_2d(ring + i * Cfg::kStage, &p.tm_x, &full[i], (kb0 + i) * kKB, m0, pol_x);
            issued = pre;
            for (int i = SS; i < nkb; ++i) {
                const int s = i % SS;
                const uint32_t r = static_cast<uint32_t>(i / SS);
                if (!mbar_wait(&empty[s], (r - 1) & 1, abort_flag, p.timeout_ns, p.status)) break;
                mbar_arrive_expect_tx(&full[s], Cfg::kStage);
                tma_load_2d(ring + s * Cfg::kStage + Cfg::kXStage, tmw, &full[s],
                            (kb0 + i) * Cfg::kCodeBytes, n0, pol_w);
                tma_load_2d(ring + s * Cfg::kStage, &p.tm_x, &full[s], (kb0 + i) * kKB, m0, pol_x);
                issued = i + 1;
            }
            // Wait (bounded, regardless of abort) until the copies this thread
            // issued have landed, so none is in flight when the CTA exits.
            int dummy_abort = 0;
            const int first = issued > SS ? issued - SS : 0;
            for (int i = first; i < issued; ++i)
                mbar_wait(&full[i % SS], static_cast<uint32_t>(i / SS) & 1, &dummy_abort,
                          p.timeout_ns, p.status);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------- MMA issuer --
        if (elect_one()) {
            const uint32_t idesc = idesc_f16_f32(kRows, BNT);
            for (int i = 0; i < nkb; ++i) {
                const int s = i % SS;
                const int a = i % SA;
                if (!mbar_wait(&full[s], static_cast<uint32_t>(i / SS) & 1, abort_flag,
                               p.timeout_ns, p.status))
                    break;
                if (!mbar_wait(&afull[a], static_cast<uint32_t>(i / SA) & 1, abort_flag,
                               p.timeout_ns, p.status))
                    break;
                tc_fence_after();
                const uint32_t xs = smem_u32(ring + s * Cfg::kStage);
#pragma unroll
                for (int t = 0; t < kKB / 16; ++t) {
                    const uint64_t bdesc = smem_desc_k_sw128(xs + t * 32);
                    const uint32_t a_taddr = tmem_base + a_col0 + a * Cfg::kAStageCols + t * 8;
                    const int step = i * (kKB / 16) + t;
                    const uint32_t d_taddr = tmem_base + acc_col + (step % Cfg::kNAcc) * BNT;
                    tc_mma_ts(d_taddr, a_taddr, bdesc, idesc, step >= Cfg::kNAcc);
                }
                tc_commit(&empty[s]);
                tc_commit(&aempty[a]);
            }
            tc_commit(accf);
        }
        __syncwarp();
    } else {
        // ---------------------------------------- dequantise into TMEM --
        const int dw = warp - 2;
        const int grp = dw >> 2;                // dequant group: k-blocks grp, grp+G, ...
        const int q = warp & 3;                 // TMEM lane quarter of this warp
        const int r = q * 32 + lane;            // weight row within the tile
        const int n = n0 + r;
        const bool row_ok = n < p.N;
        const uint16_t* srow = p.scales[mat] + static_cast<int64_t>(row_ok ? n : 0) * p.kblocks;
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
        // scale prefetch: this group's next two k-blocks
        uint16_t sc0 = (row_ok && grp < nkb) ? __ldg(srow + kb0 + grp) : 0;
        uint16_t sc1 = (row_ok && grp + G < nkb) ? __ldg(srow + kb0 + grp + G) : 0;
        for (int i = grp; i < nkb; i += G) {
            const int s = i % SS;
            const int a = i % SA;
            const uint16_t s_cur = sc0;
            sc0 = sc1;
            sc1 = (row_ok && i + 2 * G < nkb) ? __ldg(srow + kb0 + i + 2 * G) : 0;
            if (!mbar_wait(&full[s], static_cast<uint32_t>(i / SS) & 1, abort_flag, p.timeout_ns,
                           p.status))
                break;
            const uint8_t* wt = ring + s * Cfg::kStage + Cfg::kXStage;
            uint4 v[Cfg::kChunks];
#pragma unroll
            for (int c = 0; c < Cfg::kChunks; ++c) v[c] = load_code_chunk<BITS>(wt, r, c);
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);          // codes consumed: stage reusable
            if (i >= SA && !mbar_wait(&aempty[a], static_cast<uint32_t>(i / SA - 1) & 1,
                                      abort_flag, p.timeout_ns, p.status))
                break;
            tc_fence_after();
            const __half2 s2 = __halves2half2(__ushort_as_half(s_cur), __ushort_as_half(s_cur));
            uint32_t regs[32];
            dequant_row<BITS>(v, s2, regs);
            tmem_st_32x32b_x32(lane_base + a_col0 + a * Cfg::kAStageCols, regs);
            tc_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&afull[a]);
        }

        // ------------------------------------------------------ epilogue --
        if (grp == 0) {
            const bool acc_ok = mbar_wait(accf, 0, abort_flag, p.timeout_ns, p.status);
            tc_fence_after();
            if (acc_ok && !*abort_flag) {
                float* red = reinterpret_cast<float*>(ring);
                float* y = p.y[mat];
                const int used = nkb * (kKB / 16) < Cfg::kNAcc ? nkb * (kKB / 16) : Cfg::kNAcc;
#pragma unroll 1
                for (int j0 = 0; j0 < BNT; j0 += 16) {
                    uint32_t vv[16];
                    tmem_ld_32x32b_x16(lane_base + acc_col + j0, vv);
                    tc_wait_ld();
                    for (int u = 1; u < used; ++u) {
                        uint32_t w2[16];
                        tmem_ld_32x32b_x16(lane_base + acc_col + u * BNT + j0, w2);
                        tc_wait_ld();
#pragma unroll
                        for (int jj = 0; jj < 16; ++jj)
                            vv[jj] = __float_as_uint(__uint_as_float(vv[jj]) + __uint_as_float(w2[jj]));
                    }
                    if (ksplit == 1) {
                        if (row_ok) {
#pragma unroll
                            for (int jj = 0; jj < 16; ++jj) {
                                const int m = m0 + j0 + jj;
                                if (m < p.M)
                                    y[static_cast<int64_t>(m) * p.N + n] = __uint_as_float(vv[jj]);
                            }
                        }
                    } else {
#pragma unroll
                        for (int jj = 0; jj < 16; ++jj)
                            red[(j0 + jj) * kRows + r] = __uint_as_float(vv[jj]);
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();

    if (ksplit > 1) {
        // Fixed-order sum of the cluster's partials through distributed shared
        // memory.  Every CTA reaches both cluster barriers on every path.
        cluster_sync();
        if (!*abort_flag) {
            constexpr int E4 = kRows * BNT / 4;
            const int e0 = static_cast<int>((static_cast<int64_t>(kq) * E4) / ksplit);
            const int e1 = static_cast<int>((static_cast<int64_t>(kq + 1) * E4) / ksplit);
            const uint32_t red_local = smem_u32(ring);
            float* y = p.y[mat];
            for (int e = e0 + static_cast<int>(threadIdx.x); e < e1; e += Cfg::kThreads) {
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
                for (int src = 0; src < ksplit; ++src) {
                    const float4 v = ld_dsmem_f32x4(map_to_rank(red_local + e * 16, src));
                    acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
                }
                const int j = (e * 4) / kRows;
                const int r = (e * 4) % kRows;
                const int m = m0 + j;
                if (m < p.M) {
                    const float out[4] = {acc.x, acc.y, acc.z, acc.w};
                    float* yrow = y + static_cast<int64_t>(m) * p.N;
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        if (n0 + r + u < p.N) yrow[n0 + r + u] = out[u];
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

// Shared-memory ring depth per configuration: as many stages as fit in about
// 190 KB (one CTA per SM), at most 32, and a multiple of the dequantiser group
// count.  The multiple matters for correctness: k-block i uses stage i % SS
// and group i % G, so with G | SS every stage belongs to one group, which
// waits on that stage's barrier round after round.  Otherwise a group could
// wait for round r+1 of a stage while round r is still in flight, and the
// parity wait would report the earlier phase as complete.
constexpr int ring_stages(int bits, int bnt) {
    return ((190 * 1024) / (bnt * 128 + kRows * kKB * bits / 8) > 32
                ? 32
                : (190 * 1024) / (bnt * 128 + kRows * kKB * bits / 8)) /
           4 * 4;
}
constexpr int kGroups = 4;
static_assert(ring_stages(4, 256) % kGroups == 0 && ring_stages(8, 256) >= kGroups,
              "ring depth must be a positive multiple of the group count");

struct TcChoice {
    int bnt;      // tokens per tile (MMA N)
    int ksplit;   // cluster size along K
};

static TcChoice choose(int64_t M, int64_t N, int64_t K, int nmat) {
    TcChoice c;
    if (M <= 16) c.bnt = 16;
    else if (M <= 32) c.bnt = 32;
    else if (M <= 64) c.bnt = 64;
    else if (M <= 128) c.bnt = 128;
    else c.bnt = 256;
    const int64_t kblocks = K / kGroup;
    const int64_t tiles = nmat * ((N + kRows - 1) / kRows) * ((M + c.bnt - 1) / c.bnt);
    const int64_t slots = static_cast<int64_t>(num_sms());
    // Split K across a cluster while the grid still fits in one wave of
    // resident CTAs and every CTA keeps at least 4 k-blocks.
    int ks = 1;
    while (ks < 8 && tiles * (ks + 1) <= slots && kblocks / (ks + 1) >= 4) ++ks;
    c.ksplit = ks;
    return c;
}

// Dynamic shared memory for a configuration, raised if needed so that the
// CTAs that can be co-resident on one SM never ask for more than the SM's 512
// TMEM columns together.  tcgen05.alloc blocks until columns are free; with
// clusters, a CTA blocked there while its cluster peers wait for it at the
// cluster barrier could otherwise wait on CTAs that wait on it.
template <int BITS, int BNT, int SS, int GR>
static cudaError_t resident_safe_smem(int* out) {
    using Cfg = TcCfg<BITS, BNT, SS, GR>;
    static int cached[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64 && cached[dev] > 0) {
        *out = cached[dev];
        return cudaSuccess;
    }
    auto kern = tc_wq_kernel<BITS, BNT, SS, GR>;
    int max_optin = 0;
    e = cudaDeviceGetAttribute(&max_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e != cudaSuccess) return e;
    if (Cfg::kSmem > max_optin) return cudaErrorInvalidConfiguration;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, max_optin);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    int smem = Cfg::kSmem;
    const int max_resident = 512 / Cfg::kTmemCols;
    while (true) {
        int occ = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, Cfg::kThreads, smem);
        if (e != cudaSuccess) return e;
        if (occ <= max_resident) break;
        smem += 2048;
        if (smem > max_optin) return cudaErrorInvalidConfiguration;
    }
    if (dev >= 0 && dev < 64) cached[dev] = smem;
    *out = smem;
    return cudaSuccess;
}

template <int BITS, int BNT>
static cudaError_t launch_cfg(const TcParams& prm, int64_t M, int ksplit, int nmat,
                              cudaStream_t s) {
    constexpr int SS = ring_stages(BITS, BNT);
    using Cfg = TcCfg<BITS, BNT, SS, kGroups>;
    auto kern = tc_wq_kernel<BITS, BNT, SS, kGroups>;
    int smem = 0;
    cudaError_t e = resident_safe_smem<BITS, BNT, SS, kGroups>(&smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(ksplit), static_cast<unsigned>(nmat * prm.n_tiles),
                       static_cast<unsigned>((M + BNT - 1) / BNT));
    cfg.blockDim = dim3(Cfg::kThreads, 1, 1);
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    cfg.stream = s;
    cudaLaunchAttribute attrs[2];
    int na = 0;
    attrs[na].id = cudaLaunchAttributeClusterDimension;
    attrs[na].val.clusterDim.x = static_cast<unsigned>(ksplit);
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

template <int BITS>
static cudaError_t launch_bits(const TcParams& prm, int64_t M, const TcChoice& c, int nmat,
                               cudaStream_t s) {
    switch (c.bnt) {
        case 16: return launch_cfg<BITS, 16>(prm, M, c.ksplit, nmat, s);
        case 32: return launch_cfg<BITS, 32>(prm, M, c.ksplit, nmat, s);
        case 64: return launch_cfg<BITS, 64>(prm, M, c.ksplit, nmat, s);
        case 128: return launch_cfg<BITS, 128>(prm, M, c.ksplit, nmat, s);
        default: return launch_cfg<BITS, 256>(prm, M, c.ksplit, nmat, s);
    }
}

cudaError_t launch_tc_product(const uint16_t* x, int64_t M, int64_t K, int64_t N, int bits,
                              const WOperand* w, int nmat, cudaStream_t s) {
    const TcChoice c = choose(M, N, K, nmat);
    TcParams prm;
    memset(&prm, 0, sizeof(prm));
    if (!make_tmap_2d(&prm.tm_x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, x, static_cast<uint64_t>(K),
                      static_cast<uint64_t>(M), static_cast<uint64_t>(K) * 2, kKB,
                      static_cast<uint32_t>(c.bnt), CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
    const uint64_t row_bytes = static_cast<uint64_t>(K) * bits / 8;
    const uint32_t box_bytes = kKB * bits / 8;
    for (int i = 0; i < nmat; ++i) {
        if (!make_tmap_2d(&prm.tm_w[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, w[i].codes, row_bytes,
                          static_cast<uint64_t>(N), row_bytes, box_bytes, kRows,
                          bits == 4 ? CU_TENSOR_MAP_SWIZZLE_32B : CU_TENSOR_MAP_SWIZZLE_64B))
            return cudaErrorInvalidValue;
        prm.scales[i] = w[i].scales;
        prm.y[i] = w[i].y;
    }
    prm.M = static_cast<int>(M);
    prm.N = static_cast<int>(N);
    prm.K = static_cast<int>(K);
    prm.n_tiles = static_cast<int>((N + kRows - 1) / kRows);
    prm.kblocks = static_cast<int>(K / kGroup);
    prm.status = device_status_ptr();
    prm.timeout_ns = wait_limit_ns();
    return bits == 4 ? launch_bits<4>(prm, M, c, nmat, s) : launch_bits<8>(prm, M, c, nmat, s);
}

// ------------------------------------------------ bounded-wait self test --
// Waits on an mbarrier that nothing ever completes; the bounded wait must
// give up, raise RQ_ERR_TIMEOUT in the status word and let the kernel exit.
__global__ void wait_selftest_kernel(int* status, uint64_t limit_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, limit_ns, status);
    __syncthreads();
}

cudaError_t launch_wait_selftest(uint64_t limit_ns, cudaStream_t s) {
    wait_selftest_kernel<<<1, 32, 0, s>>>(device_status_ptr(), limit_ns);
    return cudaGetLastError();
}

}  // namespace rq
