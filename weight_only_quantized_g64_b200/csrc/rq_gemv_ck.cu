// rq_gemv_ck.cu -- decode product (1 <= M <= 32) with K split over the CTAs
// of a thread-block cluster.
//
//   y[m, n] = sum_g s16[n, g] * sum_{k in g} x[m, k] * code[n, k]
//
// The same product as rq_gemv.cu (the "Hakureirm/rwkv7-sglang-w4gptq-1.5b"
// model card's small-M int4 kernel streaming the g64 codes; the fused R/K/V
// launch of the "RWKV-7 Quantization Toolkit" "Key Design"), decomposed for
// batches where the activations are no longer small next to the weights.
//
// Decomposition.  A row block is R = 128 or 64 consecutive rows of one
// matrix (the NMAT matrices of a fused call are stacked).  Each row block
// belongs to one cluster of C CTAs (C = 1: no split); CTA rank c of the
// cluster takes the 128-byte code stages [c*S/C, (c+1)*S/C) of every row (S
// stages per row), so the cluster splits K and one row block's codes are
// read exactly once.  The host picks (R, C) per launch from an estimate of
// the per-CTA streaming and MMA time, the waves and the reduction bytes, and
// keeps one CTA per SM.
//
// Data path.  A piece is ks <= 2 stages of the row block: their codes (one
// 3D TMA box), scales (one box) and the x of their groups for all M tokens
// (one 3D box), in one ring slot on one mbarrier.  Thread 0 issues the codes
// and scales of the first slots before the kernel waits on the previous grid
// (they never depend on it), x after; later pieces are issued by the warp
// whose turn it is once every warp has released the slot.  Eight warps, all
// computing, split the row block into WR = 8 / WK row strips of 16 * MTW
// rows; WK > 1 k-warps split each stage's groups (or, with more k-warps than
// a stage has groups, take whole groups of a piece); a warp keeps MTW
// m-tiles, so every x fragment it loads serves MTW * 16 rows.
//
// Reduction.  Each warp leaves its fp32 sums in shared memory; the CTA adds
// its k-warps' sums row by row.  With C = 1 it stores y from there.
// Otherwise the sum of row r goes, by plain distributed-shared-memory stores,
// to the CTA of the cluster that owns r (rows [c*share, (c+1)*share) belong
// to rank c); one release/acquire cluster barrier makes the stores visible;
// each rank adds the C sums of its rows in rank order and stores y.  Every
// addition has a fixed order, so results are deterministic; nothing goes
// through global memory but x, codes, scales and y, and no counters or
// workspace are needed.
//
// Inner math (rq_gemv_unit.cuh): codes become exact fp16 values in registers
// (Kim et al., arXiv:2211.10017), mma.sync.m16n8k16 sums x * code of one
// group in fp32, the group's fp16 scale is applied in fp32.
#include "rq_internal.h"
#include "rq_ptx.cuh"
#include "rq_gemv_unit.cuh"

#include <algorithm>
#include <cstring>

namespace rq {

// NW warps, all computing; loads are issued by single lanes between their
// math.  With eight warps (two per SM sub-partition) a thread may use up to
// 255 registers.
constexpr int kCkMaxSlots = 8;
constexpr int kCkMaxCluster = 8;
constexpr int kCkSRow = 16;                              // staged scale row: 16 fp16 (32 B)
constexpr int kCkMaxKs = 2;                              // stages per piece: ks * GPS + 7 <= 16

struct CkParams {
    CUtensorMap tm_w[3];  // codes: 3D {128 B, N, S} box {128, R, ks}, or 2D {row bytes, N} box {128, R}
    CUtensorMap tm_s[3];  // scales [N, K/64] fp16, box {16 groups, R} (when ssc)
    CUtensorMap tm_x;     // x [M, K] fp16 as 3D {64, M, K/64}, box {64, M, ks*GPS}, SWIZZLE_128B
    const uint16_t* scales[3];
    float* y[3];
    int M, N, K, groups;
    int S;                // 128-byte code stages per row
    int C;                // CTAs per cluster, along K
    int rbpm;             // row blocks per matrix: ceil(N / R)
    int ks;               // stages per piece
    int nslot;            // ring slots
    int slot_bytes;       // codes [ks][R][128 B] (swizzled), scales [R][16] fp16, x [ks*GPS][M][128 B]
    int s_off, x_off;     // offsets of the scales and x within a slot
    int recv_off;         // received row sums [C][share][MP] fp32 (16-byte aligned)
    int bar_off;
    int share;            // rows of the row block each rank sums and stores (multiple of 4)
    int mp;               // token pitch of the sums: a multiple of 8 plus 4, >= M + 4
    int ssc;              // scales staged by TMA (scale rows a multiple of 16 bytes)
    int* status;
    uint64_t timeout_ns;
};

struct CkBars {
    uint64_t full[kCkMaxSlots];    // piece landed (codes, scales, x)
    uint64_t empty[kCkMaxSlots];   // every warp is done with the slot
    int issued_hi[kCkMaxSlots];    // last piece issued into each slot
    int abort;
};

// NW warps; WK of them along k (groups of a stage dealt round-robin); WR =
// NW / WK row strips of MTW m-tiles.  R = WR * 16 * MTW rows per row block.
template <int BITS, int MTW, int NT, int WK, int NW>
struct CkCfg {
    static constexpr int kThreads = NW * 32;
    static constexpr int kWR = NW / WK;
    static constexpr int kR = kWR * 16 * MTW;
    static constexpr int kGPS = BITS == 4 ? 4 : 2;
    static constexpr int kKPS = BITS == 4 ? 256 : 128;    // k per 128-byte stage
    static constexpr int kCStage = kR * 128;               // code bytes per stage
    static_assert(kR == 64 || kR == 128, "row blocks of 64 or 128 rows");
    static_assert(kGPS % WK == 0 || WK % kGPS == 0, "k-warps split a stage's groups evenly, or "
                                                    "take whole groups of a piece");
    static_assert(kCkMaxKs * kGPS + 7 <= kCkSRow, "scale box holds a piece's groups");
};

template <int BITS, int MTW, int NT, int WK, int NW>
__global__ void __launch_bounds__(NW * 32, 1)
    gemv_ck_kernel(const __grid_constant__ CkParams p) {
    using Cfg = CkCfg<BITS, MTW, NT, WK, NW>;
    constexpr int kCkWarps = NW;
    constexpr int kCkThreads = Cfg::kThreads;
    constexpr int R = Cfg::kR;
    constexpr int GPS = Cfg::kGPS;
    constexpr int MT = MTW;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint8_t* ring = smem;
    float* recv = reinterpret_cast<float*>(smem + p.recv_off);
    CkBars* bars = reinterpret_cast<CkBars*>(smem + p.bar_off);
    volatile int* abort_flag = &bars->abort;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int C = p.C;
    const int rank = static_cast<int>(cluster_ctarank());
    const int rb = static_cast<int>(blockIdx.x) / C;       // row block of the cluster
    const int mat = rb / p.rbpm;
    const int row0 = (rb - mat * p.rbpm) * R;              // first row within the matrix
    const int s0 = rank * p.S / C;
    const int s1 = (rank + 1) * p.S / C;
    const int npieces = (s1 - s0 + p.ks - 1) / p.ks;
    const int M = p.M;
    const int NS = p.nslot;
    const int share = p.share;
    const int MP = p.mp;
    const int r_lo = rank * share;                         // rows this CTA sums and stores
    const int r_hi = min(R, r_lo + share);

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&bars->full[s], 1);
            mbar_init(&bars->empty[s], kCkWarps);
            bars->issued_hi[s] = -1;
        }
        bars->abort = 0;
        fence_mbar_init();
        tma_prefetch_desc(&p.tm_x);
        tma_prefetch_desc(&p.tm_w[mat]);
        if (p.ssc) tma_prefetch_desc(&p.tm_s[mat]);
    }
    __syncthreads();
    pdl_launch_dependents();

    // Loads: a piece is ks stages of the row block's codes, their scales and
    // the x of their groups, in one ring slot on one barrier.  Thread 0
    // issues the codes and scales of the first NS pieces (they do not depend
    // on the previous grid), waits on the previous grid, then issues their x.
    // Piece i + NS refills slot i % NS; warp i % 8 issues it once every warp
    // has released piece i.
    const uint64_t pol_w = l2_policy_evict_first();
    const uint64_t pol_x = l2_policy_evict_last();
    const uint32_t x_bytes = static_cast<uint32_t>(p.ks * GPS * M * 128);
    const uint32_t piece_bytes = static_cast<uint32_t>(p.ks * Cfg::kCStage) +
                                 (p.ssc ? static_cast<uint32_t>(R * kCkSRow * 2) : 0u) + x_bytes;
    auto issue_w = [&](int i, int slot) {
        const int st = s0 + i * p.ks;
        uint8_t* dst = ring + slot * p.slot_bytes;
        bars->issued_hi[slot] = i;
        mbar_arrive_expect_tx(&bars->full[slot], piece_bytes);
        if (p.ks > 1)
            tma_load_3d(dst, &p.tm_w[mat], &bars->full[slot], 0, row0, st, pol_w);
        else
            tma_load_2d(dst, &p.tm_w[mat], &bars->full[slot], st * 128, row0, pol_w);
        if (p.ssc)
            tma_load_2d(dst + p.s_off, &p.tm_s[mat], &bars->full[slot], (st * GPS) & ~7, row0,
                        pol_w);
    };
    auto issue_x = [&](int i, int slot) {
        tma_load_3d(ring + slot * p.slot_bytes + p.x_off, &p.tm_x, &bars->full[slot], 0, 0,
                    (s0 + i * p.ks) * GPS, pol_x);
    };
    if (threadIdx.x == 0) {
        const int n0 = NS < npieces ? NS : npieces;
        for (int i = 0; i < n0; ++i) issue_w(i, i);
        pdl_wait();   // x may be written by the previous kernel
        for (int i = 0; i < n0; ++i) issue_x(i, i);
    }

    // ===================================================== the products ==
    const int kw = warp % WK;
    const int rw = warp / WK;
    const int g = lane >> 2;
    const int t = lane & 3;
    const int prow = phys_row<BITS>(g);
    const int wrow = rw * 16 * MT;                      // the warp's first row in the block
    float acc[MT][NT][4];
#pragma unroll
    for (int i = 0; i < MT; ++i)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[i][nt][e] = 0.0f;
    {
        int xtok[NT];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) xtok[nt] = min(nt * 8 + g, M - 1);
        bool dead = false;
        for (int i = 0; i < npieces; ++i) {
            const int slot = i % NS;
            if (!dead && !mbar_wait_suspend(&bars->full[slot], static_cast<uint32_t>(i / NS) & 1,
                                            abort_flag, p.timeout_ns, p.status))
                dead = true;
            if (!dead) {
                const int st = s0 + i * p.ks;
                const int n = min(p.ks, s1 - st);
                const uint8_t* base = ring + slot * p.slot_bytes;
                if constexpr (WK > GPS) {
                    // more k-warps than groups in a stage: warp kw takes groups
                    // kw, kw + WK, ... of the piece, one at a time
                    for (int gi = kw; gi < n * GPS; gi += WK) {
                        const int j = gi / GPS;
                        const uint8_t* wt = base + j * Cfg::kCStage + wrow * 128;
                        const uint8_t* sc =
                            base + p.s_off + (wrow * kCkSRow + ((st * GPS) & 7) + j * GPS) * 2;
                        gv_unit_strided<BITS, MT, NT, GPS, kCkSRow>(
                            wt, sc, base + p.x_off, j * GPS, gi - j * GPS, M, xtok, prow, t,
                            p.ssc != 0, p.scales[mat], row0 + wrow, st + j, p.N, p.groups, acc);
                    }
                } else
                for (int j = 0; j < n; ++j) {
                    const uint8_t* wt = base + j * Cfg::kCStage + wrow * 128;
                    const uint8_t* sc =
                        base + p.s_off + (wrow * kCkSRow + ((st * GPS) & 7) + j * GPS) * 2;
                    if constexpr (WK == 1)
                        gv_unit<BITS, MT, NT, MT, kCkSRow, 0>(
                            wt, 0, sc, base + p.x_off, j * GPS, M, xtok, prow, t, p.ssc != 0,
                            &p.scales[mat], row0 + wrow, st + j, p.N, p.groups, acc);
                    else
                        gv_unit_strided<BITS, MT, NT, WK, kCkSRow>(
                            wt, sc, base + p.x_off, j * GPS, kw, M, xtok, prow, t, p.ssc != 0,
                            p.scales[mat], row0 + wrow, st + j, p.N, p.groups, acc);
                }
            }
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bars->empty[slot]);
                // refill the slot with piece i + NS once every warp is done with it
                if (i + NS < npieces && warp == i % kCkWarps && !dead) {
                    if (mbar_wait_suspend(&bars->empty[slot], static_cast<uint32_t>(i / NS) & 1,
                                          abort_flag, p.timeout_ns, p.status)) {
                        issue_w(i + NS, i % NS);
                        issue_x(i + NS, i % NS);
                    }
                }
            }
            __syncwarp();
        }
    }

    // ============================================== cluster reduction ==
    // The warps' sums go to shared memory as [k-warp][row][token] (in the
    // ring, idle by now); the k-warps of each row are added here, and the sum
    // of row r is stored into recv[this rank][r - owner*share] of the rank
    // that owns r (r / share) with plain distributed-shared-memory stores.  A
    // release/acquire cluster barrier then makes every rank's stores visible,
    // and each rank adds the C ranks' sums of its rows in rank order.
    float* part = reinterpret_cast<float*>(ring);
    __syncthreads();   // every warp is done with the ring
#pragma unroll
    for (int i = 0; i < MT; ++i)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float* dst = part + (kw * R + wrow + 16 * i + 8 * h + prow) * MP;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int tok = nt * 8 + 2 * t;
                if (tok < MP)
                    *reinterpret_cast<float2*>(dst + tok) =
                        make_float2(acc[i][nt][2 * h], acc[i][nt][2 * h + 1]);
            }
        }
    __syncthreads();
    if (C == 1) {
        // no K split: add the k-warps' sums and store y; a warp's lanes take
        // consecutive rows, so each token's stores coalesce
        pdl_wait();   // y may be read by the previous kernel
        if (*abort_flag == 0) {
            const int nq = (M + 3) / 4;
            float* y = p.y[mat];
            for (int o = threadIdx.x; o < R * nq; o += kCkThreads) {
                const int q = o / R;
                const int row = o - q * R;
                float4 v = *reinterpret_cast<const float4*>(part + row * MP + 4 * q);
#pragma unroll
                for (int k2 = 1; k2 < WK; ++k2) {
                    const float4 u = *reinterpret_cast<const float4*>(part + (k2 * R + row) * MP + 4 * q);
                    v.x += u.x;
                    v.y += u.y;
                    v.z += u.z;
                    v.w += u.w;
                }
                const int n = row0 + row;
                if (n < p.N) {
                    const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        if (4 * q + e < M) y[static_cast<int64_t>(4 * q + e) * p.N + n] = vv[e];
                }
            }
        }
    } else {
    {
        const int nq = (M + 3) / 4;
        const uint32_t recv_s = smem_u32(recv) + static_cast<uint32_t>(rank * share * MP * 4);
        for (int o = threadIdx.x; o < R * nq; o += kCkThreads) {
            const int row = o / nq;
            const int q = o - row * nq;
            float4 v = *reinterpret_cast<const float4*>(part + row * MP + 4 * q);
#pragma unroll
            for (int k2 = 1; k2 < WK; ++k2) {
                const float4 u = *reinterpret_cast<const float4*>(part + (k2 * R + row) * MP + 4 * q);
                v.x += u.x;
                v.y += u.y;
                v.z += u.z;
                v.w += u.w;
            }
            const int owner = row / share;
            st_dsmem_f32x4(map_to_rank(recv_s + static_cast<uint32_t>(((row - owner * share) * MP + 4 * q) * 4),
                                       static_cast<uint32_t>(owner)),
                           v);
        }
    }
    cluster_sync();   // every rank's sums are in place
    pdl_wait();       // y may be read by the previous kernel
    if (*abort_flag == 0) {
        // per (row, 4 tokens), rank order; a warp's lanes take consecutive
        // rows, so each token's stores coalesce
        const int nr = r_hi - r_lo;
        const int nq = (M + 3) / 4;
        float* y = p.y[mat];
        for (int o = threadIdx.x; o < nr * nq; o += kCkThreads) {
            const int q = o / nr;
            const int rl = o - q * nr;
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int c = 0; c < C; ++c) {
                const float4 u = *reinterpret_cast<const float4*>(recv + (c * share + rl) * MP + 4 * q);
                v.x += u.x;
                v.y += u.y;
                v.z += u.z;
                v.w += u.w;
            }
            const int n = row0 + r_lo + rl;
            if (n < p.N) {
                const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    if (4 * q + e < M) y[static_cast<int64_t>(4 * q + e) * p.N + n] = vv[e];
            }
        }
    }
    }   // C > 1
    // After a timeout some copies may still be in flight: wait (bounded) for
    // the last piece of every slot, so nothing lands after the CTA exits.
    if (threadIdx.x == 0 && *abort_flag) {
        int dummy_abort = 0;
        for (int s = 0; s < NS; ++s) {
            const int il = bars->issued_hi[s];
            if (il >= 0)
                mbar_wait(&bars->full[s], static_cast<uint32_t>(il / NS) & 1, &dummy_abort,
                          p.timeout_ns, p.status);
        }
    }
}

// ------------------------------------------------------------- launcher --


constexpr int kCkSmemMax = 227 * 1024;
constexpr int kCkSmemOneCta = 120 * 1024;   // more than half an SM's shared memory

static int ck_align(int v, int a) { return (v + a - 1) / a * a; }

struct CkPlan {
    int C, ks, nslot, slot_bytes, s_off, x_off, recv_off, bar_off, share, mp, smem, grid;
    double est;
};

// Shared-memory layout for a cluster size: ring slots (codes, scales and x of
// a piece), the received partial sums, the barriers.
template <int BITS, int MTW, int NT, int WK, int NW>
static bool ck_layout(int M, int S, int C, bool three_d, CkPlan* L) {
    using Cfg = CkCfg<BITS, MTW, NT, WK, NW>;
    const int sc_max = (S + C - 1) / C;                    // stages of the busiest rank
    L->C = C;
    L->ks = three_d ? (sc_max < kCkMaxKs ? sc_max : kCkMaxKs) : 1;
    const int pieces = (sc_max + L->ks - 1) / L->ks;
    L->s_off = L->ks * Cfg::kCStage;
    L->x_off = ck_align(L->s_off + Cfg::kR * kCkSRow * 2, 1024);   // swizzled x box: 1024-aligned
    L->slot_bytes = ck_align(L->x_off + L->ks * Cfg::kGPS * M * 128, 1024);
    L->share = ck_align((Cfg::kR + C - 1) / C, 4);
    L->mp = (M + 7) / 8 * 8 + 4;   // 4 (mod 8): float4 rows of 8 lanes hit distinct banks
    const int recv_bytes = C * L->share * L->mp * 4;
    const int part_bytes = WK * Cfg::kR * L->mp * 4;       // the warps' sums, in the ring
    for (int ns = pieces < kCkMaxSlots ? pieces : kCkMaxSlots; ns >= 1; --ns) {
        L->nslot = ns;
        // the ring also holds the warps' sums at the end
        const int ring = ns * L->slot_bytes > part_bytes ? ns * L->slot_bytes : ck_align(part_bytes, 1024);
        L->recv_off = ring;
        L->bar_off = ck_align(L->recv_off + recv_bytes, 16);
        L->smem = 1024 + L->bar_off + static_cast<int>(sizeof(CkBars));
        // one CTA per SM: two CTAs of one launch on an SM (which the block
        // scheduler does when it can) finish last and hold the launch back
        if (L->smem < kCkSmemOneCta) L->smem = kCkSmemOneCta;
        if (L->smem <= kCkSmemMax && (ns >= 2 || pieces == 1)) return true;
    }
    return false;
}

// Clusters of C CTAs with this shared memory that fit on the GPU at once.
template <int BITS, int MTW, int NT, int WK, int NW>
static int ck_max_clusters(int C, int smem) {
    static int cache[kCkMaxCluster + 1][64] = {};
    const int sb = smem / 4096;
    if (sb < 64 && cache[C][sb] > 0) return cache[C][sb];
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(C), 1, 1);
    cfg.blockDim = dim3(NW * 32, 1, 1);
    cfg.dynamicSmemBytes = static_cast<size_t>((sb + 1) * 4096 < kCkSmemMax ? (sb + 1) * 4096 : kCkSmemMax);
    cudaLaunchAttribute a;
    a.id = cudaLaunchAttributeClusterDimension;
    a.val.clusterDim.x = static_cast<unsigned>(C);
    a.val.clusterDim.y = 1;
    a.val.clusterDim.z = 1;
    cfg.attrs = &a;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, gemv_ck_kernel<BITS, MTW, NT, WK, NW>, &cfg) != cudaSuccess ||
        n <= 0) {
        cudaGetLastError();
        n = num_sms() / C;
    }
    if (sb < 64) cache[C][sb] = n;
    return n;
}

// Cluster size: the estimated time of one launch, over C = 1..8.  A CTA
// streams its codes at about the HBM rate divided by the SMs (~40 GB/s on
// B200: one CTA cannot pull much more, however few run) and does its MMA work
// at about half of the 1024 MAC per cycle and SM; waves add up, each with a
// fixed latency; a cluster's reduction costs a barrier and its bytes.  So the estimate favours enough
// CTAs to cover the SMs with the least work each, and no K split when that
// is possible.
template <int BITS, int MTW, int NT, int WK, int NW>
static bool ck_choose(int M, int N, int S, int nmat, bool three_d, CkPlan* best) {
    using Cfg = CkCfg<BITS, MTW, NT, WK, NW>;
    const int rbt = nmat * ((N + Cfg::kR - 1) / Cfg::kR);
    bool found = false;
    for (int C = 1; C <= kCkMaxCluster && C <= S; ++C) {
        CkPlan L;
        if (!ck_layout<BITS, MTW, NT, WK, NW>(M, S, C, three_d, &L)) continue;
        const int sc_max = (S + C - 1) / C;
        const int64_t ctas = static_cast<int64_t>(rbt) * C;
        const int64_t cap = static_cast<int64_t>(ck_max_clusters<BITS, MTW, NT, WK, NW>(C, L.smem)) * C;
        const int64_t waves = (ctas + cap - 1) / cap;
        const double bytes = static_cast<double>(Cfg::kR) * sc_max * (128 + 2 * Cfg::kGPS);
        const double macs = static_cast<double>(Cfg::kR) * sc_max * Cfg::kKPS * NT * 8;
        const double t_cta = bytes / 40e9 + macs / (512.0 * 1.8e9);
        // a cluster's reduction: a barrier plus R x MP sums per CTA through
        // distributed shared memory (tens of GB/s per SM)
        const double t_red = C > 1 ? 0.3e-6 + static_cast<double>(Cfg::kR) * L.mp * 4 / 20e9 : 0.0;
        // every wave also pays the latency of a CTA's start, first loads,
        // barriers and exit (about 1.5 us measured)
        const double est = static_cast<double>(waves) * (t_cta + 1.5e-6) + t_red;
        if (!found || est < best->est * 0.98) {
            L.est = est;
            L.grid = static_cast<int>(ctas);
            *best = L;
            found = true;
        }
    }
    return found;
}

// The best plan of one configuration for this product (false: none fits).
template <int BITS, int MTW, int NT, int WK, int NW>
static bool ck_plan(const CkParams& prm, int nmat, CkPlan* L, cudaError_t* err) {
    auto kern = gemv_ck_kernel<BITS, MTW, NT, WK, NW>;
    static bool attr_set[64] = {};
    int dev = 0;
    *err = cudaGetDevice(&dev);
    if (*err != cudaSuccess) return false;
    if (dev < 0 || dev >= 64) {
        *err = cudaErrorInvalidDevice;
        return false;
    }
    if (!attr_set[dev]) {
        // (before the occupancy query, which checks it)
        *err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kCkSmemMax);
        if (*err != cudaSuccess) return false;
        attr_set[dev] = true;
    }
    const int64_t row_bytes = static_cast<int64_t>(prm.K) * BITS / 8;
    const int S = static_cast<int>((row_bytes + 127) / 128);
    // the 3D code view needs rows of whole 128-byte stages
    return ck_choose<BITS, MTW, NT, WK, NW>(prm.M, prm.N, S, nmat, row_bytes % 128 == 0, L);
}

template <int BITS, int MTW, int NT, int WK, int NW>
static cudaError_t ck_launch(CkParams& prm, const uint16_t* x, const void* const* codes, int nmat,
                             cudaStream_t s, const CkPlan& L) {
    using Cfg = CkCfg<BITS, MTW, NT, WK, NW>;
    auto kern = gemv_ck_kernel<BITS, MTW, NT, WK, NW>;
    const int64_t row_bytes = static_cast<int64_t>(prm.K) * BITS / 8;
    prm.S = static_cast<int>((row_bytes + 127) / 128);
    prm.C = L.C;
    prm.rbpm = (prm.N + Cfg::kR - 1) / Cfg::kR;
    prm.ks = L.ks;
    prm.nslot = L.nslot;
    prm.slot_bytes = L.slot_bytes;
    prm.s_off = L.s_off;
    prm.x_off = L.x_off;
    prm.recv_off = L.recv_off;
    prm.bar_off = L.bar_off;
    prm.share = L.share;
    prm.mp = L.mp;
    prm.ssc = (prm.groups * 2) % 16 == 0 ? 1 : 0;

    // The kernel loads a piece with a 3D box when ks > 1 and a 2D box
    // otherwise; the map's rank must match the load's.
    const bool map3d = prm.ks > 1;
    for (int i = 0; i < nmat; ++i) {
        const bool okw =
            map3d ? make_tmap_3d(&prm.tm_w[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, codes[i], 128,
                                   static_cast<uint64_t>(prm.N), static_cast<uint64_t>(prm.S),
                                   static_cast<uint64_t>(row_bytes), 128, 128, Cfg::kR,
                                   static_cast<uint32_t>(prm.ks), CU_TENSOR_MAP_SWIZZLE_128B)
                    : make_tmap_2d(&prm.tm_w[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, codes[i],
                                   static_cast<uint64_t>(row_bytes), static_cast<uint64_t>(prm.N),
                                   static_cast<uint64_t>(row_bytes), 128, Cfg::kR,
                                   CU_TENSOR_MAP_SWIZZLE_128B);
        if (!okw) return cudaErrorInvalidValue;
        if (prm.ssc &&
            !make_tmap_2d(&prm.tm_s[i], CU_TENSOR_MAP_DATA_TYPE_UINT16, prm.scales[i],
                          static_cast<uint64_t>(prm.groups), static_cast<uint64_t>(prm.N),
                          static_cast<uint64_t>(prm.groups) * 2, kCkSRow, Cfg::kR,
                          CU_TENSOR_MAP_SWIZZLE_NONE))
            return cudaErrorInvalidValue;
    }
    if (!make_tmap_3d(&prm.tm_x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, x, 64, static_cast<uint64_t>(prm.M),
                      static_cast<uint64_t>(prm.groups), static_cast<uint64_t>(prm.K) * 2, 128, 64,
                      static_cast<uint32_t>(prm.M), static_cast<uint32_t>(prm.ks * Cfg::kGPS),
                      CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(L.grid), 1, 1);
    cfg.blockDim = dim3(Cfg::kThreads, 1, 1);
    cfg.dynamicSmemBytes = static_cast<size_t>(L.smem);
    cfg.stream = s;
    cudaLaunchAttribute attrs[3];
    int na = 0;
    attrs[na].id = cudaLaunchAttributeClusterDimension;
    attrs[na].val.clusterDim.x = static_cast<unsigned>(L.C);
    attrs[na].val.clusterDim.y = 1;
    attrs[na].val.clusterDim.z = 1;
    ++na;
    // spread a launch's clusters over the GPCs
    attrs[na].id = cudaLaunchAttributeClusterSchedulingPolicyPreference;
    attrs[na].val.clusterSchedulingPolicyPreference = cudaClusterSchedulingPolicySpread;
    ++na;
    if (pdl_enabled()) {
        attrs[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attrs[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    cfg.attrs = attrs;
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<const CkParams&>(prm));
}

// Warp split by batch (eight warps; sixteen measured no faster), for row
// blocks of 128 or 64 rows: M <= 8 one m-tile per warp (64 rows: the stage's
// groups split 2 ways); M <= 16 two m-tiles, groups split 2 (4) ways; M <= 32
// (int4) four m-tiles, groups split 4 ways (64 rows: each warp takes whole
// groups of a piece, 8 ways), so each x fragment serves 64 rows; int8 stages
// hold two groups: two m-tiles, 2 (4) ways.  The plan with the lower
// estimate runs.
template <int BITS, int MTW, int NT, int WK, int MTW2, int WK2>
static cudaError_t ck_pick(CkParams& prm, const uint16_t* x, const void* const* codes, int nmat,
                           cudaStream_t s) {
    CkPlan a, b;
    cudaError_t ea = cudaSuccess, eb = cudaSuccess;
    const bool fa = ck_plan<BITS, MTW, NT, WK, 8>(prm, nmat, &a, &ea);
    const bool fb = ck_plan<BITS, MTW2, NT, WK2, 8>(prm, nmat, &b, &eb);
    if (ea != cudaSuccess) return ea;
    if (eb != cudaSuccess) return eb;
    if (fb && (!fa || b.est < a.est)) return ck_launch<BITS, MTW2, NT, WK2, 8>(prm, x, codes, nmat, s, b);
    if (fa) return ck_launch<BITS, MTW, NT, WK, 8>(prm, x, codes, nmat, s, a);
    return cudaErrorInvalidValue;
}

template <int BITS>
static cudaError_t ck_dispatch(CkParams& prm, const uint16_t* x, const void* const* codes,
                               int nmat, cudaStream_t s) {
    if (prm.M <= 8) return ck_pick<BITS, 1, 1, 1, 1, 2>(prm, x, codes, nmat, s);
    if (prm.M <= 16) return ck_pick<BITS, 2, 2, 2, 2, 4>(prm, x, codes, nmat, s);
    if constexpr (BITS == 4) return ck_pick<BITS, 4, 4, 4, 4, 8>(prm, x, codes, nmat, s);
    else return ck_pick<BITS, 2, 4, 2, 2, 4>(prm, x, codes, nmat, s);
}

template <int BITS, int MTW, int NT, int WK, int NW>
static bool ck_fits_cfg(int M, int K) {
    const int64_t row_bytes = static_cast<int64_t>(K) * BITS / 8;
    const int S = static_cast<int>((row_bytes + 127) / 128);
    CkPlan L;
    for (int C = 1; C <= kCkMaxCluster && C <= S; ++C)
        if (ck_layout<BITS, MTW, NT, WK, NW>(M, S, C, row_bytes % 128 == 0, &L)) return true;
    return false;
}

template <int BITS>
static bool ck_fits(int M, int K) {
    if (M <= 8) return ck_fits_cfg<BITS, 1, 1, 1, 8>(M, K) || ck_fits_cfg<BITS, 1, 1, 2, 8>(M, K);
    if (M <= 16) return ck_fits_cfg<BITS, 2, 2, 2, 8>(M, K) || ck_fits_cfg<BITS, 2, 2, 4, 8>(M, K);
    if constexpr (BITS == 4)
        return ck_fits_cfg<BITS, 4, 4, 4, 8>(M, K) || ck_fits_cfg<BITS, 4, 4, 8, 8>(M, K);
    else return ck_fits_cfg<BITS, 2, 4, 2, 8>(M, K) || ck_fits_cfg<BITS, 2, 4, 4, 8>(M, K);
}

bool gemv_cluster_fits(int64_t M, int64_t K, int bits) {
    if (M < 1 || M > RQ_MAX_DECODE_M || K > (int64_t{1} << 30)) return false;
    return bits == 4 ? ck_fits<4>(static_cast<int>(M), static_cast<int>(K))
                     : ck_fits<8>(static_cast<int>(M), static_cast<int>(K));
}

cudaError_t launch_gemv_cluster(const uint16_t* x, int64_t M, int64_t K, int64_t N, int bits,
                                const WOperand* w, int nmat, cudaStream_t s) {
    CkParams prm;
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
    return bits == 4 ? ck_dispatch<4>(prm, x, codes, nmat, s) : ck_dispatch<8>(prm, x, codes, nmat, s);
}

}  // namespace rq
