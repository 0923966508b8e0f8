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
// Work decomposition.  A row tile is RBM = WR * 16 * MTW consecutive rows of
// each of the NMAT matrices (NMAT = 3 for the fused R/K/V call, whose
// matrices share x).  A unit is one row tile times one 128-byte column stage
// of codes (int4: 256 k = 4 groups; int8: 128 k = 2 groups).  The units,
// tile-major, are cut into equal contiguous runs, one per CTA (stream-K), or
// whole tiles are dealt one run per CTA when they balance over the SMs.  A
// CTA walks its run as load groups: up to ks consecutive stages of one row
// tile.  The 8 compute warps split a group WK ways along k (warp w takes
// stage w % WK) and 8 / WK ways along rows; the k-split warps' partial sums
// are added in shared memory, in warp order, by a reduction warp.  A tile
// shared by several CTAs is stored as pieces in a global workspace and
// summed, in a fixed CTA order, by whichever contributor arrives last (an
// atomic counter per tile), so results stay deterministic.
//
// Data path: a producer warp fills a ring of 2..8 load-group slots, each
// holding the group's codes (one 3D TMA box per matrix: ks stages x RBM
// rows, 128-byte swizzled), its scales (one box per matrix) and its x (one
// 3D box of the group's 64-k groups x M tokens).  Codes and scales of the
// first slots are requested before the kernel waits on the previous grid;
// x after.  Compute warps release a slot with an mbarrier arrive and the
// producer refills it.
// Thread (g = lane/4, t = lane%4) owns, per group of 64 k, the 16 k
// [16t, 16t+16) of rows g and g+8 of each m-tile: MMA k-slot sigma of step j
// maps to one of those k, the same map on the A (weights) and B (x) side, so
// the sum over k is unchanged and every thread's codes and x are contiguous in
// memory.  Codes become exact fp16 values in registers (bit placement plus
// one exact fp16 operation: Kim et al., arXiv:2211.10017); the MMA sums
// x * code for one group in fp32 registers; the group's scale is applied in
// fp32 (acc = fma(partial, s, acc)).  Nothing dequantised is stored.
#include "rq_internal.h"
#include "rq_ptx.cuh"
#include "rq_gemv_unit.cuh"

namespace rq {

struct GvParams {
    CUtensorMap tm_w[3];  // codes [N, K*bits/8] u8; ks > 1: 3D {128 B, N rows, stages}, box
                          // {128, RBM, ks}; ks == 1: 2D {row bytes, N}, box {128, RBM}; SWIZZLE_128B
    CUtensorMap tm_s[3];  // scales [N, K/64] fp16: box {SROW groups, RBM}, no swizzle (when ssc)
    CUtensorMap tm_x;     // x [M, K] fp16 as 3D {64, M tokens, K/64 groups}: box {64, M, ks*GPS}, SWIZZLE_128B
    const uint16_t* scales[3];
    float* y[3];
    int M, N, K;
    int groups;           // K / 64
    int tiles;            // row tiles (RBM rows of every matrix)
    int kstages;          // 128-byte code stages per row: ceil(K * bits / 8 / 128)
    int units;            // tiles * kstages
    int chunk;            // units are dealt in chunks: kstages (whole tiles) or 1 (stream-K)
    int uq, ur;           // chunks / gridDim.x and chunks % gridDim.x: CTA c owns chunks
                          // [c*uq + min(c, ur), (c+1)*uq + min(c+1, ur))
    int ks;               // stages per load group: WK, or 1 when rows are not whole stages
    int sg;               // ring depth in load groups (2..8)
    int slot_bytes;       // bytes per ring slot: codes, then scales, then x
    int s_off, x_off;     // offsets of the scales and x within a slot
    int red_off;          // offset of the reduction buffers
    int red_nbuf;         // reduction buffers (1 or 2)
    int bar_off;          // offset of the barriers
    int ssc;              // scales staged by TMA with the codes (rows a multiple of 16 bytes)
    float* ws;            // partial-tile slots: [2 * gridDim.x][M][RB] fp32
    int* cnt;             // per-tile arrival counters, zero between launches
    int* status;
    uint64_t timeout_ns;
};

constexpr int kGvConsumers = 8;                         // warps that multiply
constexpr int kGvProducer = kGvConsumers;               // warp that fills the ring
constexpr int kGvReducer = kGvConsumers + 1;            // warp that reduces and stores
constexpr int kGvThreads = (kGvConsumers + 2) * 32;
constexpr int kGvMaxSG = 8;                             // ring depth limit, in load groups

// BITS: 4 or 8.  NMAT: matrices sharing x (1, or 3 for fused R/K/V).  MTW:
// 16-row m-tiles per warp and matrix.  NT: 8-token n-tiles (M <= 8 NT).  WK:
// compute warps along k (8, 2 or 1); the other factor WR = 8 / WK splits the
// rows.  Warp w takes stage w % WK of each load group and rows block w / WK.
template <int BITS, int NMAT, int MTW, int NT, int WK>
struct GvCfg {
    static constexpr int kWR = kGvConsumers / WK;            // warps along rows
    static constexpr int kMT = NMAT * MTW;                   // m-tiles per warp
    static constexpr int kRBM = kWR * 16 * MTW;              // rows per matrix in a row tile
    static constexpr int kRB = NMAT * kRBM;                  // rows per row tile
    static constexpr int kKPS = BITS == 4 ? 256 : 128;       // k per stage (128 code bytes)
    static constexpr int kGPS = kKPS / 64;                   // groups per stage
    static constexpr int kTok = 8 * NT;
    // a load group: ks <= WK stages of a row tile, per matrix [ks][RBM rows][128 B]
    static constexpr int kCStage = kRBM * 128;               // code bytes per matrix and stage
    // scales: per matrix [RBM rows][SROW] fp16, SROW = the group's WK*GPS
    // groups plus 8 of slack (so the box can start at a 16-byte boundary),
    // rounded up to 16 bytes
    static constexpr int kSRow = (WK * kGPS + 8 + 7) / 8 * 8;
    static constexpr int kSMat = kRBM * kSRow * 2;
    static constexpr int kSGroup = NMAT * kSMat;
    static constexpr int kRedStride = kRB + 4;               // floats per token row (bank spread)
    static constexpr int kRedTok = kTok < 16 ? kTok : 16;    // tokens per reduction round
    static constexpr int kRedWarp = kRedTok * kRedStride;    // floats per k-warp deposit
    static constexpr int kRedBuf = WK * kRedWarp;            // floats per reduction buffer
    static_assert(kCStage % 1024 == 0, "group alignment");
    static_assert((kSRow * 2) % 16 == 0, "scale rows must be 16-byte multiples");
    static_assert(kSMat % 128 == 0, "TMA destinations must be 128-byte aligned");
};

// Barriers and flags after the buffers.
struct GvBars {
    uint64_t full[kGvMaxSG];   // ring slot holds its group's codes, scales and x
    uint64_t empty[kGvMaxSG];  // every compute warp is done with the slot
    uint64_t red_full[2];      // every warp has deposited its partial sums
    uint64_t red_free[2];      // the reducing warp has read the buffer
    int issued_hi[kGvMaxSG];   // last group issued into each slot
    int abort;
};

// First work chunk of CTA c: the first ur CTAs take uq + 1 chunks, the rest uq.
__device__ __forceinline__ int range_begin(int c, int uq, int ur) {
    return c * uq + (c < ur ? c : ur);
}

// The CTA whose unit range holds unit u (stream-K: chunks of one unit).
__device__ __forceinline__ int range_owner(int u, int uq, int ur) {
    const int big = ur * (uq + 1);
    return u < big ? u / (uq + 1) : ur + (u - big) / uq;
}

// Walks a CTA's units as load groups: up to ks consecutive stages of one row
// tile, never past the tile or the CTA's range.
struct GvWalk {
    int tile, st, left, ks;
    __device__ __forceinline__ int next(int S, int& g_tile, int& g_st) {   // returns the group's units
        int n = S - st;
        if (n > ks) n = ks;
        if (n > left) n = left;
        g_tile = tile;
        g_st = st;
        st += n;
        left -= n;
        if (st == S) {
            st = 0;
            ++tile;
        }
        return n;
    }
};

template <int BITS, int NMAT, int MTW, int NT, int WK>
__global__ void __launch_bounds__(kGvThreads, 1) gemv_wq_kernel(const __grid_constant__ GvParams p) {
    using Cfg = GvCfg<BITS, NMAT, MTW, NT, WK>;
    constexpr int MT = Cfg::kMT;
    constexpr int RBM = Cfg::kRBM;
    constexpr int RB = Cfg::kRB;
    constexpr int GPS = Cfg::kGPS;
    constexpr int RS = Cfg::kRedStride;
    constexpr int NW = kGvConsumers;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    const int SG = p.sg;
    const int cmat = p.ks * Cfg::kCStage;                   // code bytes per matrix and group
    // ring slot: codes [NMAT][ks][RBM][128 B] (swizzled), scales
    // [NMAT][RBM][SROW] fp16, x [ks*GPS groups][M][128 B] (swizzled)
    uint8_t* ring = smem;
    float* red = reinterpret_cast<float*>(smem + p.red_off);   // [red_nbuf][WK][kRedTok][RS]
    GvBars* bars = reinterpret_cast<GvBars*>(smem + p.bar_off);
    volatile int* abort_flag = &bars->abort;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int cta = static_cast<int>(blockIdx.x);
    const int S = p.kstages;
    const int M = p.M;
    const int u0 = range_begin(cta, p.uq, p.ur) * p.chunk;
    const int nu = (p.uq + (cta < p.ur ? 1 : 0)) * p.chunk;
    const int tile0 = u0 / S;
    const int st0 = u0 - tile0 * S;

    if (threadIdx.x == 0) {
        for (int s = 0; s < SG; ++s) {
            mbar_init(&bars->full[s], 1);
            mbar_init(&bars->empty[s], NW);
            bars->issued_hi[s] = -1;
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars->red_full[b], NW);
            mbar_init(&bars->red_free[b], 1);
        }
        bars->abort = 0;
        fence_mbar_init();
        tma_prefetch_desc(&p.tm_x);
#pragma unroll
        for (int m = 0; m < NMAT; ++m) {
            tma_prefetch_desc(&p.tm_w[m]);
            if (p.ssc) tma_prefetch_desc(&p.tm_s[m]);
        }
    }
    __syncthreads();
    pdl_launch_dependents();

    if (warp == kGvProducer) {
        // ================================================= producer warp ==
        // Fills the ring, one load group per slot: codes and scales of the
        // first SG groups before waiting on the previous grid (they do not
        // depend on it), their x after; then group i (codes, scales, x) as
        // soon as every compute warp is done with group i - SG, which used
        // the same slot.
        if (lane == 0) {
            const uint64_t pol_w = l2_policy_evict_first();
            const uint64_t pol_x = l2_policy_evict_last();
            const uint32_t x_bytes = static_cast<uint32_t>(p.ks * GPS * M * 128);
            auto issue_w = [&](int slot, int g_tile, int g_st) {
                uint8_t* dst = ring + slot * p.slot_bytes;
                mbar_arrive_expect_tx(&bars->full[slot],
                                      static_cast<uint32_t>(NMAT * cmat + (p.ssc ? Cfg::kSGroup : 0)) +
                                          x_bytes);
                const int sx = (g_st * GPS) & ~7;   // 16-byte aligned first scale group
#pragma unroll
                for (int m = 0; m < NMAT; ++m) {
                    if (p.ks > 1)
                        tma_load_3d(dst + m * cmat, &p.tm_w[m], &bars->full[slot], 0, g_tile * RBM,
                                    g_st, pol_w);
                    else
                        tma_load_2d(dst + m * cmat, &p.tm_w[m], &bars->full[slot], g_st * 128,
                                    g_tile * RBM, pol_w);
                    if (p.ssc)
                        tma_load_2d(dst + p.s_off + m * Cfg::kSMat, &p.tm_s[m], &bars->full[slot],
                                    sx, g_tile * RBM, pol_w);
                }
            };
            auto issue_x = [&](int slot, int g_st) {
                tma_load_3d(ring + slot * p.slot_bytes + p.x_off, &p.tm_x, &bars->full[slot], 0, 0,
                            g_st * GPS, pol_x);
            };
            GvWalk wk{tile0, st0, nu, p.ks};
            int first_st[kGvMaxSG];
            int i = 0;
            for (; i < SG && wk.left > 0; ++i) {
                int g_tile, g_st;
                wk.next(S, g_tile, g_st);
                bars->issued_hi[i] = i;
                issue_w(i, g_tile, g_st);
                first_st[i] = g_st;
            }
            pdl_wait();   // x may be produced by the previous kernel
            for (int j = 0; j < i; ++j) issue_x(j, first_st[j]);
            int slot = i == SG ? 0 : i;
            for (; wk.left > 0; ++i) {
                if (!mbar_wait(&bars->empty[slot], static_cast<uint32_t>(i / SG - 1) & 1, abort_flag,
                               p.timeout_ns, p.status))
                    break;
                int g_tile, g_st;
                wk.next(S, g_tile, g_st);
                bars->issued_hi[slot] = i;
                issue_w(slot, g_tile, g_st);
                issue_x(slot, g_st);
                if (++slot == SG) slot = 0;
            }
        }
        __syncwarp();
        pdl_wait();
    } else if (warp == kGvReducer) {
        // ================================================ reduction warp ==
        // Walks the same row tiles as the compute warps; for every round it
        // adds the WK deposits of each row in k order (deterministic) and
        // stores the tile, or this CTA's piece of a tile that several CTAs
        // share.  It issues no loads of its own, so its fences are cheap.
        pdl_wait();   // (its stores follow the compute warps' waits anyway)
        const int rounds = (M + Cfg::kRedTok - 1) / Cfg::kRedTok;
        const int nbl = p.red_nbuf - 1;                 // log2 of the buffer count (0 or 1)
        int j = 0, tile = tile0, st_seg = st0;
        for (int k = 0; j < nu; ++k) {
            const int len = (S - st_seg) < (nu - j) ? (S - st_seg) : (nu - j);
            const bool whole = st_seg == 0 && len == S;
            const int n_out = M * RB;
            const int slotw = 2 * cta + (j == 0 ? 0 : 1);   // workspace slot of a shared tile
            bool ok_all = true;
            for (int pi = 0; pi < rounds; ++pi) {
                const int r = k * rounds + pi;
                const int b = r & nbl;
                const float* rb = red + b * Cfg::kRedBuf;
                const bool ok = mbar_wait(&bars->red_full[b], static_cast<uint32_t>(r >> nbl) & 1,
                                          abort_flag, p.timeout_ns, p.status);
                ok_all = ok_all && ok;
                const int tok0 = pi * Cfg::kRedTok;
                const int ntok = (M - tok0) < Cfg::kRedTok ? (M - tok0) : Cfg::kRedTok;
                if (ok && *abort_flag == 0) {
                    for (int o = lane; o < ntok * RB; o += 32) {
                        const int tl = o / RB;
                        const int rho = o - tl * RB;
                        float v = 0.0f;
#pragma unroll
                        for (int kw = 0; kw < WK; ++kw) v += rb[kw * Cfg::kRedWarp + tl * RS + rho];
                        const int tok = tok0 + tl;
                        if (whole) {
                            const int m = rho / RBM;
                            const int n = tile * RBM + (rho - m * RBM);
                            if (n < p.N) p.y[m][static_cast<int64_t>(tok) * p.N + n] = v;
                        } else {
                            // slot 2c for the CTA's first segment, 2c+1 for its last
                            p.ws[static_cast<int64_t>(slotw) * n_out + tok * RB + rho] = v;
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars->red_free[b]);
            }
            if (!whole) {
                // combine the pieces: the last of the tile's CTAs to arrive
                // sums every piece in CTA order and writes the tile
                const int tb = tile * S;
                const int c_first = range_owner(tb, p.uq, p.ur);
                const int c_last = range_owner(tb + S - 1, p.uq, p.ur);
                int last = 0;
                if (lane == 0 && ok_all && *abort_flag == 0) {
                    __threadfence();
                    last = atomicAdd(&p.cnt[tile], 1) == c_last - c_first;
                }
                last = __shfl_sync(0xffffffffu, last, 0);
                if (last) {
                    __threadfence();
                    // 4 outputs per lane and step, every contributor's piece
                    // loaded before any is added (loads in flight together);
                    // the sum runs over the contributors in CTA order
                    constexpr int kMaxC = 16;
                    const int nc = c_last - c_first + 1;
                    for (int o4 = lane * 4; o4 < n_out; o4 += 128) {
                        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                        for (int c0 = 0; c0 < nc; c0 += kMaxC) {
                            float4 part[kMaxC];
#pragma unroll
                            for (int ci = 0; ci < kMaxC; ++ci) {
                                const int c = c_first + c0 + ci;
                                if (c0 + ci < nc) {
                                    const int sl = 2 * c + (range_begin(c, p.uq, p.ur) < tb ? 1 : 0);
                                    part[ci] = __ldcg(reinterpret_cast<const float4*>(
                                        p.ws + static_cast<int64_t>(sl) * n_out + o4));
                                }
                            }
#pragma unroll
                            for (int ci = 0; ci < kMaxC; ++ci)
                                if (c0 + ci < nc) {
                                    v.x += part[ci].x;
                                    v.y += part[ci].y;
                                    v.z += part[ci].z;
                                    v.w += part[ci].w;
                                }
                        }
                        const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int o = o4 + e;
                            const int tok = o / RB;
                            const int rho = o - tok * RB;
                            const int m = rho / RBM;
                            const int n = tile * RBM + (rho - m * RBM);
                            if (n < p.N) p.y[m][static_cast<int64_t>(tok) * p.N + n] = vv[e];
                        }
                    }
                    if (lane == 0) p.cnt[tile] = 0;   // ready for the next launch
                }
            }
            j += len;
            ++tile;
            st_seg = 0;
        }
    } else {
        // ================================================= compute warps ==
        // Warp w takes stage w % WK of every load group (if the group has that
        // many stages) and row block w / WK, so it alone consumes that part
        // of every ring slot, round after round.
        const int kw = warp % WK;
        const int rw = warp / WK;
        const int g = lane >> 2;
        const int t = lane & 3;
        const int prow = phys_row<BITS>(g);
        int xtok[NT];   // this thread's token per n-tile, clamped to a valid one
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) xtok[nt] = min(nt * 8 + g, M - 1);
        const int rounds = (M + Cfg::kRedTok - 1) / Cfg::kRedTok;
        const int nbl = p.red_nbuf - 1;
        bool dead = false;
        GvWalk wk{tile0, st0, nu, p.ks};
        int gi = 0, slot = 0;             // load group index and its ring slot
        int k = 0;                        // segment (row tile) index
        float acc[MT][NT][4];
#pragma unroll
        for (int i = 0; i < MT; ++i)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[i][nt][e] = 0.0f;
        while (wk.left > 0) {
            int g_tile, g_st;
            const int n = wk.next(S, g_tile, g_st);
            const bool seg_end = wk.left == 0 || wk.st == 0;   // the group ends this CTA's part of the tile
            // Every warp waits for the group, also one without a stage in it:
            // it must not release the slot (and later wait on the slot's next
            // round) before this round has completed.
            if (!dead && !mbar_wait(&bars->full[slot], static_cast<uint32_t>(gi / SG) & 1,
                                    abort_flag, p.timeout_ns, p.status))
                dead = true;
            if (kw < n && !dead) {
                const int st = g_st + kw;
                const uint8_t* base = ring + slot * p.slot_bytes;
                const uint8_t* wt = base + kw * Cfg::kCStage + rw * (16 * MTW * 128);
                // the stage's first group within the slack-padded scale rows
                const uint8_t* sc = base + p.s_off + rw * (16 * MTW) * Cfg::kSRow * 2 +
                                    (((g_st * GPS) & 7) + kw * GPS) * 2;
                gv_unit<BITS, MT, NT, MTW, Cfg::kSRow, Cfg::kSMat>(
                    wt, cmat, sc, base + p.x_off, kw * GPS, M, xtok, prow, t, p.ssc != 0, p.scales,
                    g_tile * RBM + rw * 16 * MTW, st, p.N, p.groups, acc);
            }
            // ---- the slot is read: release it to the producer
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->empty[slot]);
            ++gi;
            if (++slot == SG) slot = 0;

            if (seg_end) {
                // ---- end of the segment: deposit this warp's partial sums,
                // in rounds of up to 16 tokens, for the reduction warp
#pragma unroll
                for (int pi = 0; pi < (NT * 8 + Cfg::kRedTok - 1) / Cfg::kRedTok; ++pi) {
                    if (pi >= rounds) break;                    // uniform over the CTA
                    const int r = k * rounds + pi;              // reduction round of this CTA
                    const int b = r & nbl;
                    float* rw_ = red + b * Cfg::kRedBuf + kw * Cfg::kRedWarp;
                    if (r > nbl && !mbar_wait(&bars->red_free[b],
                                              static_cast<uint32_t>((r >> nbl) - 1) & 1,
                                              abort_flag, p.timeout_ns, p.status))
                        dead = true;
#pragma unroll
                    for (int i = 0; i < MT; ++i) {
                        // m-tile i: matrix i / MTW, rows rw*16*MTW + 16*(i % MTW) of it
                        const int rbase = (i / MTW) * RBM + rw * 16 * MTW + 16 * (i % MTW);
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            if (nt * 8 < pi * Cfg::kRedTok || nt * 8 >= (pi + 1) * Cfg::kRedTok)
                                continue;
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int tok = nt * 8 + 2 * t + (e & 1);
                                if (tok < M)
                                    rw_[(tok - pi * Cfg::kRedTok) * RS + rbase + 8 * (e >> 1) + prow] =
                                        acc[i][nt][e];
                            }
                        }
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars->red_full[b]);
                }
                ++k;
#pragma unroll
                for (int i = 0; i < MT; ++i)
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int e = 0; e < 4; ++e) acc[i][nt][e] = 0.0f;
            }
        }
    }
    // After a timeout some issued copies may never have been waited for:
    // wait (bounded) for the last one of every slot, so none is in flight
    // when the CTA exits.
    __syncthreads();
    if (threadIdx.x == 0 && *abort_flag) {
        int dummy_abort = 0;
        for (int s = 0; s < SG; ++s) {
            const int il = bars->issued_hi[s];
            if (il >= 0)
                mbar_wait(&bars->full[s], static_cast<uint32_t>(il / SG) & 1, &dummy_abort,
                          p.timeout_ns, p.status);
        }
    }
}

// ------------------------------------------------------------- launcher --


constexpr int kSmemMaxCTA = 227 * 1024;   // dynamic shared memory per CTA, opt-in limit

static int align_up(int v, int a) { return (v + a - 1) / a * a; }

// Shared-memory layout of one launch: SG ring slots (codes, scales, x of a
// load group), reduction buffers, barriers.
struct GvLayout {
    int ks, sg, red_nbuf, slot_bytes, s_off, x_off, red_off, bar_off, smem;
};

template <int BITS, int NMAT, int MTW, int NT, int WK>
static GvLayout gv_layout_for(int M, int ks, int sg, int red_nbuf) {
    using Cfg = GvCfg<BITS, NMAT, MTW, NT, WK>;
    GvLayout L;
    L.ks = ks;
    L.sg = sg;
    L.red_nbuf = red_nbuf;
    L.s_off = NMAT * ks * Cfg::kCStage;                    // a multiple of 1024
    L.x_off = align_up(L.s_off + Cfg::kSGroup, 1024);      // swizzled x box: 1024-aligned
    L.slot_bytes = align_up(L.x_off + ks * Cfg::kGPS * M * 128, 1024);
    L.red_off = sg * L.slot_bytes;
    L.bar_off = align_up(L.red_off + red_nbuf * Cfg::kRedBuf * 4, 16);
    L.smem = 1024 /* alignment slack */ + L.bar_off + static_cast<int>(sizeof(GvBars));
    return L;
}

// Within the shared memory of one CTA: the deepest ring (2..8 groups, no
// deeper than the busiest CTA's groups), with two reduction buffers if
// possible, for groups of ks stages.
template <int BITS, int NMAT, int MTW, int NT, int WK>
static bool gv_layout(int M, int ks, int nu_max, int S, GvLayout* out) {
    const int groups_max = (nu_max + ks - 1) / ks + (nu_max + S - 1) / S + 1;
    const int want = groups_max < 2 ? 2 : (groups_max > kGvMaxSG ? kGvMaxSG : groups_max);
    for (int sg = want; sg >= 2; --sg)
        for (int rbuf = 2; rbuf >= 1; --rbuf) {
            const GvLayout L = gv_layout_for<BITS, NMAT, MTW, NT, WK>(M, ks, sg, rbuf);
            if (L.smem <= kSmemMaxCTA) {
                *out = L;
                return true;
            }
        }
    return false;
}

// Share of the SMs' time spent working when whole row tiles are dealt to
// one CTA per SM: tiles / (SMs * the busiest CTA's tiles).
static double gv_tile_balance(int tiles, int sms) {
    const int per = (tiles + sms - 1) / sms;
    return static_cast<double>(tiles) / (static_cast<double>(per) * sms);
}

// Whole tiles per CTA (nothing then waits on another CTA) when they keep the
// SMs at least 85% busy, e.g. 128 16-row tiles of a 2048-row projection.
static bool gv_whole_tiles(int tiles, int sms) {
    return gv_tile_balance(tiles, sms) >= 0.85;
}

template <int BITS, int NMAT, int MTW, int NT, int WK>
static cudaError_t gv_launch(GvParams& prm, const uint16_t* x, const void* const* codes,
                             cudaStream_t s, const GemvScratch* scratch) {
    using Cfg = GvCfg<BITS, NMAT, MTW, NT, WK>;
    auto kern = gemv_wq_kernel<BITS, NMAT, MTW, NT, WK>;
    static bool attr_set[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!attr_set[dev]) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemMaxCTA);
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    prm.tiles = (prm.N + Cfg::kRBM - 1) / Cfg::kRBM;
    const int64_t row_bytes = static_cast<int64_t>(prm.K) * BITS / 8;
    prm.kstages = static_cast<int>((row_bytes + 127) / 128);
    const int64_t units = static_cast<int64_t>(prm.tiles) * prm.kstages;
    if (units >= (int64_t{1} << 31)) return cudaErrorInvalidValue;
    prm.units = static_cast<int>(units);

    // Grid: one CTA per SM at most.  Whole row tiles per CTA (nothing is
    // reduced across CTAs) when they balance over the SMs -- one tile per CTA
    // for small projections; otherwise stream-K over equal runs of units.
    const int sms = num_sms();
    int grid = 0;
    if (gv_whole_tiles(prm.tiles, sms)) {
        grid = prm.tiles < sms ? prm.tiles : sms;
        prm.chunk = prm.kstages;
    } else {
        grid = static_cast<int>(units < sms ? units : sms);
        prm.chunk = 1;
    }
    const int chunks = prm.units / prm.chunk;
    prm.uq = chunks / grid;
    prm.ur = chunks % grid;
    // The 3D code view needs rows of whole 128-byte stages; otherwise one
    // stage per group.  Fewer stages per group (fewer warps busy) when WK
    // stages of codes and x do not fit twice in shared memory.
    GvLayout L;
    bool fits = false;
    for (int ks = row_bytes % 128 == 0 ? WK : 1; ks >= 1 && !fits; ks /= 2)
        fits = gv_layout<BITS, NMAT, MTW, NT, WK>(prm.M, ks, (prm.uq + 1) * prm.chunk, prm.kstages, &L);
    if (!fits) return cudaErrorInvalidValue;
    prm.ks = L.ks;
    prm.sg = L.sg;
    prm.slot_bytes = L.slot_bytes;
    prm.s_off = L.s_off;
    prm.x_off = L.x_off;
    prm.red_off = L.red_off;
    prm.red_nbuf = L.red_nbuf;
    prm.bar_off = L.bar_off;
    // scales by TMA when a scale row is a multiple of 16 bytes
    prm.ssc = (prm.groups * 2) % 16 == 0 ? 1 : 0;

    // partial-tile slots and arrival counters: stream-K only
    const bool sk = prm.chunk == 1;
    const size_t ws_bytes = sk ? static_cast<size_t>(2) * grid * prm.M * Cfg::kRB * sizeof(float) : 0;
    const size_t n_cnt = sk ? static_cast<size_t>(prm.tiles) : 0;
    if (scratch == nullptr) {
        e = workspace_get(ws_bytes, n_cnt, &prm.ws, &prm.cnt);
        if (e != cudaSuccess) return e;
    } else {
        if (ws_bytes > scratch->ws_bytes || n_cnt > scratch->n_cnt) {
            if (scratch->too_large) *scratch->too_large = true;
            return cudaErrorInvalidValue;   // refused before anything is enqueued
        }
        prm.ws = scratch->ws;
        prm.cnt = scratch->cnt;
        // a completed launch leaves its counters at zero, an aborted one might
        // not: clear the ones this launch uses
        if (n_cnt > 0) {
            e = cudaMemsetAsync(prm.cnt, 0, n_cnt * sizeof(int), s);
            if (e != cudaSuccess) return e;
        }
    }

    // Codes as {128 B of a stage, row, stage}: a box is ks consecutive stages
    // of RBM rows, stage-major in shared memory (each stage a [RBM][128 B]
    // block, 128-byte swizzled like a 2D box).  With one stage per group, a
    // 2D map, whose columns past the row's end read zeros.
    for (int i = 0; i < NMAT; ++i) {
        const bool okw =
            prm.ks > 1
                ? make_tmap_3d(&prm.tm_w[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, codes[i], 128,
                               static_cast<uint64_t>(prm.N), static_cast<uint64_t>(prm.kstages),
                               static_cast<uint64_t>(row_bytes), 128, 128, Cfg::kRBM,
                               static_cast<uint32_t>(prm.ks), CU_TENSOR_MAP_SWIZZLE_128B)
                : make_tmap_2d(&prm.tm_w[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, codes[i],
                               static_cast<uint64_t>(row_bytes), static_cast<uint64_t>(prm.N),
                               static_cast<uint64_t>(row_bytes), 128, Cfg::kRBM,
                               CU_TENSOR_MAP_SWIZZLE_128B);
        if (!okw) return cudaErrorInvalidValue;
        if (prm.ssc &&
            !make_tmap_2d(&prm.tm_s[i], CU_TENSOR_MAP_DATA_TYPE_UINT16, prm.scales[i],
                          static_cast<uint64_t>(prm.groups), static_cast<uint64_t>(prm.N),
                          static_cast<uint64_t>(prm.groups) * 2, Cfg::kSRow, Cfg::kRBM,
                          CU_TENSOR_MAP_SWIZZLE_NONE))
            return cudaErrorInvalidValue;
    }
    // x as {64 k of a group, token, group}: a box is the ks stages' groups
    // of all M tokens, group-major in shared memory, 128-byte swizzled
    if (!make_tmap_3d(&prm.tm_x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, x, 64,
                      static_cast<uint64_t>(prm.M), static_cast<uint64_t>(prm.groups),
                      static_cast<uint64_t>(prm.K) * 2, 128, 64, static_cast<uint32_t>(prm.M),
                      static_cast<uint32_t>(prm.ks * Cfg::kGPS), CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
    cfg.blockDim = dim3(kGvThreads, 1, 1);
    cfg.dynamicSmemBytes = static_cast<size_t>(L.smem);
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

// Row tile and warp split.  M <= 16: warps split k (WK = 8) and a tile has
// 16 * MTW rows per matrix: 16 while that gives at most one tile per SM
// (small projections then run as one wave of whole tiles, no reduction
// across CTAs); else the tile height whose whole tiles balance best over the
// SMs, weighted by the unit speed (x fragments shared by more rows); else
// stream-K.  M > 16: warps split the rows of 128-row tiles (WK = 1), so the
// x of a stage, large at this M, is loaded once for all 8 warps.
static int gv_pick_mtw(int N) {
    const int sms = num_sms();
    if ((N + 15) / 16 <= sms) return 1;
    // relative speed of a warp's unit by m-tiles per unit, measured on B200:
    // 44 / 47 / 49 weights per cycle and SM for 1 / 2 / 4 m-tiles
    const double speed[5] = {0.0, 44.0, 47.0, 0.0, 49.0};
    int best = 0;
    double best_score = 0.0;
    for (int mtw = 4; mtw >= 1; mtw /= 2) {
        const int tiles = (N + 16 * mtw - 1) / (16 * mtw);
        const double bal = gv_tile_balance(tiles, sms);
        if (bal >= 0.85 && bal * speed[mtw] > best_score) {
            best = mtw;
            best_score = bal * speed[mtw];
        }
    }
    return best ? best : 2;   // stream-K
}

template <int BITS, int NMAT, int NT>
static cudaError_t gv_dispatch_mt(GvParams& prm, const uint16_t* x, const void* const* codes,
                                  cudaStream_t s, const GemvScratch* sc) {
    if constexpr (NT == 4) {
        // rows split over the warps (x of a stage loaded once for 8 warps) when
        // whole 128-row tiles balance; else k split with fewer stages per
        // group (the x of 8 stages of 32 tokens does not fit twice)
        if (gv_whole_tiles((prm.N + 127) / 128, num_sms()))
            return gv_launch<BITS, NMAT, 1, 4, 1>(prm, x, codes, s, sc);
        return gv_launch<BITS, NMAT, 1, 4, 8>(prm, x, codes, s, sc);
    } else if constexpr (NMAT == 3) {
        return gv_launch<BITS, 3, 1, NT, 8>(prm, x, codes, s, sc);
    } else {
        int mtw = gv_pick_mtw(prm.N);
        // M up to 16 with 8-stage groups: the x of a group (8 stages of M
        // tokens) shares the slot with the codes; fall back to fewer rows
        if constexpr (NT == 2)
            if (mtw > 2) mtw = 2;
        if (mtw == 1) return gv_launch<BITS, 1, 1, NT, 8>(prm, x, codes, s, sc);
        if (mtw == 2) return gv_launch<BITS, 1, 2, NT, 8>(prm, x, codes, s, sc);
        if constexpr (NT == 1) return gv_launch<BITS, 1, 4, NT, 8>(prm, x, codes, s, sc);
        return cudaErrorInvalidValue;
    }
}

template <int BITS, int NMAT>
static cudaError_t gv_dispatch_nt(GvParams& prm, const uint16_t* x, const void* const* codes,
                                  cudaStream_t s, const GemvScratch* sc) {
    // 8 tokens per n-tile
    if (prm.M <= 8) return gv_dispatch_mt<BITS, NMAT, 1>(prm, x, codes, s, sc);
    if (prm.M <= 16) return gv_dispatch_mt<BITS, NMAT, 2>(prm, x, codes, s, sc);
    return gv_dispatch_mt<BITS, NMAT, 4>(prm, x, codes, s, sc);
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
    if (nmat == 3)
        return bits == 4 ? gv_dispatch_nt<4, 3>(prm, x, codes, s, sc)
                         : gv_dispatch_nt<8, 3>(prm, x, codes, s, sc);
    return bits == 4 ? gv_dispatch_nt<4, 1>(prm, x, codes, s, sc)
                     : gv_dispatch_nt<8, 1>(prm, x, codes, s, sc);
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
