// rq_gemv_rb.cuh -- decode product (1 <= M <= 32) on group-64 quantized
// weights, row blocks over full K: the row-block decode kernel.
//
//   y[m, n] = sum_g s16[n, g] * sum_{k in g} x[m, k] * code[n, k]
//
// The "Hakureirm/rwkv7-sglang-w4gptq-1.5b" model card (opening summary)
// credits its decode speed-up to a hand-written int4 GEMV / small-M kernel
// family streaming the g64 codes; the "RWKV-7 Quantization Toolkit"
// (rwkv-quant-nv 1.2.1), "Key Design", keeps weights quantized on the path and
// runs R/K/V in one launch.  This is the B200 form of that decode step.
//
// Work decomposition.  The rows of each matrix are cut into 16-row m-tiles
// and the m-tiles into blocks of TC consecutive m-tiles (TC = the m-tiles
// per SM, rounded up); a CTA owns whole blocks over the FULL K range, so
// every output is finished inside one CTA: no partial sums leave the SM, no
// workspace, no counters.  (An SM that owns fewer m-tiles than another simply
// finishes early; one CTA can pull well above its share of HBM bandwidth, so
// the busiest SMs set the pace only when their share exceeds what one SM can
// stream.)  Fused R/K/V: the three matrices' blocks are concatenated; a block
// never straddles two matrices.
//
// Data path.  A ring of slots in shared memory; a slot holds, for the
// block's rows, S consecutive 128-byte code stages (one 3-D TMA box
// {128 B, 16*TC rows, S stages}, 128-byte swizzled), their fp16 scales (one
// 2-D box) and the x of their groups (one 3-D box {64 k, M tokens, groups}).
// Codes and scales of the first slots are requested by thread 0 before the
// kernel waits on the previous grid (they never depend on it); x after.  The
// last warp to finish with a slot refills it (an arrival counter in shared
// memory), so no warp waits to refill.  The 8 warps, all computing, split a
// slot's group columns (warp w takes columns w, w+8, ...) and
// each takes every m-tile of the block for its columns, so an x fragment is
// loaded once per warp and column and used TC times.  At the end of a block
// the warps' partial sums meet in shared memory (the ring, reused) and are
// added in warp order, so the result is deterministic.
//
// Math.  Thread (g = lane/4, t = lane%4) owns, per group of 64 k, the 16 k
// [16t, 16t+16) of rows g and g+8 of each m-tile (a k-permutation inside the
// group, the same on the A and B side, so the sum over k is unchanged).  Codes
// are turned into BIASED fp16 values with one lop3 per pair (the bit placement
// of Kim et al., arXiv:2211.10017, without the exact bias subtraction): int4
// low nibbles become 1032 + c (exponent of [1024, 2048)), high nibbles
// 72 + c (exponent of [64, 128), the nibble at mantissa bits 4..7); int8
// bytes 1152 + c.  mma.sync.m16n8k16 sums x * (code + bias) in fp32, starting
// from -sum_k bias_k x_k of the group, which one chain of MMAs with a
// constant A operand (-bias) computes once per group and 8-token tile and
// every m-tile reuses.  The group's scale is applied in fp32
// (acc = fma(part, s16, acc)).  Products x * (code + bias) are exact in fp32
// (11 x 11 significant bits), so the bias costs only the fp32 rounding of
// sums of magnitude ~1000 |x|: about 1e-4 of the error budget
// 2e-3 * sum |x||w_hat| per output.
#pragma once
#include <cuda_fp16.h>

#include <cstring>

#include "rq_internal.h"
#include "rq_ptx.cuh"
#include "rq_gemv_unit.cuh"

namespace rq {

struct RbParams {
    CUtensorMap tm_w[3];  // codes: 3-D {128 B, N rows, stages} box {128, RB, S}, or (rows not whole
                          // stages) 2-D {row bytes, N} box {128, RB}; SWIZZLE_128B
    CUtensorMap tm_s[3];  // scales [N, groups] fp16: box {SROW, RB} (when ssc)
    CUtensorMap tm_x[3];  // x of each matrix as 3-D {64, M, groups}: box {64, M, J}, SWIZZLE_128B
    const uint16_t* scales[3];
    void* y[3];           // fp32 or (yh) fp16 [M, N]
    int M, N, K;
    int groups;           // K / 64
    int stages;           // 128-byte code stages per row
    int tc;               // m-tiles per block (TC)
    int bpm;              // blocks per matrix
    int nblocks;          // blocks in all matrices
    int S;                // stages per slot
    int J;                // group columns per slot (S * groups per stage)
    int slots;            // slots per block: ceil(stages / S)
    int sg;               // ring depth (slots)
    int three_d;          // codes through the 3-D map
    int ssc;              // scales staged by TMA
    int srow;             // scale row length in a slot (fp16, 16-byte multiple)
    int slot_bytes, s_off, x_off, bar_off, red_stride;
    int nx;               // distinct inputs: 1 (shared x) or 3 (one per matrix)
    const uint32_t* sup[3];  // asymmetric preset: fp16 (ds, dm) pairs [N, K/256] as 32-bit words
    int nsb;              // super-blocks per row (K / 256)
    int yh;               // y stored as fp16 (round to nearest even)
    int epi;              // epilogue: 0 none, 1 relu(y)^2
    int* status;
    uint64_t timeout_ns;
};

constexpr int kRbSrow = 40;                     // fp16 scales per staged row (J <= 32, + slack)
constexpr int kRbSrowP8 = 72;                   // int8 g16 preset: 4 J (J <= 16) + slack
constexpr int kRbWarps = 8;                     // warps, all computing
constexpr int kRbThreads = kRbWarps * 32;
constexpr int kRbMaxSG = 8;

struct RbBars {
    uint64_t full[kRbMaxSG];   // the slot holds its codes, scales and x
    int done[kRbMaxSG];        // warps finished with the slot's current round
    int issued_hi[kRbMaxSG];   // last slot index issued into each ring slot
    int abort;
};

// D = A * B + C (fp16 inputs, fp32 accumulate), C and D distinct.
__device__ __forceinline__ void mma16816_c(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                           uint32_t b1, const float (&c)[4]) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%10,%11,%12,%13};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]),
          "f"(c[2]), "f"(c[3]));
}

// int4, permuted pair order, biased: one code word (positions 0..7 of a row,
// position 2i in the low nibble of byte i) -> pairs (p0,p4) and (p2,p6) as
// 1032 + c, pairs (p1,p5) and (p3,p7) as 72 + c.  5 instructions per 8 codes.
__device__ __forceinline__ void i4_word_biased(uint32_t w, uint32_t (&P)[4]) {
    const uint32_t w8 = w >> 8;
    P[0] = lop3_bmux(w, 0x000F000Fu, 0x64086408u);    // 0x6400 | (nibble ^ 8)       = 1032 + c
    P[1] = lop3_bmux(w, 0x00F000F0u, 0x54805480u);    // 0x5400 | (nibble ^ 8) << 4  = 72 + c
    P[2] = lop3_bmux(w8, 0x000F000Fu, 0x64086408u);
    P[3] = lop3_bmux(w8, 0x00F000F0u, 0x54805480u);
}

// int8, biased: one 32-bit word (positions 0..3) -> pairs (p0,p1), (p2,p3) as
// 1152 + c.  3 instructions per 4 codes.
__device__ __forceinline__ void i8_word_biased(uint32_t w, uint32_t (&Q)[2]) {
    w ^= 0x80808080u;
    Q[0] = __byte_perm(w, 0x64646464u, 0x5140u);
    Q[1] = __byte_perm(w, 0x64646464u, 0x5342u);
}

// Group columns of one warp (NC of them, processed together for independent
// dependency chains): every m-tile of the block (MT of them) times the x of
// the column's group, for NT 8-token tiles.  Per column c:
//   cw0[c]  codes of the column's stage, m-tile 0, this thread's physical row
//           and chunk (rows 16i + prow and +8 of m-tile i are 16*128*i and
//           8*128 further)
//   sp[c]   scales: (row 16i + 8h + prow, this group) at sp[c][(16i + 8h) * kRbSrow]
//   xrow    byte offsets (from xbase) of the 128-byte x rows of the column's
//           group for the tokens nt*8+g; xph[nt] their swizzle phase
//   grp[c]  the group (for scales read from global memory when !SSC)
// The group's four MMA steps run as one chain that starts from the bias term
// (so no additions are needed), and the scale is applied with one fma.  With
// several token tiles and few m-tiles the bias MMAs (4 per token tile and
// column, shared by the m-tiles) would cost more tensor-pipe time than they
// save: there the codes are unbiased exactly in fp16 instead (one
// subtraction per register) and the chain starts from zero.
template <int MT, int NT>
constexpr bool rb_unbias() { return NT >= 4 || (NT == 2 && MT <= 4); }

// MT: m-tiles this warp takes (of the block's MTALL, from m-tile mi0 on).
template <int BITS, int MT, int NT, int NC, bool SSC, int MTALL = MT>
__device__ __forceinline__ void rb_columns(const uint8_t* const (&cw0)[NC],
                                           const uint16_t* const (&sp)[NC], const uint8_t* xbase,
                                           const int (&xrow)[NC][NT], const int (&xph)[NT], int t,
                                           float (&acc)[MT][NT][4], const uint16_t* gscales,
                                           int64_t grow0, int groups, const int (&grp)[NC], int N,
                                           int mi0 = 0) {
    constexpr int CW = BITS == 4 ? 2 : 4;   // code words per row and group
    // ---- x fragments: token nt*8+g, positions 16t .. 16t+15 of the group
    uint32_t b[NC][NT][4][2];
#pragma unroll
    for (int c = 0; c < NC; ++c)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const uint8_t* xr = xbase + xrow[c][nt];
            const int c0 = ((2 * t) ^ xph[nt]) << 4;
            const uint4 v0 = lds128(xr + c0);
            const uint4 v1 = lds128(xr + (c0 ^ 16));
            const uint32_t X[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                if constexpr (BITS == 4) {
                    // step jj pairs (p0,p4),(p1,p5) or (p2,p6),(p3,p7) of word jj/2
                    const int wb = (jj >> 1) * 4 + (jj & 1);
                    b[c][nt][jj][0] = __byte_perm(X[wb], X[wb + 2], 0x5410);
                    b[c][nt][jj][1] = __byte_perm(X[wb], X[wb + 2], 0x7632);
                } else {
                    b[c][nt][jj][0] = X[2 * jj];
                    b[c][nt][jj][1] = X[2 * jj + 1];
                }
            }
        }
    // ---- -sum_k bias_k x_k of each column's group, per token tile (the same
    // for every row)
    constexpr bool kUnbias = rb_unbias<MTALL, NT>();
    float negc[NC][NT][4];
    if constexpr (!kUnbias) {
        uint32_t an[4];
        if constexpr (BITS == 4) {
            an[0] = an[1] = 0xE408E408u;   // -1032 (slots 2t, 2t+1: low-nibble pairs)
            an[2] = an[3] = 0xD480D480u;   // -72   (slots 2t+8, 2t+9: high-nibble pairs)
        } else {
            an[0] = an[1] = an[2] = an[3] = 0xE480E480u;   // -1152
        }
#pragma unroll
        for (int c = 0; c < NC; ++c)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                mma16816(negc[c][nt], an, b[c][nt][0][0], b[c][nt][0][1], true);
#pragma unroll
                for (int jj = 1; jj < 4; ++jj)
                    mma16816(negc[c][nt], an, b[c][nt][jj][0], b[c][nt][jj][1], false);
            }
    }
    // ---- every m-tile of this warp
#pragma unroll
    for (int i = 0; i < MT; ++i) {
        const int mi = mi0 + i;                // m-tile within the block
        if (MT != MTALL && mi >= MTALL) break;   // (odd split: the second half is short)
#pragma unroll
        for (int c = 0; c < NC; ++c) {
            uint32_t cw[2][CW];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint8_t* cp = cw0[c] + (16 * mi + 8 * h) * 128;
                if constexpr (BITS == 4) {
                    const uint2 v = lds64(cp);
                    cw[h][0] = v.x;
                    cw[h][1] = v.y;
                } else {
                    const uint4 v = lds128(cp);
                    cw[h][0] = v.x; cw[h][1] = v.y; cw[h][2] = v.z; cw[h][3] = v.w;
                }
            }
            float sv[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint16_t s16;
                if constexpr (SSC) {
                    s16 = sp[c][(16 * mi + 8 * h) * kRbSrow];
                } else {
                    const int64_t n = grow0 + 16 * mi + 8 * h;
                    s16 = (n < N && grp[c] < groups) ? __ldg(gscales + n * groups + grp[c])
                                                     : static_cast<uint16_t>(0);
                }
                sv[h] = __half2float(__ushort_as_half(s16));
            }
            uint32_t A[4][4];   // [step][a-reg]
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                if constexpr (BITS == 4) {
                    uint32_t P0[4], P1[4];
                    i4_word_biased(cw[h][0], P0);
                    i4_word_biased(cw[h][1], P1);
                    A[0][h] = P0[0]; A[0][h + 2] = P0[1];
                    A[1][h] = P0[2]; A[1][h + 2] = P0[3];
                    A[2][h] = P1[0]; A[2][h + 2] = P1[1];
                    A[3][h] = P1[2]; A[3][h + 2] = P1[3];
                } else {
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        uint32_t Q[2];
                        i8_word_biased(cw[h][jj], Q);
                        A[jj][h] = Q[0];
                        A[jj][h + 2] = Q[1];
                    }
                }
            }
            if constexpr (kUnbias) {
                // exact: 1032 + c, 72 + c and 1152 + c minus their bias is c
                const __half2 blo = __halves2half2(__ushort_as_half(BITS == 4 ? 0x6408 : 0x6480),
                                                   __ushort_as_half(BITS == 4 ? 0x6408 : 0x6480));
                const __half2 bhi = __halves2half2(__ushort_as_half(BITS == 4 ? 0x5480 : 0x6480),
                                                   __ushort_as_half(BITS == 4 ? 0x5480 : 0x6480));
#pragma unroll
                for (int jj = 0; jj < 4; ++jj)
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        __half2 v = *reinterpret_cast<const __half2*>(&A[jj][r]);
                        v = __hsub2(v, r < 2 ? blo : bhi);
                        A[jj][r] = *reinterpret_cast<const uint32_t*>(&v);
                    }
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                float part[4];
                if constexpr (kUnbias)
                    mma16816(part, A[0], b[c][nt][0][0], b[c][nt][0][1], true);
                else
                    mma16816_c(part, A[0], b[c][nt][0][0], b[c][nt][0][1], negc[c][nt]);
#pragma unroll
                for (int jj = 1; jj < 4; ++jj) mma16816(part, A[jj], b[c][nt][jj][0], b[c][nt][jj][1], false);
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[i][nt][e] = fmaf(part[e], sv[e >> 1], acc[i][nt][e]);
            }
        }
    }
}


// ---------------------------------------------------- preset formats --------
// Column math of the two rwkv-quant preset formats.  A column is again 64 k
// of the block's rows; the k-permutation keeps every MMA step inside one
// group:
//   int8, groups of 16: step jj is group jj of the column; thread t holds k
//     16jj + 4t .. +3 of rows g and g+8 (one 32-bit word per row and step)
//     and the matching four x values; the bias term of each step is its own
//     constant-operand MMA, and each step's sum gets its group's scale;
//   int4, groups of 32, asymmetric: steps 0-1 are the column's first group,
//     steps 2-3 its second; thread t holds k 8t .. 8t+7 of the first group and
//     32+8t .. 32+8t+7 of the second (one 32-bit word each), x permuted to the
//     pair order of the unpacking.  Unsigned codes q become 1024 + q (low
//     nibbles) and 64 + q (high nibbles) with one lop3 per pair; a constant-
//     operand MMA gives, in rows 0-7, -sum beta_k x_k and, in rows 8-15,
//     sum x_k, so the group adds S (P - sum beta x) + O sum x, where P =
//     sum (beta + q) x comes from the MMAs and S = ds a, O = -(dm b).

// Unsigned int4, permuted pair order, biased: (p0,p4), (p2,p6) as 1024 + q;
// (p1,p5), (p3,p7) as 64 + q.
__device__ __forceinline__ void u4_word_biased(uint32_t w, uint32_t (&P)[4]) {
    const uint32_t w8 = w >> 8;
    asm("lop3.b32 %0, %1, %2, %3, 0xea;" : "=r"(P[0]) : "r"(w), "r"(0x000F000Fu), "r"(0x64006400u));
    asm("lop3.b32 %0, %1, %2, %3, 0xea;" : "=r"(P[1]) : "r"(w), "r"(0x00F000F0u), "r"(0x54005400u));
    asm("lop3.b32 %0, %1, %2, %3, 0xea;" : "=r"(P[2]) : "r"(w8), "r"(0x000F000Fu), "r"(0x64006400u));
    asm("lop3.b32 %0, %1, %2, %3, 0xea;" : "=r"(P[3]) : "r"(w8), "r"(0x00F000F0u), "r"(0x54005400u));
}

// Byte k of v as the fp32 2^23 + v.byte[k] (one prmt, no conversion).
template <int k>
__device__ __forceinline__ float byte_plus_2p23(uint32_t v) {
    return __uint_as_float(__byte_perm(v, 0x4B000000u, 0x7540u + k));
}

__device__ __forceinline__ uint32_t lds32(const uint8_t* p) { return *reinterpret_cast<const uint32_t*>(p); }

// int8 preset, one column: cwa[jj] codes of step jj (m-tile 0, this thread's
// physical row and word); sp scales of the column's four groups for this
// thread's row (m-tile i, half h at + (16i + 8h) * kRbSrowP8); x as for
// rb_columns, xr the column's token rows.
template <int MT, int NT>
__device__ __forceinline__ void rb_column_p8(const uint8_t* const (&cwa)[4], const uint16_t* sp,
                                             const uint8_t* xbase, const int (&xr)[NT],
                                             const int (&xph)[NT], int t, float (&acc)[MT][NT][4]) {
    uint32_t b[NT][4][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const uint8_t* row = xbase + xr[nt];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            const uint2 v = lds64(row + ((((2 * jj + (t >> 1)) ^ xph[nt]) << 4) + ((t & 1) << 3)));
            b[nt][jj][0] = v.x;
            b[nt][jj][1] = v.y;
        }
    }
    constexpr bool kUnbias = rb_unbias<MT, NT>();
    float negc[NT][4][4];   // [nt][step][element]
    if constexpr (!kUnbias) {
        uint32_t an[4];
        an[0] = an[1] = an[2] = an[3] = 0xE480E480u;   // -1152
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) mma16816(negc[nt][jj], an, b[nt][jj][0], b[nt][jj][1], true);
    }
#pragma unroll
    for (int i = 0; i < MT; ++i) {
        uint32_t A[4][4];
        float sv[4][2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                uint32_t Q[2];
                i8_word_biased(lds32(cwa[jj] + (16 * i + 8 * h) * 128), Q);
                if constexpr (kUnbias) {
                    const __half2 bias = __halves2half2(__ushort_as_half(0x6480), __ushort_as_half(0x6480));
#pragma unroll
                    for (int r = 0; r < 2; ++r) {
                        __half2 v = *reinterpret_cast<const __half2*>(&Q[r]);
                        v = __hsub2(v, bias);
                        Q[r] = *reinterpret_cast<const uint32_t*>(&v);
                    }
                }
                A[jj][h] = Q[0];
                A[jj][h + 2] = Q[1];
                sv[jj][h] = __half2float(__ushort_as_half(sp[(16 * i + 8 * h) * kRbSrowP8 + jj]));
            }
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                float part[4];
                if constexpr (kUnbias)
                    mma16816(part, A[jj], b[nt][jj][0], b[nt][jj][1], true);
                else
                    mma16816_c(part, A[jj], b[nt][jj][0], b[nt][jj][1], negc[nt][jj]);
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[i][nt][e] = fmaf(part[e], sv[jj][e >> 1], acc[i][nt][e]);
            }
    }
}

// int4 asymmetric preset, one column: cwa / cwb the words of the column's two
// groups (m-tile 0, this thread's row); subp the (a, b) sub-codes of the two
// groups for this thread's row (m-tile i, half h at + (16i + 8h) * sstride);
// supp the (ds, dm) words of the column's super-block for rows row0 + prow +
// 16i + 8h (global, nsb words apart per row).
template <int MT, int NT>
__device__ __forceinline__ void rb_column_p4a(const uint8_t* cwa, const uint8_t* cwb,
                                              const uint8_t* subp, int sstride,
                                              const uint32_t* supp, int nsb, int64_t grow0, int N,
                                              const uint8_t* xbase, const int (&xr)[NT],
                                              const int (&xph)[NT], int t, float (&acc)[MT][NT][4]) {
    uint32_t b[NT][4][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const uint8_t* row = xbase + xr[nt];
        const uint4 v0 = lds128(row + ((t ^ xph[nt]) << 4));
        const uint4 v1 = lds128(row + (((4 + t) ^ xph[nt]) << 4));
        const uint32_t X[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            const int wb = (jj >> 1) * 4 + (jj & 1);
            b[nt][jj][0] = __byte_perm(X[wb], X[wb + 2], 0x5410);
            b[nt][jj][1] = __byte_perm(X[wb], X[wb + 2], 0x7632);
        }
    }
    // per group and token tile: rows 0-7 -sum beta x, rows 8-15 sum x
    float cor[NT][2][4];
    {
        uint32_t an[4];
        an[0] = 0xE400E400u;   // -1024, rows g:   slots 2t, 2t+1 (low-nibble pairs)
        an[1] = 0x3C003C00u;   // 1,     rows g+8
        an[2] = 0xD400D400u;   // -64,   rows g:   slots 2t+8, 2t+9 (high-nibble pairs)
        an[3] = 0x3C003C00u;   // 1,     rows g+8
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int gg = 0; gg < 2; ++gg) {
                mma16816(cor[nt][gg], an, b[nt][2 * gg][0], b[nt][2 * gg][1], true);
                mma16816(cor[nt][gg], an, b[nt][2 * gg + 1][0], b[nt][2 * gg + 1][1], false);
            }
    }
#pragma unroll
    for (int i = 0; i < MT; ++i) {
        uint32_t A[4][4];
        float S[2][2], O[2][2];   // [group][half]
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            uint32_t Pa[4], Pb[4];
            u4_word_biased(lds32(cwa + (16 * i + 8 * h) * 128), Pa);
            u4_word_biased(lds32(cwb + (16 * i + 8 * h) * 128), Pb);
            A[0][h] = Pa[0]; A[0][h + 2] = Pa[1];
            A[1][h] = Pa[2]; A[1][h + 2] = Pa[3];
            A[2][h] = Pb[0]; A[2][h + 2] = Pb[1];
            A[3][h] = Pb[2]; A[3][h + 2] = Pb[3];
            const uint32_t ab = lds32(subp + (16 * i + 8 * h) * sstride);   // a_a, b_a, a_b, b_b
            const int64_t n = grow0 + 16 * i + 8 * h;
            const uint32_t dd = n < N ? __ldg(supp + (16 * i + 8 * h) * nsb) : 0u;
            const float ds = __half2float(__ushort_as_half(static_cast<unsigned short>(dd & 0xFFFFu)));
            const float dm = __half2float(__ushort_as_half(static_cast<unsigned short>(dd >> 16)));
            // S = ds a = ds (2^23 + a) - ds 2^23 and O = -(dm b) likewise, each
            // one fused multiply-add: exact (ds a and dm b fit in 17 bits)
            const float ds23 = ds * 8388608.0f, dm23 = dm * 8388608.0f;
            S[0][h] = fmaf(ds, byte_plus_2p23<0>(ab), -ds23);
            O[0][h] = fmaf(-dm, byte_plus_2p23<1>(ab), dm23);
            S[1][h] = fmaf(ds, byte_plus_2p23<2>(ab), -ds23);
            O[1][h] = fmaf(-dm, byte_plus_2p23<3>(ab), dm23);
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int gg = 0; gg < 2; ++gg) {
                // start from -sum beta x (rows g and g+8 of the MMA both take
                // the token's value, held in elements 0 and 1)
                const float c0[4] = {cor[nt][gg][0], cor[nt][gg][1], cor[nt][gg][0], cor[nt][gg][1]};
                float part[4];
                mma16816_c(part, A[2 * gg], b[nt][2 * gg][0], b[nt][2 * gg][1], c0);
                mma16816(part, A[2 * gg + 1], b[nt][2 * gg + 1][0], b[nt][2 * gg + 1][1], false);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    acc[i][nt][e] = fmaf(part[e], S[gg][e >> 1], acc[i][nt][e]);
                    acc[i][nt][e] = fmaf(cor[nt][gg][2 + (e & 1)], O[gg][e >> 1], acc[i][nt][e]);
                }
            }
    }
}

// WARPS = 8: every warp takes all MT m-tiles of its columns; WARPS = 16 (the
// group-64 format at M <= 8 on blocks of >= 2 m-tiles): warps w and w + 8
// share the columns and split the m-tiles, so twice the warps (with half the
// accumulators each) hide the shared-memory latency of the loop.
template <int FMT, int BITS, int MT, int NT, bool SSC, int WARPS = 8>
__global__ void __launch_bounds__(WARPS * 32, 1) gemv_rb_kernel(const __grid_constant__ RbParams p) {
    static_assert(WARPS == 8 || (WARPS == 16 && FMT == FMT_G64), "m-tile halves: group-64 only");
    constexpr int GPS = BITS == 4 ? 4 : 2;      // groups per 128-byte stage
    constexpr int MTH = WARPS == 16 ? (MT + 1) / 2 : MT;   // m-tiles per warp
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte aligned start, reached by an offset from the shared array
    // itself so every access below stays a shared-memory access
    const uint32_t s0 = static_cast<uint32_t>(__cvta_generic_to_shared(smem_raw));
    uint8_t* smem = smem_raw + ((1024u - (s0 & 1023u)) & 1023u);
    uint8_t* ring = smem;
    RbBars* bars = reinterpret_cast<RbBars*>(smem + p.bar_off);
    volatile int* abort_flag = &bars->abort;
    const int warp_id = threadIdx.x >> 5;
    const int warp = warp_id & 7;               // column warp: columns warp, warp + 8, ...
    const int mi0 = (warp_id >> 3) * MTH;       // first m-tile of this warp
    const int lane = threadIdx.x & 31;
    const int SG = p.sg;
    const int RB = 16 * MT;                     // rows of a block (== 16 * p.tc)
    const int cbytes = RB * 128 * p.S;          // code bytes of a slot
    const uint32_t x_bytes = static_cast<uint32_t>(p.J * p.M * 128);
    // staged scale metadata per slot: g64 fp16 [RB][kRbSrow]; int8 preset
    // fp16 [RB][kRbSrowP8]; int4 preset sub-codes u8 [RB][4 J]
    const uint32_t s_bytes = !SSC ? 0u
                             : static_cast<uint32_t>(RB * (FMT == FMT_G64 ? kRbSrow * 2
                                                           : FMT == FMT_P8 ? kRbSrowP8 * 2 : p.srow));

    // Loads of the CTA's slot i (block blk, slot sl of the block) into ring slot r.
    auto issue_w = [&](int r, int blk, int sl) {
        uint8_t* dst = ring + r * p.slot_bytes;
        const int m = blk / p.bpm;
        const int row0 = (blk - m * p.bpm) * RB;
        const int st0 = sl * p.S;
        const uint64_t pol = l2_policy_evict_first();
        mbar_arrive_expect_tx(&bars->full[r], static_cast<uint32_t>(cbytes) + s_bytes + x_bytes);
        if (p.three_d) {
            tma_load_3d(dst, &p.tm_w[m], &bars->full[r], 0, row0, st0, pol);
        } else {
            for (int s = 0; s < p.S; ++s)
                tma_load_2d(dst + s * RB * 128, &p.tm_w[m], &bars->full[r], (st0 + s) * 128, row0, pol);
        }
        if constexpr (SSC) {
            // first element of the slot's metadata, rounded down to 16 bytes
            const int sx = FMT == FMT_G64 ? ((st0 * GPS) & ~7)
                           : FMT == FMT_P8 ? ((st0 * GPS * 4) & ~7)
                                           : st0 * GPS * 4;
            tma_load_2d(dst + p.s_off, &p.tm_s[m], &bars->full[r], sx, row0, pol);
        }
    };
    auto issue_x = [&](int r, int blk, int sl) {
        const int m = p.nx > 1 ? blk / p.bpm : 0;
        tma_load_3d(ring + r * p.slot_bytes + p.x_off, &p.tm_x[m], &bars->full[r], 0, 0, sl * p.J,
                    l2_policy_evict_last());
    };

    if (threadIdx.x == 0) {
        for (int r = 0; r < SG; ++r) {
            mbar_init(&bars->full[r], 1);
            bars->done[r] = 0;
            bars->issued_hi[r] = -1;
        }
        bars->abort = 0;
        fence_mbar_init();
        for (int m = 0; m < 3; ++m) {
            if (p.y[m] == nullptr) break;
            if (m < p.nx) tma_prefetch_desc(&p.tm_x[m]);
            tma_prefetch_desc(&p.tm_w[m]);
            if (SSC) tma_prefetch_desc(&p.tm_s[m]);
        }
        // codes and scales of the first block's first slots: they never
        // depend on the previous grid, so they go out before waiting on it
        const int n_pre = min(SG, p.slots);
        for (int r = 0; r < n_pre; ++r) {
            bars->issued_hi[r] = r;
            issue_w(r, blockIdx.x, r);
        }
    }
    __syncthreads();
    pdl_launch_dependents();
    pdl_wait();   // x (and y) may be used by the previous kernel
    if (threadIdx.x == 0) {
        const int n_pre = min(SG, p.slots);
        for (int r = 0; r < n_pre; ++r) issue_x(r, blockIdx.x, r);
    }

    const int g = lane >> 2;
    const int t = lane & 3;
    const int prow = phys_row<BITS>(g);
    // This warp's columns of a slot are j = warp + 8c: for int4 stage
    // warp/4 + 2c, group warp%4 of it; for int8 stage warp/2 + 4c, group
    // warp%2.  Every per-column offset below is a constant plus c strides.
    constexpr int CPS = kRbWarps / GPS;                 // stages between a warp's columns
    const int q0 = warp % GPS;
    int coff;
    if constexpr (BITS == 4)
        coff = prow * 128 + (((2 * q0 + (t >> 1)) ^ (prow & 7)) << 4) + ((t & 1) << 3);
    else
        coff = prow * 128 + (((4 * q0 + t) ^ (prow & 7)) << 4);
    const int code0 = (warp / GPS) * RB * 128 + coff;   // the warp's first column in a slot
    const int code_step = CPS * RB * 128;
    int xrow0[NT], xph[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int line = warp * p.M + min(nt * 8 + g, p.M - 1);
        xrow0[nt] = p.x_off + line * 128;
        xph[nt] = line & 7;                             // unchanged by the 8*M-line column stride
    }
    const int x_step = kRbWarps * p.M * 128;
    int gi = 0;                 // the CTA's slot index (over all its blocks)
    int r = 0;                  // its ring slot (gi % SG) and that slot's phase
    uint32_t ph = 0;
    bool dead = false;
    int kb = 0;                 // blocks done by this CTA
    for (int blk = blockIdx.x; blk < p.nblocks; blk += gridDim.x, ++kb) {
        const int m = blk / p.bpm;
        const int row0 = (blk - m * p.bpm) * RB;
        if (kb > 0 && threadIdx.x == 0) {
            // a later block: the ring was the previous block's reduction
            // buffer, so its first slots go out only now
            const int n_pre = min(SG, p.slots);
            int rq = r;
            for (int q = 0; q < n_pre; ++q) {
                bars->issued_hi[rq] = gi + q;
                issue_w(rq, blk, q);
                issue_x(rq, blk, q);
                if (++rq == SG) rq = 0;
            }
        }
        float acc[MTH][NT][4];
#pragma unroll
        for (int i = 0; i < MTH; ++i)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[i][nt][e] = 0.0f;
        for (int sl = 0; sl < p.slots; ++sl, ++gi) {
            if (!dead && !mbar_wait(&bars->full[r], ph, abort_flag, p.timeout_ns, p.status))
                dead = true;
            const int grp0 = sl * p.J;                  // first group of the slot
            int jn = p.groups - grp0;                   // group columns holding data
            if (jn > p.J) jn = p.J;
            if constexpr (FMT == FMT_P8) {
                if (!dead) {
                    const uint8_t* base = ring + r * p.slot_bytes;
                    for (int c = 0; warp + kRbWarps * c < jn; ++c) {
                        const uint8_t* cb = base + (warp / 2 + 4 * c) * RB * 128;
                        const uint8_t* cwa[4];
#pragma unroll
                        for (int jj = 0; jj < 4; ++jj)
                            cwa[jj] = cb + prow * 128 + ((((4 * (warp & 1) + jj) ^ (prow & 7))) << 4) + 4 * t;
                        const uint16_t* sp = reinterpret_cast<const uint16_t*>(base + p.s_off) +
                                             prow * kRbSrowP8 + 4 * (warp + kRbWarps * c);
                        int xr[NT];
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) xr[nt] = xrow0[nt] + c * x_step;
                        rb_column_p8<MT, NT>(cwa, sp, base, xr, xph, t, acc);
                    }
                }
            } else if constexpr (FMT == FMT_P4A) {
                if (!dead) {
                    const uint8_t* base = ring + r * p.slot_bytes;
                    for (int c = 0; warp + kRbWarps * c < jn; ++c) {
                        const int jcol = warp + kRbWarps * c;
                        const uint8_t* cb = base + (warp / 4 + 2 * c) * RB * 128 + prow * 128 + 4 * t;
                        const int q = warp & 3;
                        const uint8_t* cwa = cb + (((2 * q) ^ (prow & 7)) << 4);
                        const uint8_t* cwb = cb + (((2 * q + 1) ^ (prow & 7)) << 4);
                        const uint8_t* subp = base + p.s_off + prow * p.srow + 4 * jcol;
                        const uint32_t* supp = p.sup[m] + (row0 + prow) * static_cast<int64_t>(p.nsb) +
                                               (grp0 + jcol) / 4;
                        int xr[NT];
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) xr[nt] = xrow0[nt] + c * x_step;
                        rb_column_p4a<MT, NT>(cwa, cwb, subp, p.srow, supp, p.nsb, row0 + prow, p.N,
                                              base, xr, xph, t, acc);
                    }
                }
            } else
            if (!dead) {
                const uint8_t* base = ring + r * p.slot_bytes;
                const uint8_t* cbase = base + code0;
                const uint16_t* sbase = reinterpret_cast<const uint16_t*>(base + p.s_off) +
                                        prow * kRbSrow + (grp0 & 7) + warp;
                int c = 0;
                // (pairs only for one token tile: larger M takes one column
                // per warp and slot, and the registers go to its tiles)
                if constexpr (NT == 1)
                for (; warp + kRbWarps * (c + 1) < jn; c += 2) {
                    const uint8_t* cw0[2] = {cbase + c * code_step, cbase + (c + 1) * code_step};
                    const uint16_t* sp[2] = {sbase + kRbWarps * c, sbase + kRbWarps * (c + 1)};
                    int xr[2][NT];
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        xr[0][nt] = xrow0[nt] + c * x_step;
                        xr[1][nt] = xrow0[nt] + (c + 1) * x_step;
                    }
                    const int gr[2] = {grp0 + warp + kRbWarps * c, grp0 + warp + kRbWarps * (c + 1)};
                    rb_columns<BITS, MTH, NT, 2, SSC, MT>(cw0, sp, base, xr, xph, t, acc, p.scales[m],
                                                          row0 + prow, p.groups, gr, p.N, mi0);
                }
                for (; warp + kRbWarps * c < jn; ++c) {
                    const uint8_t* cw0[1] = {cbase + c * code_step};
                    const uint16_t* sp[1] = {sbase + kRbWarps * c};
                    int xr[1][NT];
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) xr[0][nt] = xrow0[nt] + c * x_step;
                    const int gr[1] = {grp0 + warp + kRbWarps * c};
                    rb_columns<BITS, MTH, NT, 1, SSC, MT>(cw0, sp, base, xr, xph, t, acc, p.scales[m],
                                                          row0 + prow, p.groups, gr, p.N, mi0);
                }
            }
            // ---- release the slot; the last warp out refills it with the
            // block's slot sl + SG (later blocks refill after their reduction)
            __syncwarp();
            if (lane == 0) {
                __threadfence_block();
                const int prev = atomicAdd(&bars->done[r], 1);
                if (prev == WARPS - 1) {
                    __threadfence_block();
                    bars->done[r] = 0;
                    const int nsl = sl + SG;
                    if (nsl < p.slots && !dead && *abort_flag == 0) {
                        bars->issued_hi[r] = gi + SG;
                        // order every warp's generic reads of the slot before
                        // the asynchronous writes into it
                        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                        issue_w(r, blk, nsl);
                        issue_x(r, blk, nsl);
                    }
                }
            }
            if (++r == SG) {
                r = 0;
                ph ^= 1u;
            }
        }
        // ---- the block's sums: warps deposit, then add in warp order
        __syncthreads();   // every warp is done reading the ring
        float* red = reinterpret_cast<float*>(ring);
        const int RS = p.red_stride;                   // floats per (warp, token)
        for (int nt0 = 0; nt0 < NT; ++nt0) {
            // round nt0: tokens [8 nt0, 8 nt0 + 8)
#pragma unroll
            for (int i = 0; i < MTH; ++i)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    if (MTH != MT && mi0 + i >= MT) break;   // (odd split)
                    const int tl = 2 * t + (e & 1);
                    const int rr = 16 * (mi0 + i) + 8 * (e >> 1) + prow;
                    float v = 0.0f;
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
                        if (nt == nt0) v = acc[i][nt][e];
                    red[(warp * 8 + tl) * RS + rr] = v;
                }
            __syncthreads();
            const int ntok = min(8, p.M - 8 * nt0);
            for (int o = threadIdx.x; o < ntok * RB; o += WARPS * 32) {
                const int tl = o / RB;
                const int rr = o - tl * RB;
                float v = 0.0f;
#pragma unroll
                for (int w = 0; w < kRbWarps; ++w) v += red[(w * 8 + tl) * RS + rr];
                if (p.epi == 1) {
                    v = fmaxf(v, 0.0f);
                    v = v * v;
                }
                const int n = row0 + rr;
                if (n < p.N && !dead && *abort_flag == 0) {
                    const int64_t at = static_cast<int64_t>(8 * nt0 + tl) * p.N + n;
                    if (p.yh)
                        static_cast<__half*>(p.y[m])[at] = __float2half_rn(v);
                    else
                        static_cast<float*>(p.y[m])[at] = v;
                }
            }
            __syncthreads();
        }
    }
    // After a timeout some issued copies may never have been waited for:
    // wait (bounded) for the last one of every slot before the CTA exits.
    __syncthreads();
    if (threadIdx.x == 0 && *abort_flag) {
        int dummy_abort = 0;
        for (int r = 0; r < SG; ++r) {
            const int il = bars->issued_hi[r];
            if (il >= 0)
                mbar_wait(&bars->full[r], static_cast<uint32_t>(il / SG) & 1, &dummy_abort,
                          p.timeout_ns, p.status);
        }
    }
}

// ------------------------------------------------------------- launcher --

// How a decode product of this shape is cut for the row-block kernel.
struct RbPlan {
    int tc, bpm, nblocks, grid, stages, S, J, slots, sg, srow;
    int slot_bytes, s_off, x_off, bar_off, red_stride, smem;
    bool three_d;
};

template <int FMT, int BITS, int MT, int NT, bool SSC, int WARPS>
inline cudaError_t rb_launch_w(RbParams& prm, const RbPlan& P, const uint16_t* const* xs,
                               const void* const* codes, int nmat, cudaStream_t s) {
    auto kern = gemv_rb_kernel<FMT, BITS, MT, NT, SSC, WARPS>;
    static bool attr_set[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!attr_set[dev]) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    const int RB = 16 * MT;
    const uint64_t row_bytes = static_cast<uint64_t>(prm.K) * BITS / 8;
    for (int i = 0; i < nmat; ++i) {
        const bool okw =
            P.three_d
                ? make_tmap_3d(&prm.tm_w[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, codes[i], 128,
                               static_cast<uint64_t>(prm.N), static_cast<uint64_t>(P.stages),
                               row_bytes, 128, 128, static_cast<uint32_t>(RB),
                               static_cast<uint32_t>(P.S), CU_TENSOR_MAP_SWIZZLE_128B)
                : make_tmap_2d(&prm.tm_w[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, codes[i], row_bytes,
                               static_cast<uint64_t>(prm.N), row_bytes, 128,
                               static_cast<uint32_t>(RB), CU_TENSOR_MAP_SWIZZLE_128B);
        if (!okw) return cudaErrorInvalidValue;
        // the staged metadata: g64 scales fp16 [N, K/64]; int8 preset scales
        // fp16 [N, K/16]; int4 preset sub-codes u8 [N, K/16] ((a, b) pairs)
        const uint64_t mlen = FMT == FMT_G64 ? static_cast<uint64_t>(prm.groups)
                                             : static_cast<uint64_t>(prm.K) / 16;
        const bool okm =
            FMT == FMT_P4A
                ? make_tmap_2d(&prm.tm_s[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, prm.scales[i], mlen,
                               static_cast<uint64_t>(prm.N), mlen, static_cast<uint32_t>(P.srow),
                               static_cast<uint32_t>(RB), CU_TENSOR_MAP_SWIZZLE_NONE)
                : make_tmap_2d(&prm.tm_s[i], CU_TENSOR_MAP_DATA_TYPE_UINT16, prm.scales[i], mlen,
                               static_cast<uint64_t>(prm.N), mlen * 2, static_cast<uint32_t>(P.srow),
                               static_cast<uint32_t>(RB), CU_TENSOR_MAP_SWIZZLE_NONE);
        if (prm.ssc && !okm) return cudaErrorInvalidValue;
    }
    for (int i = 0; i < prm.nx; ++i)
        if (!make_tmap_3d(&prm.tm_x[i], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, xs[i], 64,
                          static_cast<uint64_t>(prm.M), static_cast<uint64_t>(prm.groups),
                          static_cast<uint64_t>(prm.K) * 2, 128, 64, static_cast<uint32_t>(prm.M),
                          static_cast<uint32_t>(P.J), CU_TENSOR_MAP_SWIZZLE_128B))
            return cudaErrorInvalidValue;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(P.grid), 1, 1);
    cfg.blockDim = dim3(WARPS * 32, 1, 1);
    cfg.dynamicSmemBytes = static_cast<size_t>(P.smem);
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
    return cudaLaunchKernelEx(&cfg, kern, static_cast<const RbParams&>(prm));
}

// 16 warps (two halves splitting each block's m-tiles) measured faster only
// for int4 at M <= 8 on rows of <= 2048 k with blocks of >= 3 m-tiles (fused
// R/K/V 3 x 2048 x 2048: 4.08 -> 3.68 us; 8192 x 2048: 4.67 -> 4.22 us); with
// longer rows, fewer m-tiles or int8 the 8-warp form is faster.
template <int FMT, int BITS, int MT, int NT, bool SSC>
inline cudaError_t rb_launch(RbParams& prm, const RbPlan& P, const uint16_t* const* xs,
                             const void* const* codes, int nmat, cudaStream_t s) {
    if constexpr (FMT == FMT_G64 && BITS == 4 && NT == 1 && MT >= 3) {
        if (prm.K <= 2048) return rb_launch_w<FMT, BITS, MT, NT, SSC, 16>(prm, P, xs, codes, nmat, s);
    }
    return rb_launch_w<FMT, BITS, MT, NT, SSC, 8>(prm, P, xs, codes, nmat, s);
}

template <int FMT, int BITS, int NT, bool SSC>
inline cudaError_t rb_dispatch_mt(RbParams& prm, const RbPlan& P, const uint16_t* const* x,
                                  const void* const* codes, int nmat, cudaStream_t s) {
    // preset blocks with four token tiles stay at 4 m-tiles (taller ones spill)
    constexpr int kMaxMT = FMT != FMT_G64 && NT == 4 ? 4 : 8;
    switch (P.tc) {
        case 1: return rb_launch<FMT, BITS, 1, NT, SSC>(prm, P, x, codes, nmat, s);
        case 2: return rb_launch<FMT, BITS, 2, NT, SSC>(prm, P, x, codes, nmat, s);
        case 3: return rb_launch<FMT, BITS, 3, NT, SSC>(prm, P, x, codes, nmat, s);
        case 4: return rb_launch<FMT, BITS, 4, NT, SSC>(prm, P, x, codes, nmat, s);
        default: break;
    }
    if constexpr (kMaxMT == 8) {
        switch (P.tc) {
            case 5: return rb_launch<FMT, BITS, 5, NT, SSC>(prm, P, x, codes, nmat, s);
            case 6: return rb_launch<FMT, BITS, 6, NT, SSC>(prm, P, x, codes, nmat, s);
            case 7: return rb_launch<FMT, BITS, 7, NT, SSC>(prm, P, x, codes, nmat, s);
            case 8: return rb_launch<FMT, BITS, 8, NT, SSC>(prm, P, x, codes, nmat, s);
            default: break;
        }
    }
    return cudaErrorInvalidValue;
}

// One translation unit per format (and bits) instantiates the kernels:
// launches the kernel for prm.M's token tiles and the plan's block height.
cudaError_t rb_run_g64_4(RbParams& prm, const RbPlan& P, const uint16_t* const* x,
                         const void* const* codes, int nmat, cudaStream_t s);
cudaError_t rb_run_g64_8(RbParams& prm, const RbPlan& P, const uint16_t* const* x,
                         const void* const* codes, int nmat, cudaStream_t s);
cudaError_t rb_run_p8(RbParams& prm, const RbPlan& P, const uint16_t* const* x,
                      const void* const* codes, int nmat, cudaStream_t s);
cudaError_t rb_run_p4a(RbParams& prm, const RbPlan& P, const uint16_t* const* x,
                       const void* const* codes, int nmat, cudaStream_t s);

}  // namespace rq
