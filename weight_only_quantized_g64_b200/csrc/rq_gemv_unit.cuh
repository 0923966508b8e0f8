// rq_gemv_unit.cuh -- the decode product's inner step: one unit (16*MT
// weight rows x one 128-byte code stage) of one warp, from shared memory into
// fp32 accumulators.
//
// Thread (g = lane/4, t = lane%4) owns, per group of 64 k, the 16 k
// [16t, 16t+16) of rows g and g+8 of each m-tile.  MMA k-slot sigma of step j
// maps to one of those k, the same map on the A (weights) and B (x) side, so
// the sum over k is unchanged and every thread's codes and x are contiguous in
// memory.  Codes become exact fp16 values in registers (bit placement plus one
// exact fp16 operation: Kim et al., "Who Says Elephants Can't Run?",
// arXiv:2211.10017); mma.sync.m16n8k16 sums x * code for one group in fp32;
// the group's scale is applied in fp32 (acc = fma(partial, s, acc)).
#pragma once

#include <cuda_fp16.h>
#include <cstdint>

namespace rq {

__device__ __forceinline__ uint4 lds128(const uint8_t* p) { return *reinterpret_cast<const uint4*>(p); }
__device__ __forceinline__ uint2 lds64(const uint8_t* p) { return *reinterpret_cast<const uint2*>(p); }

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
// interleave independent accumulation chains (different m-tiles / n-tiles).
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


// The math of one group of 64 k for one warp: x fragments xv[nt] (positions
// 16t .. 16t+15 of token nt*8+g, two 16-byte chunks), code words cw[i][h]
// (this thread's 16 k of row 8h + g of m-tile i) and fp32 scales sv[i][h].
// Codes become exact fp16 A registers, 4 MMA steps per n-tile sum x * code in
// fp32, and the group's scale is applied in fp32.
template <int BITS, int MT, int NT>
__device__ __forceinline__ void gv_group_math(const uint4 (&xv)[NT][2],
                                              const uint32_t (&cw)[MT][2][BITS == 4 ? 2 : 4],
                                              const float (&sv)[MT][2], float (&acc)[MT][NT][4]) {
    constexpr bool PERM = BITS == 4 && 2 * MT >= NT;   // permuted pair order (x permuted per group)
    // x fragments of this group: token nt*8+g, positions 16t .. 16t+15
    uint32_t b[NT][4][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const uint32_t X[8] = {xv[nt][0].x, xv[nt][0].y, xv[nt][0].z, xv[nt][0].w,
                               xv[nt][1].x, xv[nt][1].y, xv[nt][1].z, xv[nt][1].w};
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            if constexpr (PERM) {
                // step jj pairs (p0,p4),(p1,p5) or (p2,p6),(p3,p7) of word jj/2
                const int wb = (jj >> 1) * 4 + (jj & 1);
                b[nt][jj][0] = __byte_perm(X[wb], X[wb + 2], 0x5410);
                b[nt][jj][1] = __byte_perm(X[wb], X[wb + 2], 0x7632);
            } else {
                b[nt][jj][0] = X[2 * jj];
                b[nt][jj][1] = X[2 * jj + 1];
            }
        }
    }
#pragma unroll
    for (int i = 0; i < MT; ++i) {
        uint32_t A[4][4];   // [step][a-reg]
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            if constexpr (BITS == 4) {
                uint32_t P0[4], P1[4];
                if constexpr (PERM) {
                    i4_word_to_pairs_perm(cw[i][h][0], P0);
                    i4_word_to_pairs_perm(cw[i][h][1], P1);
                } else {
                    i4_word_to_pairs_nat(cw[i][h][0], P0);
                    i4_word_to_pairs_nat(cw[i][h][1], P1);
                }
                // step jj: a0a1 (h = 0) / a2a3 (h = 1), and a4a5 / a6a7
                A[0][h] = P0[0]; A[0][h + 2] = P0[1];
                A[1][h] = P0[2]; A[1][h + 2] = P0[3];
                A[2][h] = P1[0]; A[2][h + 2] = P1[1];
                A[3][h] = P1[2]; A[3][h + 2] = P1[3];
            } else {
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    uint32_t Q[2];
                    i8_word_to_pairs(cw[i][h][jj], Q);
                    A[jj][h] = Q[0];
                    A[jj][h + 2] = Q[1];
                }
            }
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            float part[4];
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) mma16816(part, A[jj], b[nt][jj][0], b[nt][jj][1], jj == 0);
            acc[i][nt][0] = fmaf(part[0], sv[i][0], acc[i][nt][0]);
            acc[i][nt][1] = fmaf(part[1], sv[i][0], acc[i][nt][1]);
            acc[i][nt][2] = fmaf(part[2], sv[i][1], acc[i][nt][2]);
            acc[i][nt][3] = fmaf(part[3], sv[i][1], acc[i][nt][3]);
        }
    }
}

// One unit of one warp.  MT = NMAT * MTM m-tiles: m-tile i is rows
// [16 (i % MTM), +16) of matrix i / MTM.
//   wt    codes of the stage, matrix 0: [16*MTM rows][128 B], SWIZZLE_128B
//         (TMA layout); matrix m's block starts cmstr bytes further per m
//   sc    scales of the stage, matrix 0: rows of SROW fp16, offset to the
//         stage's first group (when ssc); matrix m's rows start SMSTR bytes
//         further per m
//   xt    x of the load group: [groups][M tokens][64 fp16], SWIZZLE_128B
//         (TMA layout: 128-byte row r's 16-byte chunks permuted by r & 7);
//         the unit's groups start at group row gq0; xtok[nt] = this thread's
//         token nt*8+g (any valid token for tokens >= M: those columns of the
//         MMA are never stored)
//   prow  phys_row<BITS>(g)
//   ssc   scales are staged; otherwise read from global memory (ragged K:
//         groups past the end get scale 0), needing scales/row0/st/N/groups,
//         row0 = the global row of the warp's first m-tile in each matrix
// The shared-memory operands of QB groups at a time are loaded into registers
// first (one burst of loads, so their latency is paid once per batch), then
// the batch is unpacked and multiplied.
template <int BITS, int MT, int NT, int MTM, int SROW, int SMSTR>
__device__ __forceinline__ void gv_unit(const uint8_t* wt, int cmstr, const uint8_t* sc,
                                        const uint8_t* xt, int gq0, int M, const int (&xtok)[NT],
                                        int prow, int t, bool ssc,
                                        const uint16_t* const* scales, int row0, int st, int N,
                                        int groups, float (&acc)[MT][NT][4]) {
    constexpr int GPS = BITS == 4 ? 4 : 2;
    constexpr int CW = BITS == 4 ? 2 : 4;              // code words per row and group
    constexpr int QB = MT * NT <= 2 ? GPS : (MT * NT <= 4 ? 2 : 1);   // groups per load batch
#pragma unroll
    for (int q0 = 0; q0 < GPS; q0 += QB) {
        // ---------------------------------------------------- load burst --
        uint4 xv[QB][NT][2];
        uint32_t cw[QB][MT][2][CW];
        uint32_t sw[MT][2][(QB + 1) / 2];               // packed fp16 scales of the batch
#pragma unroll
        for (int qq = 0; qq < QB; ++qq) {
            const int q = q0 + qq;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                // positions 16t .. 16t+15 of the group: chunks 2t and 2t+1
                const int row = (gq0 + q) * M + xtok[nt];
                const uint8_t* xr = xt + row * 128;
                const int c0 = ((2 * t) ^ (row & 7)) << 4;
                xv[qq][nt][0] = lds128(xr + c0);
                xv[qq][nt][1] = lds128(xr + (c0 ^ 16));
            }
            // this thread's codes of group q in row `prow` of the stage
            // (rows 16i + 8h + prow share the swizzle phase prow & 7)
            int coff;
            if constexpr (BITS == 4)
                coff = prow * 128 + (((2 * q + (t >> 1)) ^ (prow & 7)) << 4) + ((t & 1) << 3);
            else
                coff = prow * 128 + (((4 * q + t) ^ (prow & 7)) << 4);
#pragma unroll
            for (int i = 0; i < MT; ++i)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint8_t* cp =
                        wt + (i / MTM) * cmstr + coff + (16 * (i % MTM) + 8 * h) * 128;
                    if constexpr (BITS == 4) {
                        const uint2 v = lds64(cp);
                        cw[qq][i][h][0] = v.x;
                        cw[qq][i][h][1] = v.y;
                    } else {
                        const uint4 v = lds128(cp);
                        cw[qq][i][h][0] = v.x; cw[qq][i][h][1] = v.y;
                        cw[qq][i][h][2] = v.z; cw[qq][i][h][3] = v.w;
                    }
                }
        }
        if (ssc) {
#pragma unroll
            for (int i = 0; i < MT; ++i)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint8_t* sp =
                        sc + (i / MTM) * SMSTR + ((16 * (i % MTM) + 8 * h + prow) * SROW + q0) * 2;
                    if constexpr (QB == 4) {
                        const uint2 v = lds64(sp);
                        sw[i][h][0] = v.x;
                        sw[i][h][1] = v.y;
                    } else if constexpr (QB == 2) {
                        sw[i][h][0] = *reinterpret_cast<const uint32_t*>(sp);
                    } else {
                        sw[i][h][0] = *reinterpret_cast<const uint16_t*>(sp);
                    }
                }
        } else {
            // ragged K: the stage may run past the last group (scale 0)
#pragma unroll
            for (int i = 0; i < MT; ++i)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int m = i / MTM;
                    const int n = row0 + 16 * (i % MTM) + 8 * h + prow;
                    uint16_t v[QB];
#pragma unroll
                    for (int qq = 0; qq < QB; ++qq) {
                        const int grp = st * GPS + q0 + qq;
                        v[qq] = (n < N && grp < groups)
                                    ? __ldg(scales[m] + static_cast<int64_t>(n) * groups + grp)
                                    : static_cast<uint16_t>(0);
                    }
#pragma unroll
                    for (int w2 = 0; w2 < (QB + 1) / 2; ++w2)
                        sw[i][h][w2] = static_cast<uint32_t>(v[2 * w2]) |
                                       (2 * w2 + 1 < QB ? (static_cast<uint32_t>(v[2 * w2 + 1]) << 16) : 0u);
                }
        }
        // ---------------------------------------------------- math --------
#pragma unroll
        for (int qq = 0; qq < QB; ++qq) {
            float sv[MT][2];
#pragma unroll
            for (int i = 0; i < MT; ++i)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint32_t w2 = sw[i][h][qq >> 1];
                    sv[i][h] = __half2float(__ushort_as_half(
                        static_cast<unsigned short>((qq & 1) ? (w2 >> 16) : (w2 & 0xFFFFu))));
                }
            gv_group_math<BITS, MT, NT>(xv[qq], cw[qq], sv, acc);
        }
    }
}

// One warp's share of one stage when WK warps split the stage's groups:
// groups q = kw, kw + WK, ... of the stage (GPS / WK of them).  Operands as
// for gv_unit with one matrix (MTM = MT); scales, when staged, are rows of
// SROW fp16 starting at the stage's first group.
template <int BITS, int MT, int NT, int WK, int SROW>
__device__ __forceinline__ void gv_unit_strided(const uint8_t* wt, const uint8_t* sc,
                                                const uint8_t* xt, int gq0, int kw, int M,
                                                const int (&xtok)[NT], int prow, int t, bool ssc,
                                                const uint16_t* scales, int row0, int st, int N,
                                                int groups, float (&acc)[MT][NT][4]) {
    constexpr int GPS = BITS == 4 ? 4 : 2;
    constexpr int NQ = GPS / WK;                       // groups of the stage for this warp
    constexpr int CW = BITS == 4 ? 2 : 4;
    constexpr int QB = NQ < 2 ? NQ : (MT * NT <= 4 ? 2 : 1);
    static_assert(GPS % WK == 0 && NQ % QB == 0, "warps must split the stage's groups evenly");
#pragma unroll
    for (int qb = 0; qb < NQ; qb += QB) {
        uint4 xv[QB][NT][2];
        uint32_t cw[QB][MT][2][CW];
        float sv[QB][MT][2];
#pragma unroll
        for (int qq = 0; qq < QB; ++qq) {
            const int q = kw + WK * (qb + qq);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int row = (gq0 + q) * M + xtok[nt];
                const uint8_t* xr = xt + row * 128;
                const int c0 = ((2 * t) ^ (row & 7)) << 4;
                xv[qq][nt][0] = lds128(xr + c0);
                xv[qq][nt][1] = lds128(xr + (c0 ^ 16));
            }
            int coff;
            if constexpr (BITS == 4)
                coff = prow * 128 + (((2 * q + (t >> 1)) ^ (prow & 7)) << 4) + ((t & 1) << 3);
            else
                coff = prow * 128 + (((4 * q + t) ^ (prow & 7)) << 4);
#pragma unroll
            for (int i = 0; i < MT; ++i)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint8_t* cp = wt + coff + (16 * i + 8 * h) * 128;
                    if constexpr (BITS == 4) {
                        const uint2 v = lds64(cp);
                        cw[qq][i][h][0] = v.x;
                        cw[qq][i][h][1] = v.y;
                    } else {
                        const uint4 v = lds128(cp);
                        cw[qq][i][h][0] = v.x; cw[qq][i][h][1] = v.y;
                        cw[qq][i][h][2] = v.z; cw[qq][i][h][3] = v.w;
                    }
                    uint16_t s16;
                    if (ssc) {
                        s16 = *reinterpret_cast<const uint16_t*>(
                            sc + ((16 * i + 8 * h + prow) * SROW + q) * 2);
                    } else {
                        // ragged K: the stage may run past the last group (scale 0)
                        const int n = row0 + 16 * i + 8 * h + prow;
                        const int grp = st * GPS + q;
                        s16 = (n < N && grp < groups)
                                  ? __ldg(scales + static_cast<int64_t>(n) * groups + grp)
                                  : static_cast<uint16_t>(0);
                    }
                    sv[qq][i][h] = __half2float(__ushort_as_half(s16));
                }
        }
#pragma unroll
        for (int qq = 0; qq < QB; ++qq) gv_group_math<BITS, MT, NT>(xv[qq], cw[qq], sv[qq], acc);
    }
}

}  // namespace rq
