/*
 * rqo.c -- the ORACLE for weight-only, group-64, symmetric int4/int8
 * quantized projections.  Plain, slow, scalar C.  Test infrastructure only:
 * nothing in the product library links, includes or calls this file.  Only
 * the test suite, the smoke check and the CPU-baseline leg of the benchmark
 * may load it.
 *
 * What it follows:
 *   - "Hakureirm/rwkv7-sglang-w4gptq-1.5b" model card, opening summary and
 *     "Format & loading (important)": weights are stored group-wise with
 *     GROUP = 64, symmetric (no zero point), as packed int4 codes (.qweight)
 *     plus one scale per group (.scale); the calibration-free variant is plain
 *     round-to-nearest (RTN); the kernel's output equals a product with the
 *     offline-dequantised weight.
 *   - same card, "Accuracy warning": the int8 "w8g64" tier uses the same
 *     group of 64 with 8-bit codes.
 *   - "RWKV-7 Quantization Toolkit" (rwkv-quant-nv 1.2.1), "Key Design":
 *     products are taken directly on the quantized weights; no dequantised
 *     weight matrix exists on the inference path.  The oracle is the
 *     definition, so it may dequantise.
 *
 * Readings where the pages are silent (each one is listed in the design notes):
 *   - the group runs along the reduction axis K: 64 consecutive k of one
 *     output row n of W[N, K];
 *   - scale: s32 = amax / qmax as one IEEE fp32 division, then s16 =
 *     round-to-nearest-even of s32 to fp16; the stored scale is s16;
 *   - codes are computed against the stored scale: c = clamp(rint(w / s16),
 *     -qmax, qmax) with w / s16 one IEEE fp32 division and rint rounding half
 *     to even;  qmax = 7 (int4) or 127 (int8);
 *   - a group whose s16 is zero (all-zero group or an underflowing amax) gets
 *     codes 0;
 *   - a group holding a non-finite weight gets scale 0x7E00 (fp16 NaN) and
 *     codes 0, status NONFINITE;  a group whose s16 overflows to +inf keeps
 *     scale 0x7C00 and codes 0, status RANGE;
 *   - int4 packing: byte j of a row holds k = 2j in its low nibble and
 *     k = 2j + 1 in its high nibble, 4-bit two's complement; int8 codes are
 *     plain signed bytes; scales are row-major [N, K/64].
 *   - products: y[m, n] = sum_k x[m, k] * c[n, k] * s16[n, k/64] in fp64, with
 *     x given as fp16 bit patterns; the per-output error budget is
 *     B[m, n] = sum_k |x[m, k]| * |c[n, k] * s16[n, k/64]|.
 *
 * Build: gcc -O2 -fPIC -shared -fopenmp -ffp-contract=off -fno-fast-math.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define RQO_GROUP 64

/* status values: the same numbering as the library's public header, written
 * out here on purpose (the oracle includes no header of the product). */
enum { RQO_OK = 0, RQO_ERR_NONFINITE = 5, RQO_ERR_RANGE = 6 };

/* ---------------------------------------------------------------- fp16 --- */

/* fp32 -> IEEE binary16, round to nearest, ties to even.  Written from the
 * IEEE 754 binary16 definition: 1 sign bit, 5 exponent bits (bias 15),
 * 10 fraction bits; subnormals below 2^-14; overflow to infinity. */
uint16_t rqo_f32_to_f16(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
    uint32_t exp = (u >> 23) & 0xFFu;
    uint32_t man = u & 0x7FFFFFu;

    if (exp == 0xFFu) {                      /* inf or NaN */
        if (man == 0) return (uint16_t)(sign | 0x7C00u);
        return (uint16_t)(sign | 0x7E00u);   /* quiet NaN */
    }
    int e = (int)exp - 127;                  /* unbiased exponent */
    if (exp == 0) return sign;               /* fp32 zero/subnormal: < 2^-126, rounds to 0 */

    uint32_t m = man | 0x800000u;            /* 24-bit significand, value m * 2^(e-23) */
    if (e > 15) return (uint16_t)(sign | 0x7C00u);

    int shift;                               /* right shift applied to m */
    uint32_t hexp;                           /* biased fp16 exponent before rounding */
    if (e >= -14) {                          /* normal range: keep 11 bits */
        shift = 13;
        hexp = (uint32_t)(e + 15);
    } else {                                 /* subnormal: value = q * 2^-24 */
        shift = 13 + (-14 - e);
        hexp = 0;
        if (shift > 24) return sign;         /* below half the smallest subnormal */
    }
    uint32_t q = m >> shift;
    uint32_t rem = m & ((1u << shift) - 1u);
    uint32_t half = 1u << (shift - 1);
    if (rem > half || (rem == half && (q & 1u))) q += 1u;

    if (hexp == 0) {
        /* q counts units of 2^-24; q == 0x400 is the smallest normal, which
         * the bit pattern below encodes correctly by itself */
        return (uint16_t)(sign | q);
    }
    /* q holds 1.fraction in 11 bits, possibly carried to 0x800 */
    if (q == 0x800u) { q = 0x400u; hexp += 1; }
    if (hexp >= 31) return (uint16_t)(sign | 0x7C00u);
    return (uint16_t)(sign | (hexp << 10) | (q & 0x3FFu));
}

/* IEEE binary16 -> double, exact. */
double rqo_f16_to_f64(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int exp = (h >> 10) & 0x1F;
    int man = h & 0x3FF;
    double v;
    if (exp == 0x1F) v = man ? NAN : INFINITY;
    else if (exp == 0) v = ldexp((double)man, -24);
    else v = ldexp((double)(man | 0x400), exp - 25);
    return sign ? -v : v;
}

/* ------------------------------------------------------------ quantize --- */

static int qmax_of(int bits) { return bits == 4 ? 7 : 127; }

/* Store code c (|c| <= qmax) for element (n, k) in the packed layout. */
static void put_code(uint8_t *codes, int64_t K, int bits, int64_t n, int64_t k, int c)
{
    if (bits == 8) {
        codes[n * K + k] = (uint8_t)(int8_t)c;
    } else {
        uint8_t *b = &codes[n * (K / 2) + k / 2];
        uint8_t nib = (uint8_t)(c & 0xF);
        if (k % 2 == 0) *b = (uint8_t)((*b & 0xF0u) | nib);
        else            *b = (uint8_t)((*b & 0x0Fu) | (nib << 4));
    }
}

/* Read back code (n, k) from the packed layout. */
int rqo_get_code(const uint8_t *codes, int64_t K, int bits, int64_t n, int64_t k)
{
    if (bits == 8) return (int)(int8_t)codes[n * K + k];
    uint8_t b = codes[n * (K / 2) + k / 2];
    int nib = (k % 2 == 0) ? (b & 0xF) : (b >> 4);
    return nib >= 8 ? nib - 16 : nib;
}

/* RTN quantization of one group of 64 weights; returns a status. */
static int quantize_group(const float *w, int bits, uint16_t *scale_out, int *c_out)
{
    const int qmax = qmax_of(bits);
    int i;
    for (i = 0; i < RQO_GROUP; i++) {
        if (!isfinite(w[i])) {
            *scale_out = 0x7E00u;
            for (i = 0; i < RQO_GROUP; i++) c_out[i] = 0;
            return RQO_ERR_NONFINITE;
        }
    }
    /* step 1: amax = max |w| (exact in fp32) */
    float amax = 0.0f;
    for (i = 0; i < RQO_GROUP; i++) {
        float a = fabsf(w[i]);
        if (a > amax) amax = a;
    }
    /* step 2: s32 = amax / qmax, one IEEE fp32 division */
    volatile float s32 = amax / (float)qmax;
    /* step 3: s16 = fp16(s32), round to nearest even */
    uint16_t s16 = rqo_f32_to_f16(s32);
    *scale_out = s16;
    /* step 4: codes against the stored scale */
    float sf = (float)rqo_f16_to_f64(s16);
    if (s16 == 0x7C00u) {
        for (i = 0; i < RQO_GROUP; i++) c_out[i] = 0;
        return RQO_ERR_RANGE;
    }
    if (sf == 0.0f) {
        for (i = 0; i < RQO_GROUP; i++) c_out[i] = 0;
        return RQO_OK;
    }
    for (i = 0; i < RQO_GROUP; i++) {
        volatile float t = w[i] / sf;        /* IEEE fp32 division */
        float r = rintf(t);                  /* half to even (default mode) */
        if (r > (float)qmax) r = (float)qmax;
        if (r < (float)-qmax) r = (float)-qmax;
        c_out[i] = (int)r;
    }
    return RQO_OK;
}

/* Quantize W[N, K] (fp32, row-major).  Writes codes (N*K*bits/8 bytes) and
 * scales (N*(K/64) fp16 bit patterns).  Returns the highest-priority status
 * seen: NONFINITE over RANGE over OK.  K must be a multiple of 64 and bits
 * 4 or 8; the caller checks. */
int rqo_quantize_g64(const float *W, int64_t N, int64_t K, int bits,
                     uint8_t *codes, uint16_t *scales)
{
    const int64_t G = K / RQO_GROUP;
    int status = RQO_OK;
    int64_t n;
#pragma omp parallel for schedule(static) reduction(max : status)
    for (n = 0; n < N; n++) {
        int c[RQO_GROUP];
        int64_t g;
        for (g = 0; g < G; g++) {
            int st = quantize_group(&W[n * K + g * RQO_GROUP], bits, &scales[n * G + g], c);
            int64_t i;
            for (i = 0; i < RQO_GROUP; i++) put_code(codes, K, bits, n, g * RQO_GROUP + i, c[i]);
            if (st > status) status = st;
        }
    }
    /* NONFINITE (5) must win over RANGE (6) */
    if (status != RQO_OK) {
        int64_t i, total = N * G;
        for (i = 0; i < total; i++) if (scales[i] == 0x7E00u) return RQO_ERR_NONFINITE;
    }
    return status;
}

/* --------------------------------------------- E[x^2]-weighted search --- */
/*
 * "rwkv-quant: uma matriz em bf16 elimina 39% das perdas na quantização do
 * RWKV-7 2.9B", section "Dois presets e seis tamanhos": in both presets the
 * groups' scale (and, for the asymmetric layout, offset) is chosen by a
 * search weighted by E[x^2], the mean square of the input channel's
 * activation.  Here, on the symmetric g64 grid of rqo_quantize_g64, with the
 * readings the page leaves open:
 *   - candidates: scale factors f[0..nf) given by the caller; candidate j
 *     uses s32 = fp32(amax * f[j]) / qmax (one fp32 multiply, one fp32
 *     division), s16 = fp16_rn(s32), and codes c = clamp(rint(w / s16))
 *     exactly as RTN does (f = 1 is RTN);
 *   - criterion: err_j = sum over the group's 64 k, in k order, of
 *     e2[k] * (d * d) with d = w - c * s16, every operation one fp32
 *     rounding (t = c * s16, d = w - t, q = d * d, p = e2 * q, err = err + p);
 *   - the candidate with the smallest err_j wins; on equal err_j the earlier
 *     candidate wins; a candidate whose s16 overflows is never chosen;
 *   - e2 is the caller's vector of E[x^2] per input channel (length K,
 *     finite, >= 0); non-finite weights and an overflow of every candidate
 *     give the statuses and outputs of RTN.
 */
static int quantize_group_ex2(const float *w, const float *e2, int bits, const float *f, int nf,
                              uint16_t *scale_out, int *c_out, int *chosen_out)
{
    const int qmax = qmax_of(bits);
    int i, j;
    *chosen_out = 0;
    for (i = 0; i < RQO_GROUP; i++)
        if (!isfinite(w[i])) return quantize_group(w, bits, scale_out, c_out);
    float amax = 0.0f;
    for (i = 0; i < RQO_GROUP; i++) {
        float a = fabsf(w[i]);
        if (a > amax) amax = a;
    }
    int best = -1;
    float best_err = 0.0f;
    int cj[RQO_GROUP];
    for (j = 0; j < nf; j++) {
        volatile float a32 = amax * f[j];              /* fp32 multiply */
        volatile float s32 = a32 / (float)qmax;        /* fp32 division */
        uint16_t s16 = rqo_f32_to_f16(s32);
        if (s16 == 0x7C00u) continue;                  /* overflow: never chosen */
        float sf = (float)rqo_f16_to_f64(s16);
        volatile float err = 0.0f;
        for (i = 0; i < RQO_GROUP; i++) {
            int c = 0;
            if (sf != 0.0f) {
                volatile float t0 = w[i] / sf;
                float r = rintf(t0);
                if (r > (float)qmax) r = (float)qmax;
                if (r < (float)-qmax) r = (float)-qmax;
                c = (int)r;
            }
            cj[i] = c;
            volatile float t = (float)c * sf;
            volatile float d = w[i] - t;
            volatile float q = d * d;
            volatile float pr = e2[i] * q;
            err = err + pr;
        }
        if (best < 0 || err < best_err) {
            best = j;
            best_err = err;
            *scale_out = s16;
            for (i = 0; i < RQO_GROUP; i++) c_out[i] = cj[i];
        }
    }
    if (best < 0) return quantize_group(w, bits, scale_out, c_out);   /* every candidate overflows */
    *chosen_out = best;
    return RQO_OK;
}

/* E[x^2]-weighted scale search over W[N, K] (layouts, statuses and packing
 * as rqo_quantize_g64); e2[K], factors f[nf]; chosen (nullable) receives the
 * winning candidate of each group, [N, K/64]. */
int rqo_quantize_g64_ex2(const float *W, int64_t N, int64_t K, int bits, const float *e2,
                         const float *f, int nf, uint8_t *codes, uint16_t *scales, int32_t *chosen)
{
    const int64_t G = K / RQO_GROUP;
    int status = RQO_OK;
    int64_t n;
#pragma omp parallel for schedule(static) reduction(max : status)
    for (n = 0; n < N; n++) {
        int c[RQO_GROUP];
        int64_t g;
        for (g = 0; g < G; g++) {
            int ch = 0;
            int st = quantize_group_ex2(&W[n * K + g * RQO_GROUP], &e2[g * RQO_GROUP], bits, f, nf,
                                        &scales[n * G + g], c, &ch);
            int64_t i;
            for (i = 0; i < RQO_GROUP; i++) put_code(codes, K, bits, n, g * RQO_GROUP + i, c[i]);
            if (chosen) chosen[n * G + g] = ch;
            if (st > status) status = st;
        }
    }
    if (status != RQO_OK) {
        int64_t i, total = N * G;
        for (i = 0; i < total; i++) if (scales[i] == 0x7E00u) return RQO_ERR_NONFINITE;
    }
    return status;
}

/* ------------------------------------------------------------ products --- */

/* Dequantised weight (n, k) = c * s16, exact in fp64. */
double rqo_weight(const uint8_t *codes, const uint16_t *scales, int64_t K, int bits,
                  int64_t n, int64_t k)
{
    return (double)rqo_get_code(codes, K, bits, n, k) *
           rqo_f16_to_f64(scales[n * (K / RQO_GROUP) + k / RQO_GROUP]);
}

/* One output: y[m, n] and its error budget B[m, n] (either pointer may be
 * null).  x is fp16 bit patterns, row-major [M, K]. */
static void one_output(const uint16_t *x, int64_t K, const uint8_t *codes,
                       const uint16_t *scales, int bits, int64_t m, int64_t n,
                       double *y, double *bound)
{
    double acc = 0.0, b = 0.0;
    int64_t k;
    for (k = 0; k < K; k++) {
        double xv = rqo_f16_to_f64(x[m * K + k]);
        double wv = rqo_weight(codes, scales, K, bits, n, k);
        acc += xv * wv;
        b += fabs(xv) * fabs(wv);
    }
    if (y) *y = acc;
    if (bound) *bound = b;
}

/* Full product y[M, N] (row-major, fp64) and budget B[M, N] (nullable). */
void rqo_matmul(const uint16_t *x, int64_t M, int64_t K, const uint8_t *codes,
                const uint16_t *scales, int64_t N, int bits, double *y, double *bound)
{
    int64_t idx;
#pragma omp parallel for schedule(static)
    for (idx = 0; idx < M * N; idx++) {
        int64_t m = idx / N, n = idx % N;
        one_output(x, K, codes, scales, bits, m, n, &y[idx], bound ? &bound[idx] : 0);
    }
}

/* Sampled outputs: for each of the P pairs (ms[p], ns[p]) compute y and B. */
void rqo_matmul_sampled(const uint16_t *x, int64_t M, int64_t K, const uint8_t *codes,
                        const uint16_t *scales, int64_t N, int bits, int64_t P,
                        const int64_t *ms, const int64_t *ns, double *y, double *bound)
{
    int64_t p;
    (void)M; (void)N;
#pragma omp parallel for schedule(static)
    for (p = 0; p < P; p++)
        one_output(x, K, codes, scales, bits, ms[p], ns[p], &y[p], bound ? &bound[p] : 0);
}

/* Quantize one row-block of W (rows [n0, n0 + rows)) -- lets a caller check
 * sampled rows of a matrix too large to quantize whole on the host. */
int rqo_quantize_rows(const float *Wrows, int64_t rows, int64_t K, int bits,
                      uint8_t *codes, uint16_t *scales)
{
    return rqo_quantize_g64(Wrows, rows, K, bits, codes, scales);
}

/* ------------------------------------------------------------------ GPTQ --- */
/*
 * GPTQ on the symmetric group-64 grid.  "Hakureirm/rwkv7-sglang-w4gptq-1.5b"
 * model card, opening summary: the int4 checkpoint is GPTQ-calibrated,
 * symmetric, group 64, in the same .qweight + .scale format as the
 * calibration-free RTN it is compared with; "rwkv-quant: uma matriz em bf16
 * elimina 39% das perdas na quantização do RWKV-7 2.9B", "Vazamento de
 * calibração e medições honestas": GPTQ runs on the preset's grid without
 * changing the format, the kernels or the file size.  The method is the
 * published GPTQ (Frantar et al., arXiv:2210.17323, which the RWKVQuant page
 * lists among the works it builds on): quantize the columns of W in order and
 * spread each column's rounding error over the columns not yet quantized,
 * weighted by the inverse Hessian H^-1 of the layer's input (H = 2 X^T X / T
 * plus damping), through U, the upper Cholesky factor of H^-1 (H^-1 = U^T U).
 *
 * This function is the column loop, given U (fp32, row-major [K, K], upper
 * triangle read) and the dead-input mask (columns whose input never varies:
 * their weights are zeroed first).  Readings where the pages are silent:
 *   - the group's scale is found when the loop reaches the group's first
 *     column, from the CURRENT (already error-compensated) weights of the
 *     group's 64 columns, exactly as RTN finds it (fp32 amax / qmax, fp16
 *     round to nearest even); each column's code is then RTN against that
 *     stored scale: c_j = clamp(rint(w_j / s16), -qmax, qmax);
 *   - every operation is one fp32 rounding, in this order:
 *       d   = w_j - c_j * s16          (the product is exact in fp32)
 *       e_j = d / U[j][j]
 *       w_k = fmaf(-e_j, U[j][k], w_k)  for k = j+1 .. K-1, j ascending;
 *   - a group whose scale is unusable (a non-finite weight: scale 0x7E00,
 *     status NONFINITE; fp16 overflow: scale 0x7C00, status RANGE) gets codes
 *     0 and spreads no error (e_j = 0) from its columns;
 *   - a scale of zero (the group's weights are all zero when it starts) gives
 *     codes 0 with the error spread as usual.
 * W is overwritten with the compensated weights.  Returns the status, as
 * rqo_quantize_g64 does (NONFINITE over RANGE over OK).
 */
static int gptq_row(float *w, int64_t K, int bits, const float *U, const uint8_t *dead,
                    uint8_t *codes_row_base, int64_t n, uint16_t *scales_row)
{
    const int qmax = qmax_of(bits);
    int status = RQO_OK;
    int64_t j, k;
    if (dead)
        for (j = 0; j < K; j++) if (dead[j]) w[j] = 0.0f;
    float sf = 0.0f;
    int usable = 1;
    for (j = 0; j < K; j++) {
        if (j % RQO_GROUP == 0) {
            /* the group's scale, from its current weights */
            int i, finite = 1;
            float amax = 0.0f;
            for (i = 0; i < RQO_GROUP; i++) {
                float v = w[j + i];
                if (!isfinite(v)) finite = 0;
                float a = fabsf(v);
                if (a > amax) amax = a;
            }
            uint16_t s16;
            if (!finite) {
                s16 = 0x7E00u;
                usable = 0;
                status = RQO_ERR_NONFINITE;
            } else {
                volatile float s32 = amax / (float)qmax;
                s16 = rqo_f32_to_f16(s32);
                usable = s16 != 0x7C00u;
                if (!usable && status == RQO_OK) status = RQO_ERR_RANGE;
            }
            scales_row[j / RQO_GROUP] = s16;
            sf = usable ? (float)rqo_f16_to_f64(s16) : 0.0f;
        }
        int c = 0;
        float e = 0.0f;
        if (usable) {
            if (sf != 0.0f) {
                volatile float t = w[j] / sf;
                float r = rintf(t);
                if (r > (float)qmax) r = (float)qmax;
                if (r < (float)-qmax) r = (float)-qmax;
                c = (int)r;
            }
            volatile float dq = (float)c * sf;
            volatile float d = w[j] - dq;
            volatile float ev = d / U[j * K + j];
            e = ev;
        }
        put_code(codes_row_base, K, bits, n, j, c);
        if (e != 0.0f)
            for (k = j + 1; k < K; k++) w[k] = fmaf(-e, U[j * K + k], w[k]);
    }
    return status;
}

/* GPTQ over W[N, K] (fp32, overwritten with the compensated weights); codes,
 * scales and status as rqo_quantize_g64.  U: fp32 [K, K], the upper Cholesky
 * factor of the damped inverse Hessian; dead: nullable uint8 [K]. */
int rqo_gptq_g64(float *W, int64_t N, int64_t K, int bits, const float *U, const uint8_t *dead,
                 uint8_t *codes, uint16_t *scales)
{
    const int64_t G = K / RQO_GROUP;
    int status = RQO_OK;
    int64_t n;
#pragma omp parallel for schedule(dynamic, 1) reduction(max : status)
    for (n = 0; n < N; n++) {
        int st = gptq_row(&W[n * K], K, bits, U, dead, codes, n, &scales[n * G]);
        if (st > status) status = st;
    }
    if (status != RQO_OK) {
        int64_t i, total = N * G;
        for (i = 0; i < total; i++) if (scales[i] == 0x7E00u) return RQO_ERR_NONFINITE;
    }
    return status;
}

/* --------------------------------------------------- preset formats (f3) --- */
/*
 * The two presets of "rwkv-quant: uma matriz em bf16 elimina 39% das perdas na
 * quantização do RWKV-7 2.9B", section "Dois presets e seis tamanhos":
 * REDUCTION stores projections in 8 bits, symmetric, groups of 16 weights;
 * COMPRESSION stores them in 4 bits, asymmetric, in super-blocks, groups of
 * 32; in both, each group's scale (and offset) is chosen by a search weighted
 * by E[x^2] of the input channel.  Readings where the page is silent:
 *
 * int8 g16 symmetric ("p8"): exactly the g64 steps of rqo_quantize_g64 /
 *   rqo_quantize_g64_ex2 with groups of G = 16 (scale fp16_rn(fp32 amax * f /
 *   127), RTN codes, the smallest sum e2 (w - c s)^2 wins, earlier on ties).
 *   Written once for any G here; G = 64 reproduces the g64 functions.
 *
 * int4 g32 asymmetric in super-blocks of 8 groups ("p4a"), per row:
 *   group g (32 weights): lo = min(0, min w), hi = max(0, max w);
 *     candidate j: lo_j = fp32(lo * f_j), hi_j = fp32(hi * f_j),
 *       s_j = fp32(fp32(hi_j - lo_j) / 15), o_j = lo_j,
 *       q = clamp(rint(fp32(w - o_j) / s_j), 0, 15)  (q = 0 when s_j == 0),
 *       err_j = sum_k e2[k] * (w - (q s_j + o_j))^2, one fp32 rounding per
 *       operation in k order; the smallest err_j wins (earlier on ties);
 *     without a search (e2 NULL) the single candidate f = 1;
 *   super-block (8 groups): ds = fp16_rn(fp32(max_g s_g) / 63),
 *     dm = fp16_rn(fp32(max_g -o_g) / 63);
 *     a_g = clamp(rint(s_g / ds), 0, 63), b_g = clamp(rint(-o_g / dm), 0, 63)
 *     (0 when ds / dm is 0);
 *   stored scale and offset: S_g = ds * a_g, O_g = -(dm * b_g) (exact in fp32);
 *   codes q = clamp(rint(fp32(w - O_g) / S_g), 0, 15) (q = 0 when S_g == 0);
 *   w_hat = S_g * q + O_g.
 *   Layout: codes uint8 [N, K/2] (q unsigned, k = 2j in the low nibble);
 *   sub uint8 [N, K/32, 2] = {a_g, b_g}; sup fp16 [N, K/256, 2] = {ds, dm}.
 *   K % 256 == 0.  A super-block holding a non-finite weight gets ds = dm =
 *   0x7E00, sub-codes and codes 0, status NONFINITE; one whose ds or dm
 *   overflows fp16 keeps the inf, sub-codes and codes 0, status RANGE.
 */

/* Symmetric group of G weights, optional E[x^2] search (e2 NULL: RTN). */
static int quantize_sym_group(const float *w, int G, int bits, const float *e2, const float *f,
                              int nf, uint16_t *scale_out, int *c_out, int *chosen_out)
{
    const int qmax = qmax_of(bits);
    int i, j;
    *chosen_out = 0;
    for (i = 0; i < G; i++) {
        if (!isfinite(w[i])) {
            *scale_out = 0x7E00u;
            for (i = 0; i < G; i++) c_out[i] = 0;
            return RQO_ERR_NONFINITE;
        }
    }
    float amax = 0.0f;
    for (i = 0; i < G; i++) {
        float a = fabsf(w[i]);
        if (a > amax) amax = a;
    }
    const int ncand = e2 ? nf : 1;
    int best = -1;
    float best_err = 0.0f;
    int cj[64];
    for (j = 0; j < ncand; j++) {
        volatile float a32 = e2 ? amax * f[j] : amax;
        volatile float s32 = a32 / (float)qmax;
        uint16_t s16 = rqo_f32_to_f16(s32);
        if (s16 == 0x7C00u) continue;
        float sf = (float)rqo_f16_to_f64(s16);
        volatile float err = 0.0f;
        for (i = 0; i < G; i++) {
            int c = 0;
            if (sf != 0.0f) {
                volatile float t0 = w[i] / sf;
                float r = rintf(t0);
                if (r > (float)qmax) r = (float)qmax;
                if (r < (float)-qmax) r = (float)-qmax;
                c = (int)r;
            }
            cj[i] = c;
            if (e2) {
                volatile float t = (float)c * sf;
                volatile float d = w[i] - t;
                volatile float q = d * d;
                volatile float pr = e2[i] * q;
                err = err + pr;
            }
        }
        if (best < 0 || err < best_err) {
            best = j;
            best_err = err;
            *scale_out = s16;
            for (i = 0; i < G; i++) c_out[i] = cj[i];
        }
    }
    if (best < 0) {
        /* every candidate's scale overflows: RTN decides (as the g64 search
         * does); RTN's own overflow gives scale +inf, codes 0, RANGE */
        if (e2) return quantize_sym_group(w, G, bits, 0, f, nf, scale_out, c_out, chosen_out);
        *scale_out = 0x7C00u;
        for (i = 0; i < G; i++) c_out[i] = 0;
        return RQO_ERR_RANGE;
    }
    *chosen_out = best;
    return RQO_OK;
}

/* Symmetric group-G quantization of W[N, K] (K % G == 0, G in {16, 32, 64}):
 * codes as rqo_quantize_g64, scales fp16 [N, K/G], chosen (nullable) [N, K/G].
 * e2 NULL: RTN. */
int rqo_quantize_sym(const float *W, int64_t N, int64_t K, int bits, int G, const float *e2,
                     const float *f, int nf, uint8_t *codes, uint16_t *scales, int32_t *chosen)
{
    const int64_t NG = K / G;
    int status = RQO_OK;
    int64_t n;
#pragma omp parallel for schedule(static) reduction(max : status)
    for (n = 0; n < N; n++) {
        int c[64];
        int64_t g;
        for (g = 0; g < NG; g++) {
            int ch = 0;
            int st = quantize_sym_group(&W[n * K + g * G], G, bits, e2 ? &e2[g * G] : 0, f, nf,
                                        &scales[n * NG + g], c, &ch);
            int64_t i;
            for (i = 0; i < G; i++) put_code(codes, K, bits, n, g * G + i, c[i]);
            if (chosen) chosen[n * NG + g] = ch;
            if (st > status) status = st;
        }
    }
    if (status != RQO_OK) {
        int64_t i, total = N * NG;
        for (i = 0; i < total; i++) if (scales[i] == 0x7E00u) return RQO_ERR_NONFINITE;
    }
    return status;
}

/* Unsigned 4-bit code store / load (asymmetric format). */
static void put_ucode4(uint8_t *codes, int64_t K, int64_t n, int64_t k, int q)
{
    uint8_t *b = &codes[n * (K / 2) + k / 2];
    if (k % 2 == 0) *b = (uint8_t)((*b & 0xF0u) | (q & 0xF));
    else            *b = (uint8_t)((*b & 0x0Fu) | ((q & 0xF) << 4));
}

int rqo_get_ucode4(const uint8_t *codes, int64_t K, int64_t n, int64_t k)
{
    uint8_t b = codes[n * (K / 2) + k / 2];
    return (k % 2 == 0) ? (b & 0xF) : (b >> 4);
}

static int rint_clamp(float t, int lo, int hi)
{
    float r = rintf(t);
    if (r > (float)hi) r = (float)hi;
    if (r < (float)lo) r = (float)lo;
    return (int)r;
}

/* One asymmetric group of 32: the chosen (s, o) in fp32. */
static void p4a_group_choice(const float *w, const float *e2, const float *f, int nf, float *s_out,
                             float *o_out, int *chosen_out)
{
    int i, j;
    float lo = 0.0f, hi = 0.0f;
    for (i = 0; i < 32; i++) {
        if (w[i] < lo) lo = w[i];
        if (w[i] > hi) hi = w[i];
    }
    const int ncand = e2 ? nf : 1;
    int best = -1;
    float best_err = 0.0f, bs = 0.0f, bo = 0.0f;
    for (j = 0; j < ncand; j++) {
        volatile float loj = e2 ? lo * f[j] : lo;
        volatile float hij = e2 ? hi * f[j] : hi;
        volatile float rng = hij - loj;
        volatile float sj = rng / 15.0f;
        volatile float err = 0.0f;
        if (e2) {
            for (i = 0; i < 32; i++) {
                int q = 0;
                if (sj != 0.0f) {
                    volatile float dw = w[i] - loj;
                    volatile float t = dw / sj;
                    q = rint_clamp(t, 0, 15);
                }
                volatile float t1 = (float)q * sj;
                volatile float u = t1 + loj;
                volatile float d = w[i] - u;
                volatile float qq = d * d;
                volatile float pr = e2[i] * qq;
                err = err + pr;
            }
        }
        if (best < 0 || err < best_err) {
            best = j;
            best_err = err;
            bs = sj;
            bo = loj;
        }
    }
    *s_out = bs;
    *o_out = bo;
    *chosen_out = best;
}

/* Asymmetric int4 g32 super-block quantization of W[N, K] (K % 256 == 0).
 * codes uint8 [N, K/2]; sub uint8 [N, K/32, 2]; sup fp16 [N, K/256, 2];
 * chosen (nullable) int32 [N, K/32]; e2 NULL: no search (factor 1). */
int rqo_quantize_p4a(const float *W, int64_t N, int64_t K, const float *e2, const float *f, int nf,
                     uint8_t *codes, uint8_t *sub, uint16_t *sup, int32_t *chosen)
{
    /* statuses as rqo_quantize_g64: NONFINITE over RANGE over OK */
    const int64_t NSB = K / 256, NG = K / 32;
    int status = RQO_OK;
    int64_t n;
#pragma omp parallel for schedule(static) reduction(max : status)
    for (n = 0; n < N; n++) {
        int64_t sb;
        for (sb = 0; sb < NSB; sb++) {
            const float *w = &W[n * K + sb * 256];
            int i, g;
            int finite = 1;
            for (i = 0; i < 256; i++) if (!isfinite(w[i])) finite = 0;
            uint16_t *sp = &sup[(n * NSB + sb) * 2];
            uint8_t *ab = &sub[(n * NG + sb * 8) * 2];
            if (!finite) {
                sp[0] = sp[1] = 0x7E00u;
                for (g = 0; g < 16; g++) ab[g] = 0;
                for (i = 0; i < 256; i++) put_ucode4(codes, K, n, sb * 256 + i, 0);
                if (chosen) for (g = 0; g < 8; g++) chosen[n * NG + sb * 8 + g] = 0;
                if (RQO_ERR_NONFINITE > status) status = RQO_ERR_NONFINITE;
                continue;
            }
            float s[8], o[8];
            float smax = 0.0f, omax = 0.0f;
            for (g = 0; g < 8; g++) {
                int ch = 0;
                p4a_group_choice(&w[g * 32], e2 ? &e2[sb * 256 + g * 32] : 0, f, nf, &s[g], &o[g], &ch);
                if (chosen) chosen[n * NG + sb * 8 + g] = ch;
                if (s[g] > smax) smax = s[g];
                if (-o[g] > omax) omax = -o[g];
            }
            volatile float ds32 = smax / 63.0f;
            volatile float dm32 = omax / 63.0f;
            uint16_t ds = rqo_f32_to_f16(ds32), dm = rqo_f32_to_f16(dm32);
            sp[0] = ds;
            sp[1] = dm;
            if (ds == 0x7C00u || dm == 0x7C00u) {
                for (g = 0; g < 16; g++) ab[g] = 0;
                for (i = 0; i < 256; i++) put_ucode4(codes, K, n, sb * 256 + i, 0);
                if (RQO_ERR_RANGE > status) status = RQO_ERR_RANGE;
                continue;
            }
            const float dsf = (float)rqo_f16_to_f64(ds), dmf = (float)rqo_f16_to_f64(dm);
            for (g = 0; g < 8; g++) {
                int a = 0, b = 0;
                if (dsf != 0.0f) {
                    volatile float t = s[g] / dsf;
                    a = rint_clamp(t, 0, 63);
                }
                if (dmf != 0.0f) {
                    volatile float t = -o[g] / dmf;
                    b = rint_clamp(t, 0, 63);
                }
                ab[2 * g] = (uint8_t)a;
                ab[2 * g + 1] = (uint8_t)b;
                volatile float S = dsf * (float)a;
                volatile float O = -(dmf * (float)b);
                for (i = 0; i < 32; i++) {
                    int q = 0;
                    if (S != 0.0f) {
                        volatile float dw = w[g * 32 + i] - O;
                        volatile float t = dw / S;
                        q = rint_clamp(t, 0, 15);
                    }
                    put_ucode4(codes, K, n, sb * 256 + g * 32 + i, q);
                }
            }
        }
    }
    if (status != RQO_OK) {
        int64_t i, total = N * NSB * 2;
        for (i = 0; i < total; i++) if (sup[i] == 0x7E00u) return RQO_ERR_NONFINITE;
    }
    return status;
}

/* Dequantised weight of the preset formats, exact in fp64.
 * fmt 8: int8 g16 symmetric (meta0 = scales fp16 [N, K/16]);
 * fmt 4: int4 g32 asymmetric super-blocks (meta0 = sub, meta1 = sup). */
static double fmt_weight(int fmt, const uint8_t *codes, const void *meta0, const void *meta1,
                         int64_t K, int64_t n, int64_t k)
{
    if (fmt == 8) {
        const uint16_t *sc = (const uint16_t *)meta0;
        return (double)(int)(int8_t)codes[n * K + k] * rqo_f16_to_f64(sc[n * (K / 16) + k / 16]);
    }
    const uint8_t *sub = (const uint8_t *)meta0;
    const uint16_t *sup = (const uint16_t *)meta1;
    const int64_t g = k / 32, sb = k / 256;
    const double ds = rqo_f16_to_f64(sup[(n * (K / 256) + sb) * 2]);
    const double dm = rqo_f16_to_f64(sup[(n * (K / 256) + sb) * 2 + 1]);
    const double S = ds * (double)sub[(n * (K / 32) + g) * 2];
    const double O = -(dm * (double)sub[(n * (K / 32) + g) * 2 + 1]);
    return S * (double)rqo_get_ucode4(codes, K, n, k) + O;
}

/* y[m, n] = sum_k x[m, k] w_hat[n, k] (fp64) and the budget sum |x||w_hat|,
 * for the P pairs (ms[p], ns[p]) (ms NULL: every output, row-major). */
void rqo_matmul_fmt(int fmt, const uint16_t *x, int64_t M, int64_t K, const uint8_t *codes,
                    const void *meta0, const void *meta1, int64_t N, int64_t P, const int64_t *ms,
                    const int64_t *ns, double *y, double *bound)
{
    const int64_t total = ms ? P : M * N;
    int64_t p;
#pragma omp parallel for schedule(static)
    for (p = 0; p < total; p++) {
        const int64_t m = ms ? ms[p] : p / N, n = ms ? ns[p] : p % N;
        double acc = 0.0, b = 0.0;
        int64_t k;
        for (k = 0; k < K; k++) {
            double xv = rqo_f16_to_f64(x[m * K + k]);
            double wv = fmt_weight(fmt, codes, meta0, meta1, K, n, k);
            acc += xv * wv;
            b += fabs(xv) * fabs(wv);
        }
        y[p] = acc;
        if (bound) bound[p] = b;
    }
}
