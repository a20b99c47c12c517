/*
 * dsqref.c -- plain CPU oracle for the block-quantized projection path.
 *
 * TEST INFRASTRUCTURE ONLY (see dsqref.h).  Single-threaded loops in the
 * order the definitions are stated; compile with -O2 -ffp-contract=off and
 * without -ffast-math so each float expression is evaluated as written.
 */
#include "dsqref.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* IEEE binary16 / bfloat16 conversions, written from the IEEE 754 encoding */
/* ------------------------------------------------------------------------ */

static uint32_t f32_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }
static float bits_f32(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }

/* binary32 -> binary16, round to nearest, ties to even. */
uint16_t dsqref_f32_to_f16(float f)
{
    uint32_t x = f32_bits(f);
    uint16_t sign = (uint16_t)((x >> 16) & 0x8000u);
    uint32_t ax = x & 0x7fffffffu;
    if (ax > 0x7f800000u)                       /* NaN: keep it quiet */
        return (uint16_t)(sign | 0x7e00u | ((ax >> 13) & 0x3ffu));
    if (ax >= 0x477ff000u)                      /* >= 65520 rounds to inf */
        return (uint16_t)(sign | 0x7c00u);
    if (ax >= 0x38800000u) {                    /* normal binary16 range */
        uint32_t e = (ax >> 23) - 127u + 15u;
        uint32_t mant = ax & 0x7fffffu;
        uint32_t h = (e << 10) | (mant >> 13);
        uint32_t rem = mant & 0x1fffu;
        if (rem > 0x1000u || (rem == 0x1000u && (h & 1u)))
            h += 1u;                            /* may carry into exponent */
        return (uint16_t)(sign | h);
    }
    /* subnormal binary16 (or zero): value / 2^-24 rounded to an integer */
    uint32_t e = ax >> 23;
    if (e == 0) return sign;                    /* fp32 zero/subnormal -> 0 */
    uint32_t mant = (ax & 0x7fffffu) | 0x800000u;   /* value = mant*2^(e-150) */
    uint32_t shift = 126u - e;                  /* value*2^24 = mant>>shift */
    if (shift > 24u) return sign;
    uint32_t h = mant >> shift;
    uint32_t rem = mant & ((1u << shift) - 1u);
    uint32_t half = 1u << (shift - 1u);
    if (rem > half || (rem == half && (h & 1u)))
        h += 1u;
    return (uint16_t)(sign | h);
}

float dsqref_f16_to_f32(uint16_t h)
{
    uint32_t sign = ((uint32_t)h & 0x8000u) << 16;
    uint32_t e = ((uint32_t)h >> 10) & 0x1fu;
    uint32_t mant = (uint32_t)h & 0x3ffu;
    if (e == 0x1fu)
        return bits_f32(sign | 0x7f800000u | (mant << 13));
    if (e == 0) {
        /* subnormal: mant * 2^-24, exact in binary32 */
        float v = (float)mant * 0x1p-24f;
        return sign ? -v : v;
    }
    return bits_f32(sign | ((e - 15u + 127u) << 23) | (mant << 13));
}

uint16_t dsqref_f32_to_bf16(float f)
{
    uint32_t x = f32_bits(f);
    if ((x & 0x7fffffffu) > 0x7f800000u)
        return (uint16_t)((x >> 16) | 0x40u);   /* quiet NaN */
    uint32_t lsb = (x >> 16) & 1u;
    x += 0x7fffu + lsb;                          /* ties to even */
    return (uint16_t)(x >> 16);
}

float dsqref_bf16_to_f32(uint16_t h) { return bits_f32((uint32_t)h << 16); }

/* ------------------------------------------------------------------------ */
/* formats                                                                  */
/* ------------------------------------------------------------------------ */

int64_t dsqref_row_bytes(int type, int64_t K)
{
    if (type == DSQREF_Q8_0 && K > 0 && K % DSQREF_QK8_0 == 0)
        return K / DSQREF_QK8_0 * DSQREF_Q8_0_BYTES;
    if (type == DSQREF_Q4_K && K > 0 && K % DSQREF_QK_K == 0)
        return K / DSQREF_QK_K * DSQREF_Q4_K_BYTES;
    return 0;
}

static uint16_t rd16(const uint8_t *p) { return (uint16_t)(p[0] | (p[1] << 8)); }
static void wr16(uint8_t *p, uint16_t v) { p[0] = (uint8_t)(v & 0xff); p[1] = (uint8_t)(v >> 8); }

/* Shared 32-element rule of the Q8 formats: amax -> d32 = amax/127 (one IEEE
 * division), q = clamp(roundf(x/d32), -127, 127) (roundf: half away from
 * zero); an all-zero block gives d32 = 0 and q = 0. */
static float q8_block(const float *x, int8_t *q)
{
    float amax = 0.0f;
    for (int i = 0; i < DSQREF_QK8_0; ++i) {
        float a = fabsf(x[i]);
        if (a > amax) amax = a;
    }
    float d32 = amax / 127.0f;
    for (int i = 0; i < DSQREF_QK8_0; ++i) {
        if (d32 == 0.0f) { q[i] = 0; continue; }
        float v = roundf(x[i] / d32);
        if (v > 127.0f) v = 127.0f;
        if (v < -127.0f) v = -127.0f;
        q[i] = (int8_t)v;
    }
    return d32;
}

/* Q8_0 weight block: {fp16 d (little-endian), int8 q[32]}; d = fp16(d32),
 * q computed from the unrounded d32. */
void dsqref_quantize_q8_0(const float *x, int64_t rows, int64_t K, uint8_t *out)
{
    int64_t nb = K / DSQREF_QK8_0;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < nb; ++b) {
            const float *xb = x + r * K + b * DSQREF_QK8_0;
            uint8_t *ob = out + (r * nb + b) * DSQREF_Q8_0_BYTES;
            int8_t q[DSQREF_QK8_0];
            float d32 = q8_block(xb, q);
            wr16(ob, dsqref_f32_to_f16(d32));
            memcpy(ob + 2, q, DSQREF_QK8_0);
        }
    }
}

/* x^ = float(d) * q, one fp32 product (exact: 11 x 7 significant bits). */
void dsqref_dequantize_q8_0(const uint8_t *w, int64_t rows, int64_t K, float *out)
{
    int64_t nb = K / DSQREF_QK8_0;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t b = 0; b < nb; ++b) {
            const uint8_t *blk = w + (r * nb + b) * DSQREF_Q8_0_BYTES;
            float d = dsqref_f16_to_f32(rd16(blk));
            for (int i = 0; i < DSQREF_QK8_0; ++i)
                out[r * K + b * DSQREF_QK8_0 + i] = d * (float)(int8_t)blk[2 + i];
        }
}

/* Q4_K 12-byte scale field (GGUF packing, the reading taken for the
 * "8 x 6-bit scale/min" field):
 *   j < 4 : sc = s[j] & 63,                      m = s[j+4] & 63
 *   j >= 4: sc = (s[j+4] & 15) | (s[j-4] >> 6) << 4,
 *           m  = (s[j+4] >> 4) | (s[j]   >> 6) << 4 */
void dsqref_q4k_get_scale_min(const uint8_t *s, int j, int *sc, int *m)
{
    if (j < 4) {
        *sc = s[j] & 63;
        *m = s[j + 4] & 63;
    } else {
        *sc = (s[j + 4] & 15) | ((s[j - 4] >> 6) << 4);
        *m = (s[j + 4] >> 4) | ((s[j] >> 6) << 4);
    }
}

void dsqref_q4k_set_scale_min(uint8_t *s, int j, int sc, int m)
{
    if (j < 4) {
        s[j] = (uint8_t)((s[j] & 0xc0) | (sc & 63));
        s[j + 4] = (uint8_t)((s[j + 4] & 0xc0) | (m & 63));
    } else {
        s[j + 4] = (uint8_t)((sc & 15) | ((m & 15) << 4));
        s[j - 4] = (uint8_t)((s[j - 4] & 0x3f) | (((sc >> 4) & 3) << 6));
        s[j] = (uint8_t)((s[j] & 0x3f) | (((m >> 4) & 3) << 6));
    }
}

/* Nibble of element l of sub-block j: the 32 bytes qs[32c..32c+31] hold
 * sub-block 2c in their low nibbles and sub-block 2c+1 in their high ones. */
static int q4k_nibble(const uint8_t *qs, int j, int l)
{
    uint8_t byte = qs[32 * (j / 2) + l];
    return (j & 1) ? (byte >> 4) : (byte & 15);
}

static float clampf(float v, float lo, float hi) { return v < lo ? lo : (v > hi ? hi : v); }

/* Q4_K quantizer (the pages give none; plain min/max reading):
 *   per sub-block j: lo = min(0, min x), hi = max x, s_j = (hi-lo)/15,
 *                    mm_j = -lo
 *   d = fp16(max s_j / 63), dmin = fp16(max mm_j / 63)
 *   sc_j = clamp(roundf(s_j / d), 0, 63)   (0 when d == 0)
 *   m_j  = clamp(roundf(mm_j / dmin), 0, 63) (0 when dmin == 0)
 *   q    = clamp(roundf((x + dmin*m_j) / (d*sc_j)), 0, 15) (0 when d*sc_j == 0) */
void dsqref_quantize_q4_k(const float *x, int64_t rows, int64_t K, uint8_t *out)
{
    int64_t nsb = K / DSQREF_QK_K;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t sb = 0; sb < nsb; ++sb) {
            const float *xs = x + r * K + sb * DSQREF_QK_K;
            uint8_t *blk = out + (r * nsb + sb) * DSQREF_Q4_K_BYTES;
            float s[8], mm[8];
            float smax = 0.0f, mmax = 0.0f;
            for (int j = 0; j < 8; ++j) {
                float lo = 0.0f, hi = xs[32 * j];
                for (int l = 0; l < 32; ++l) {
                    float v = xs[32 * j + l];
                    if (v < lo) lo = v;
                    if (v > hi) hi = v;
                }
                s[j] = (hi - lo) / 15.0f;
                mm[j] = -lo;
                if (s[j] > smax) smax = s[j];
                if (mm[j] > mmax) mmax = mm[j];
            }
            uint16_t dh = dsqref_f32_to_f16(smax / 63.0f);
            uint16_t mh = dsqref_f32_to_f16(mmax / 63.0f);
            float d = dsqref_f16_to_f32(dh);
            float dmin = dsqref_f16_to_f32(mh);
            wr16(blk, dh);
            wr16(blk + 2, mh);
            uint8_t *scales = blk + 4;
            uint8_t *qs = blk + 16;
            memset(scales, 0, 12);
            memset(qs, 0, 128);
            for (int j = 0; j < 8; ++j) {
                int sc = d > 0.0f ? (int)clampf(roundf(s[j] / d), 0.0f, 63.0f) : 0;
                int m = dmin > 0.0f ? (int)clampf(roundf(mm[j] / dmin), 0.0f, 63.0f) : 0;
                dsqref_q4k_set_scale_min(scales, j, sc, m);
                float den = d * (float)sc;
                float off = dmin * (float)m;
                for (int l = 0; l < 32; ++l) {
                    int q = 0;
                    if (den != 0.0f) {
                        float t = xs[32 * j + l] + off;
                        q = (int)clampf(roundf(t / den), 0.0f, 15.0f);
                    }
                    uint8_t *byte = &qs[32 * (j / 2) + l];
                    if (j & 1) *byte = (uint8_t)((*byte & 0x0f) | (q << 4));
                    else       *byte = (uint8_t)((*byte & 0xf0) | q);
                }
            }
        }
}

/* x^ = a*q - b with a = float(d)*sc, b = float(dmin)*m, each an fp32 step in
 * that order (a*q and b are exact; the subtraction rounds once). */
void dsqref_dequantize_q4_k(const uint8_t *w, int64_t rows, int64_t K, float *out)
{
    int64_t nsb = K / DSQREF_QK_K;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t sb = 0; sb < nsb; ++sb) {
            const uint8_t *blk = w + (r * nsb + sb) * DSQREF_Q4_K_BYTES;
            float d = dsqref_f16_to_f32(rd16(blk));
            float dmin = dsqref_f16_to_f32(rd16(blk + 2));
            for (int j = 0; j < 8; ++j) {
                int sc, m;
                dsqref_q4k_get_scale_min(blk + 4, j, &sc, &m);
                float a = d * (float)sc;
                float b = dmin * (float)m;
                for (int l = 0; l < 32; ++l) {
                    float aq = a * (float)q4k_nibble(blk + 16, j, l);
                    out[r * K + sb * DSQREF_QK_K + 32 * j + l] = aq - b;
                }
            }
        }
}

void dsqref_dequantize(int type, const uint8_t *w, int64_t rows, int64_t K, float *out)
{
    if (type == DSQREF_Q8_0) dsqref_dequantize_q8_0(w, rows, K, out);
    else if (type == DSQREF_Q4_K) dsqref_dequantize_q4_k(w, rows, K, out);
}

/* Exact real value of one weight element, in double (plain definition). */
static double weight_value_f64(int type, const uint8_t *w, int64_t K, int64_t n, int64_t k)
{
    if (type == DSQREF_Q8_0) {
        int64_t nb = K / DSQREF_QK8_0;
        const uint8_t *blk = w + (n * nb + k / DSQREF_QK8_0) * DSQREF_Q8_0_BYTES;
        return (double)dsqref_f16_to_f32(rd16(blk)) * (double)(int8_t)blk[2 + k % DSQREF_QK8_0];
    } else {
        int64_t nsb = K / DSQREF_QK_K;
        const uint8_t *blk = w + (n * nsb + k / DSQREF_QK_K) * DSQREF_Q4_K_BYTES;
        int j = (int)((k % DSQREF_QK_K) / 32), l = (int)(k % 32), sc, m;
        dsqref_q4k_get_scale_min(blk + 4, j, &sc, &m);
        double d = dsqref_f16_to_f32(rd16(blk));
        double dmin = dsqref_f16_to_f32(rd16(blk + 2));
        return d * sc * q4k_nibble(blk + 16, j, l) - dmin * m;
    }
}

/* ------------------------------------------------------------------------ */
/* activation prequantization                                               */
/* ------------------------------------------------------------------------ */

/* Per 32-block of each row: the Q8 rule above with the scale kept in fp32
 * (xd) and the block sum of the codes (xs, used by the Q4_K min term). */
void dsqref_quantize_act_q8(const float *x, int64_t M, int64_t K,
                            int8_t *xq, float *xd, int32_t *xs)
{
    int64_t nb = K / DSQREF_QK8_0;
    for (int64_t m = 0; m < M; ++m)
        for (int64_t b = 0; b < nb; ++b) {
            int8_t *q = xq + m * K + b * DSQREF_QK8_0;
            xd[m * nb + b] = q8_block(x + m * K + b * DSQREF_QK8_0, q);
            int32_t s = 0;
            for (int i = 0; i < DSQREF_QK8_0; ++i) s += q[i];
            xs[m * nb + b] = s;
        }
}

/* ------------------------------------------------------------------------ */
/* block integer dot products                                               */
/* ------------------------------------------------------------------------ */

/* isum[n][b] = sum_i qw[n][32b+i] * qx[32b+i], exactly in int32.  For Q4_K,
 * b = 8*superblock + j and qw is the 4-bit code of sub-block j. */
void dsqref_block_sums(int type, const uint8_t *w, int64_t N, int64_t K,
                       const int8_t *xq, int32_t *isum)
{
    int64_t nb = K / 32;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t b = 0; b < nb; ++b) {
            int32_t s = 0;
            for (int i = 0; i < 32; ++i) {
                int qw;
                if (type == DSQREF_Q8_0) {
                    const uint8_t *blk = w + (n * nb + b) * DSQREF_Q8_0_BYTES;
                    qw = (int8_t)blk[2 + i];
                } else {
                    const uint8_t *blk = w + (n * (K / DSQREF_QK_K) + b / 8) * DSQREF_Q4_K_BYTES;
                    qw = q4k_nibble(blk + 16, (int)(b % 8), i);
                }
                s += qw * (int32_t)xq[b * 32 + i];
            }
            isum[n * nb + b] = s;
        }
}

/* ------------------------------------------------------------------------ */
/* decode GEMV                                                              */
/* ------------------------------------------------------------------------ */

/* Integer form of y = W x with both operands block-quantized:
 *   Q8_0: y_n = sum_b (d_w * d_x,b) * isum_nb
 *   Q4_K: y_n = sum_sb sum_j [(d*sc_j) * d_x * isum_j - (dmin*m_j) * d_x * xs_j]
 * Each term is formed in double (at most one rounding) and summed in
 * double in block order. */
void dsqref_gemv(int type, const uint8_t *w, int64_t N, int64_t K,
                 const int8_t *xq, const float *xd, const int32_t *xs,
                 double *y, double *absum)
{
    int64_t nb = K / 32;
    int32_t *isum = (int32_t *)malloc((size_t)nb * sizeof(int32_t));
    for (int64_t n = 0; n < N; ++n) {
        dsqref_block_sums(type, w + n * dsqref_row_bytes(type, K), 1, K, xq, isum);
        double acc = 0.0, mag = 0.0;
        if (type == DSQREF_Q8_0) {
            for (int64_t b = 0; b < nb; ++b) {
                const uint8_t *blk = w + (n * nb + b) * DSQREF_Q8_0_BYTES;
                double t = ((double)dsqref_f16_to_f32(rd16(blk)) * (double)xd[b]) * (double)isum[b];
                acc += t;
                mag += fabs(t);
            }
        } else {
            for (int64_t sb = 0; sb < K / DSQREF_QK_K; ++sb) {
                const uint8_t *blk = w + (n * (K / DSQREF_QK_K) + sb) * DSQREF_Q4_K_BYTES;
                double d = dsqref_f16_to_f32(rd16(blk));
                double dmin = dsqref_f16_to_f32(rd16(blk + 2));
                for (int j = 0; j < 8; ++j) {
                    int sc, m;
                    dsqref_q4k_get_scale_min(blk + 4, j, &sc, &m);
                    int64_t b = sb * 8 + j;
                    double t1 = ((d * sc) * (double)xd[b]) * (double)isum[b];
                    double t2 = ((dmin * m) * (double)xd[b]) * (double)xs[b];
                    acc += t1 - t2;
                    mag += fabs(t1) + fabs(t2);
                }
            }
        }
        y[n] = acc;
        if (absum) absum[n] = mag;
    }
    free(isum);
}

/* Plain definition: sum_k w^[n][k] * x^[k] with x^[k] = xd[k/32]*xq[k] and
 * w^ the exact element value, all in double. */
void dsqref_gemv_dequant_f64(int type, const uint8_t *w, int64_t N, int64_t K,
                             const int8_t *xq, const float *xd, double *y)
{
    for (int64_t n = 0; n < N; ++n) {
        double acc = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            double xv = (double)xd[k / 32] * (double)xq[k];
            acc += weight_value_f64(type, w, K, n, k) * xv;
        }
        y[n] = acc;
    }
}

/* ------------------------------------------------------------------------ */
/* prefill                                                                  */
/* ------------------------------------------------------------------------ */

void dsqref_prefill_f64(int type, const uint8_t *w, int64_t N, int64_t K,
                        const float *x, int64_t M, double *y)
{
    double *wrow = (double *)malloc((size_t)K * sizeof(double));
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) wrow[k] = weight_value_f64(type, w, K, n, k);
        for (int64_t m = 0; m < M; ++m) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) acc += (double)x[m * K + k] * wrow[k];
            y[m * N + n] = acc;
        }
    }
    free(wrow);
}

int dsqref_row_shift(const float *row, int64_t K)
{
    float amax = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
        float a = fabsf(row[k]);
        if (a > amax) amax = a;
    }
    if (!(amax > 0.0f) || isinf(amax)) return 0;
    int e;
    frexpf(amax, &e);            /* amax in [2^(e-1), 2^e) */
    int s = 15 - e;              /* amax * 2^s in [2^14, 2^15) */
    /* 2^s and 2^-s must both be normal fp32 numbers with an exponent field
     * in [1, 254]: s in [-113, 126].  -113 is reached by rows near FLT_MAX
     * (e = 128), so every row with amax >= 2^-112 lands in the binade. */
    if (s > 126) s = 126;
    if (s < -113) s = -113;
    return s;
}

static uint16_t round16_bits(int op16, float v)
{
    return op16 ? dsqref_f32_to_bf16(v) : dsqref_f32_to_f16(v);
}

static double bits16_value(int op16, uint16_t h)
{
    return op16 ? (double)dsqref_bf16_to_f32(h) : (double)dsqref_f16_to_f32(h);
}

void dsqref_prefill_operands(int type, int op16, const uint8_t *w, int64_t N,
                             int64_t K, const float *x, int64_t M,
                             uint16_t *x16, int32_t *shift, uint16_t *w16)
{
    float *wf = (float *)malloc((size_t)K * sizeof(float));
    for (int64_t n = 0; n < N; ++n) {
        dsqref_dequantize(type, w + n * dsqref_row_bytes(type, K), 1, K, wf);
        for (int64_t k = 0; k < K; ++k) w16[n * K + k] = round16_bits(op16, wf[k]);
    }
    for (int64_t m = 0; m < M; ++m) {
        shift[m] = dsqref_row_shift(x + m * K, K);
        for (int64_t k = 0; k < K; ++k)
            x16[m * K + k] = round16_bits(op16, ldexpf(x[m * K + k], shift[m]));
    }
    free(wf);
}

void dsqref_prefill_rounded(int type, int op16, const uint8_t *w, int64_t N,
                            int64_t K, const float *x, int64_t M, double *y)
{
    uint16_t *w16 = (uint16_t *)malloc((size_t)N * (size_t)K * sizeof(uint16_t));
    uint16_t *x16 = (uint16_t *)malloc((size_t)(M > 0 ? M : 1) * (size_t)K * sizeof(uint16_t));
    int32_t *shift = (int32_t *)malloc((size_t)(M > 0 ? M : 1) * sizeof(int32_t));
    dsqref_prefill_operands(type, op16, w, N, K, x, M, x16, shift, w16);
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k)
                acc += bits16_value(op16, x16[m * K + k]) * bits16_value(op16, w16[n * K + k]);
            y[m * N + n] = ldexp(acc, -shift[m]);
        }
    free(w16); free(x16); free(shift);
}
