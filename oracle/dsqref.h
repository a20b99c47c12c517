/*
 * dsqref.h -- plain CPU oracle for the block-quantized projection path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or
 * calls this code; only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg do.  It is deliberately slow: single-threaded loops, no
 * SIMD intrinsics, no blocking, built with -O2 -ffp-contract=off so every
 * float operation is one IEEE-rounded step in the order written.
 *
 * Sources (page titles; the pages print no code for any of this):
 *  - "ROCm: restore DeepSeek V4 Flash decode performance and Q4 SSD
 *    streaming" (antirez/ds4 PR #623), Summary and the per-stage timing
 *    comment: decode activations are prequantized to Q8 once and consumed by
 *    Q8_0 weight GEMVs (regular, paired, HC-expand, low-rank
 *    attention-output); the restored kernels run one warp per output row.
 *  - "Support AProjQ4 GGUFs: Q4_K dense attention projections" (antirez/ds4
 *    PR #621), GB10 test report and consolidated results: Q4_K attention
 *    projections; prefill dequantizes the weights into a dense GEMM.
 *  - "DeepSeek V4 Flash on Strix Halo: tuning ROCm, matching Vulkan",
 *    section "Why I did not keep a ROCm kernel patch": the quantized GEMV is
 *    preceded by a per-32 activation quantization (quantize_q8_1).
 *  - "DeepSeek V4" (ggml-org/llama.cpp PR #24162), comment on tensor shapes:
 *    the attention-output tensor is stored as [4096, 1024, 8] (K inner,
 *    1024 rows, 8 groups).
 *  The block formats themselves (Q8_0: fp16 d + 32 int8, x = d*q; Q4_K:
 *  256-element super-block, fp16 d/dmin, eight 6-bit scale/min pairs, 4-bit
 *  quants, x = d*sc*q - dmin*m) and the activation rule (scale = amax/127,
 *  round half away from zero) are named by the pages only by name; the
 *  byte-level readings taken here are listed with each function.
 *
 * Parity pins: every function below is checked in tests/test_oracle_*.py
 * against hand-worked blocks (tests/golden/), closed forms, invariants,
 * brute force on tiny inputs, and independent library routines (numpy
 * float16, torch bfloat16, numpy float64 matmul).
 */
#ifndef DSQREF_H
#define DSQREF_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { DSQREF_Q8_0 = 8, DSQREF_Q4_K = 12 };

#define DSQREF_QK8_0 32           /* elements per Q8_0 block            */
#define DSQREF_Q8_0_BYTES 34      /* fp16 d + 32 x int8                 */
#define DSQREF_QK_K 256           /* elements per Q4_K super-block      */
#define DSQREF_Q4_K_BYTES 144     /* fp16 d, fp16 dmin, 12 B scales, 128 B nibbles */

/* ---- IEEE conversions (bit-level, round to nearest even) ---- */
uint16_t dsqref_f32_to_f16(float x);
float dsqref_f16_to_f32(uint16_t h);
uint16_t dsqref_f32_to_bf16(float x);
float dsqref_bf16_to_f32(uint16_t h);

/* Bytes of one weight row of K elements (0 when K does not fit the type). */
int64_t dsqref_row_bytes(int type, int64_t K);

/* ---- Q8_0 weights ---- */
void dsqref_quantize_q8_0(const float *x, int64_t rows, int64_t K, uint8_t *out);
void dsqref_dequantize_q8_0(const uint8_t *w, int64_t rows, int64_t K, float *out);

/* ---- Q4_K weights ---- */
void dsqref_q4k_get_scale_min(const uint8_t *scales12, int j, int *sc, int *m);
void dsqref_q4k_set_scale_min(uint8_t *scales12, int j, int sc, int m);
void dsqref_quantize_q4_k(const float *x, int64_t rows, int64_t K, uint8_t *out);
void dsqref_dequantize_q4_k(const uint8_t *w, int64_t rows, int64_t K, float *out);
void dsqref_dequantize(int type, const uint8_t *w, int64_t rows, int64_t K, float *out);

/* ---- activation prequantization to Q8 per 32-block ---- */
void dsqref_quantize_act_q8(const float *x, int64_t M, int64_t K,
                            int8_t *xq, float *xd, int32_t *xs);

/* ---- per-block integer dot products (the exact part of the method) ---- */
void dsqref_block_sums(int type, const uint8_t *w, int64_t N, int64_t K,
                       const int8_t *xq, int32_t *isum /* N x K/32 */);

/* ---- decode GEMV, integer form, fp64 result ----
 * y[n]     = sum over blocks of the method's scaled block terms, each term
 *            formed exactly in double;
 * absum[n] = sum of the magnitudes of every product the method forms
 *            (the condition scale the GEMV tolerance is measured against);
 *            may be NULL. */
void dsqref_gemv(int type, const uint8_t *w, int64_t N, int64_t K,
                 const int8_t *xq, const float *xd, const int32_t *xs,
                 double *y, double *absum);

/* Plain definition of the same product: fp64 dot of the dequantized weight
 * row with the dequantized activation.  Shares no arithmetic with
 * dsqref_gemv beyond the format decoders. */
void dsqref_gemv_dequant_f64(int type, const uint8_t *w, int64_t N, int64_t K,
                             const int8_t *xq, const float *xd, double *y);

/* ---- prefill references ----
 * Y[m][n] = sum_k x[m][k] * deq(W)[n][k], all in fp64 (exact products). */
void dsqref_prefill_f64(int type, const uint8_t *w, int64_t N, int64_t K,
                        const float *x, int64_t M, double *y);

/* Per-row power-of-two shift used before rounding activations to a 16-bit
 * float: the smallest-magnitude choice that puts the row's largest |x| in
 * [2^14, 2^15); 0 for an all-zero row; clamped to [-113, 126], so every
 * finite row whose largest magnitude is at least 2^-112 lands in that
 * binade and smaller rows are scaled by 2^126. */
int dsqref_row_shift(const float *row, int64_t K);

/* Operand-rounded reference: the same sum with x -> r(x * 2^s_m) and
 * w -> r(fp32 dequant), r = fp16 RNE (op16 = 0) or bf16 RNE (op16 = 1),
 * the sum in fp64, then scaled back by 2^-s_m.  This is what a 16-bit
 * tensor-core contraction with exact products computes; it isolates
 * accumulation error from operand rounding. */
void dsqref_prefill_rounded(int type, int op16, const uint8_t *w, int64_t N,
                            int64_t K, const float *x, int64_t M, double *y);

/* The rounded operands of dsqref_prefill_rounded as bit patterns:
 * x16[m][k] = r(x[m][k] * 2^shift[m]), w16[n][k] = r(fp32 dequant). */
void dsqref_prefill_operands(int type, int op16, const uint8_t *w, int64_t N,
                             int64_t K, const float *x, int64_t M,
                             uint16_t *x16, int32_t *shift, uint16_t *w16);

#ifdef __cplusplus
}
#endif
#endif
