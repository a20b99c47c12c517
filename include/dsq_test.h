/*
 * dsq_test.h -- test-only entry points of libdsq (not part of the
 * projection API in dsq.h).  Same conventions as dsq.h.
 */
#ifndef DSQ_TEST_H
#define DSQ_TEST_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Per-block int32 dot products of N weight rows with one prequantized
 * activation, written by the SAME device code as the GEMV kernels (a
 * template flag adds the stores): isum[n][b] = sum_{i<32} qw[n][32b+i] *
 * xq[32b+i] for Q8_0, and the 4-bit code dot of sub-block b%8 of super-block
 * b/8 for Q4_K ("Support AProjQ4 GGUFs" / "ROCm: restore DeepSeek V4 Flash
 * decode performance": the integer part of the method is exact).  Also
 * writes y exactly as the regular GEMV would.  isum: N * K/32 int32.
 */
int dsq_test_block_sums(int type, const void *w, int64_t N, int64_t K,
                        const int8_t *xq, const float *xd, const int32_t *xs,
                        float *y, int32_t *isum, void *stream);

/*
 * The multi-token GEMV (dsq_gemv_tokens, one weight) with its per-block int32
 * dot products written out by the same device code: isum [M][N][K/32].
 */
int dsq_test_block_sums_tokens(int type, const void *w, int64_t N, int64_t K, int64_t M,
                               const int8_t *xq, const float *xd, const int32_t *xs,
                               float *y, int32_t *isum, void *stream);

/*
 * Limit, in nanoseconds, of every bounded device wait launched from now on
 * (default 1e9).  0 makes each pipeline wait expire at once without
 * waiting, which exercises the timeout path: the kernel records
 * DSQ_ERR_TIMEOUT, drains its own copies in flight (with a fixed bound),
 * releases what it holds and returns; outputs are then unspecified.
 * UINT64_MAX restores the default.
 */
int dsq_test_set_wait_limit_ns(uint64_t ns);

/*
 * The prefill operands as the kernels round them: x16 [M][K] binary16 bits
 * of x * 2^s_m, shift[M] (s_m), and w16 [N][K] binary16 bits of the fp32
 * dequantized weights.  Lets tests compare operand rounding bit-exactly.
 */
int dsq_test_prefill_operands(int type, const void *w, int64_t N, int64_t K,
                              const float *x, int64_t M, uint16_t *x16,
                              int32_t *shift, uint16_t *w16, void *stream);

#ifdef __cplusplus
}
#endif
#endif /* DSQ_TEST_H */
