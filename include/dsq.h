/*
 * dsq.h -- libdsq: block-quantized weight x activation projections on B200
 * (sm_100a), the decode GEMV with the activation prequantized to Q8 and the
 * prefill dequantize-into-dense-GEMM path of DeepSeek-V4-Flash inference.
 *
 * Sources (page titles):
 *  [ds4-623] "ROCm: restore DeepSeek V4 Flash decode performance and Q4 SSD
 *            streaming" (antirez/ds4 PR #623): Summary (prequantized Q8
 *            decode for regular, paired, HC-expand and low-rank
 *            attention-output projections) and the per-stage timing comment
 *            (matmul_q8_0_tensor, matmul_q8_0_pair_tensor,
 *            attention_output_low_q8_tensor; one warp per output row).
 *  [ds4-621] "Support AProjQ4 GGUFs: Q4_K dense attention projections"
 *            (antirez/ds4 PR #621): GB10 test report (the dequant + GEMM
 *            prefill path) and consolidated results (Q4_K attention
 *            projections, grouped attention-A prefill).
 *  [strix]   "DeepSeek V4 Flash on Strix Halo: tuning ROCm, matching
 *            Vulkan", section "Why I did not keep a ROCm kernel patch"
 *            (activation quantize step + quantized GEMV).
 *  [llama]   "DeepSeek V4" (ggml-org/llama.cpp PR #24162): attention-output
 *            tensor shape [4096, 1024, 8].
 *
 * Conventions for every call:
 *  - All tensor arguments are DEVICE pointers owned by the caller; the
 *    library never allocates, frees or retains them.  Calls are
 *    asynchronous on `stream` (a cudaStream_t passed as void*, NULL = legacy
 *    default stream) and never synchronize.
 *  - A call validates every argument first.  On any error it returns a
 *    non-zero dsq_status, launches nothing, and dsq_last_error() (per host
 *    thread) describes the failure.  There is no fallback path.
 *  - Weights are row-major by output: row n holds K/32 Q8_0 blocks or K/256
 *    Q4_K super-blocks contiguously (ggml ne0 = K inner); row stride is
 *    dsq_row_bytes(type, K).  Q8_0 block = {fp16 d, int8 q[32]} (34 B),
 *    x = d*q.  Q4_K super-block = {fp16 d, fp16 dmin, uint8 scales[12],
 *    uint8 qs[128]} (144 B), x = d*sc_j*q - dmin*m_j with the GGUF packing
 *    of the 6-bit (sc_j, m_j) pairs and sub-block 2c / 2c+1 in the low /
 *    high nibbles of qs[32c .. 32c+31].
 *  - Prequantized activations (from dsq_quantize_act_q8): xq int8 [M][K],
 *    xd fp32 [M][K/32] (block scales), xs int32 [M][K/32] (block code sums,
 *    needed by Q4_K only; may be NULL for Q8_0).
 *  - Alignment: weight, xq, xd, xs and fp32 activation pointers must be
 *    16-byte aligned; outputs 4-byte aligned (DSQ_ERR_ALIGNMENT otherwise).
 *  - A device-side wait that exceeds its time limit (default 1 s) records
 *    DSQ_ERR_TIMEOUT in a device status word instead of hanging; read it
 *    with dsq_device_status().
 *  - Kernels are launched with programmatic stream serialization: each one
 *    waits for its predecessors (griddepcontrol.wait) before it reads
 *    activations or writes outputs.  Weights are read-only inputs: some
 *    decode GEMVs (Q4_K) start loading them before that wait.  So weights
 *    must not be written by a kernel that is still running when the call is
 *    launched -- a kernel that releases its dependents early
 *    (griddepcontrol.launch_dependents) before writing them.  Ordinary
 *    kernels and every kernel of this library meet this.
 */
#ifndef DSQ_H
#define DSQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum dsq_status {
    DSQ_OK = 0,
    DSQ_ERR_INVALID_ARG = 1,        /* null pointer, bad enum, negative size */
    DSQ_ERR_ALIGNMENT = 2,          /* pointer not aligned as required       */
    DSQ_ERR_SHAPE = 3,              /* K not a multiple of the block size, or
                                       a size beyond the supported range     */
    DSQ_ERR_UNSUPPORTED_DEVICE = 4, /* current device is not compute 10.0    */
    DSQ_ERR_WORKSPACE = 5,          /* workspace NULL or smaller than needed */
    DSQ_ERR_LAUNCH = 6,             /* the CUDA launch itself failed         */
    DSQ_ERR_TIMEOUT = 7,            /* a bounded device wait expired         */
    DSQ_ERR_CUDA = 8,               /* another CUDA runtime error            */
    DSQ_ERR_RANGE = 9               /* reported by dsq_device_status: a
                                       prefill weight block admits values
                                       outside the binary16 range            */
} dsq_status;

typedef enum dsq_type { DSQ_Q8_0 = 8, DSQ_Q4_K = 12 } dsq_type;

/* Bytes of one weight row of K elements; 0 if K does not fit the type
 * (Q8_0: K % 32 == 0, Q4_K: K % 256 == 0, K > 0). */
size_t dsq_row_bytes(int type, int64_t K);

/*
 * Activation prequantization [ds4-623 Summary; strix quantize_q8_1].
 * For every 32-element block of each row of x [M][K] (fp32):
 *   amax = max |x_i|;  xd = amax / 127 (IEEE fp32 division);
 *   xq_i = clamp(round_half_away_from_zero(x_i / xd), -127, 127)
 *          (IEEE division by the unrounded fp32 xd; all 0 when amax == 0);
 *   xs   = sum_i xq_i.
 * Bit-exact with the CPU oracle.  xs may be NULL (not written).
 * Requires K % 32 == 0.  M == 0 is a no-op.
 */
int dsq_quantize_act_q8(const float *x, int64_t M, int64_t K,
                        int8_t *xq, float *xd, int32_t *xs, void *stream);

/*
 * Regular decode GEMV, Q8_0 weights [ds4-623 per-stage comment,
 * matmul_q8_0_tensor]:  y[n] = sum_b (d_w[n,b] * xd[b]) * isum[n,b],
 * isum[n,b] = sum_{i<32} qw[n,32b+i] * xq[32b+i] (exact int32),
 * accumulated in fp32.  w: N rows; xq/xd: one prequantized row of K.
 * y: N fp32.  Requires K % 32 == 0; N == 0 is a no-op.
 */
int dsq_gemv_q8_0(const void *w, int64_t N, int64_t K,
                  const int8_t *xq, const float *xd, float *y, void *stream);

/*
 * Regular decode GEMV, Q4_K weights [ds4-621 AProjQ4 projections]:
 *   y[n] = sum_{superblock, j<8} (d*sc_j)*xd_b*isum_{n,b}
 *                              - (dmin*m_j)*xd_b*xs_b,   b = 8*sb + j,
 * isum the exact int32 dot of the 4-bit codes with xq, fp32 accumulation.
 * xs (block code sums from dsq_quantize_act_q8) is required.
 * Requires K % 256 == 0.
 */
int dsq_gemv_q4_k(const void *w, int64_t N, int64_t K,
                  const int8_t *xq, const float *xd, const int32_t *xs,
                  float *y, void *stream);

/*
 * Paired decode GEMV [ds4-623 matmul_q8_0_pair_tensor]: two weight tensors
 * (N0 and N1 rows, same K and type) against ONE shared prequantized
 * activation, in one launch: y0 = W0 x, y1 = W1 x.  type: DSQ_Q8_0 or
 * DSQ_Q4_K (xs required for Q4_K).  Either N may be 0.
 */
int dsq_gemv_paired(int type, const void *w0, int64_t N0, const void *w1, int64_t N1,
                    int64_t K, const int8_t *xq, const float *xd, const int32_t *xs,
                    float *y0, float *y1, void *stream);

/*
 * Grouped low-rank attention-output GEMV [ds4-623
 * attention_output_low_q8_tensor; llama tensor shape [4096, 1024, 8]]:
 * G independent products y_g = W_g x_g in one launch.  w holds G*N rows:
 * group g's rows start at byte g*N*dsq_row_bytes(type, K) (ggml [K, N, G]).
 * xq [G][K], xd [G][K/32], xs [G][K/32] (Q4_K only), y [G][N].
 */
int dsq_gemv_grouped(int type, const void *w, int64_t G, int64_t N, int64_t K,
                     const int8_t *xq, const float *xd, const int32_t *xs,
                     float *y, void *stream);

/*
 * The three decode GEMV forms with the activation given in fp32: the same
 * computation as dsq_quantize_act_q8 followed by dsq_gemv_q8_0 / _q4_k,
 * dsq_gemv_paired or dsq_gemv_grouped (the activation prequantized to Q8
 * per 32-block once and shared by every row that reads it [ds4-623 Summary;
 * strix]), in one launch: each CTA quantizes the activation rows into its
 * shared memory while its first weight copies are in flight.  The outputs
 * equal those of the two-call path bit for bit; the quantized activation is
 * not written out.
 *   x: fp32 [rows][K], 16-byte aligned, rows = 1 (single, paired) or G
 *      (grouped, group g's row at x + g*K).
 * Requires K % 256 == 0 (both types) and rows*(K + 8*K/32) <= 65536 bytes
 * (e.g. 8 rows of K = 4096, or one row of K <= 52428); otherwise
 * DSQ_ERR_SHAPE and nothing is launched.  Other arguments, layouts and
 * errors as in the corresponding two-call entry points.
 */
int dsq_gemv_f32(int type, const void *w, int64_t N, int64_t K, const float *x,
                 float *y, void *stream);
int dsq_gemv_paired_f32(int type, const void *w0, int64_t N0, const void *w1,
                        int64_t N1, int64_t K, const float *x, float *y0,
                        float *y1, void *stream);
int dsq_gemv_grouped_f32(int type, const void *w, int64_t G, int64_t N,
                         int64_t K, const float *x, float *y, void *stream);

/*
 * Multi-token decode GEMV [ds4-621 GB10 report: the grouped-tok8 and
 * QKV-pair paths for short batches of up to 8 tokens; ds4-623 Summary: the
 * activation is prequantized to Q8 once and shared]: M = 1..8 prequantized
 * activation rows against W0 (N0 rows) and, optionally, a second weight W1
 * (N1 rows, same type and K; the Q / KV projections that read one input),
 * in one launch that reads every weight byte once for all M tokens:
 *   y0[m][n] = (W0 x_m)[n],  y1[m][n] = (W1 x_m)[n],  m < M.
 * xq [M][K], xd [M][K/32], xs [M][K/32] (Q4_K only; may be NULL for Q8_0),
 * y0 [M][N0], y1 [M][N1] (row-major, fp32).  Each token's outputs equal bit
 * for bit those of dsq_gemv_q8_0 / dsq_gemv_q4_k / dsq_gemv_paired called
 * for that token alone.  Either N may be 0 (its pointers are then unused).
 * Requires K % 256 == 0, 1 <= M <= 8 and M * (K + K/8 (+ K/8 for Q4_K)) <=
 * 65536 bytes (e.g. 8 tokens of K = 4096); otherwise DSQ_ERR_SHAPE and
 * nothing is launched.  Weights 16-byte aligned, as for every GEMV.
 */
int dsq_gemv_tokens(int type, const void *w0, int64_t N0, const void *w1, int64_t N1,
                    int64_t K, int64_t M, const int8_t *xq, const float *xd,
                    const int32_t *xs, float *y0, float *y1, void *stream);

/*
 * Prefill dequantize-into-dense-GEMM [ds4-621 GB10 report: "dequant + GEMM
 * prefill path"]:  Y[M][N] = X[M][K] * deq(W)^T, X fp32 row-major, Y fp32
 * row-major.  Tensor-core contraction with 16-bit float operands and fp32
 * accumulation:
 *   - each X row m is scaled by an exact power of two 2^s_m chosen so its
 *     largest magnitude lies in [2^14, 2^15) (s_m = 0 for a zero row,
 *     clamped to [-113, 126]: every finite row with max |x| >= 2^-112 lands
 *     in that binade, up to FLT_MAX) and rounded to IEEE binary16 (RNE);
 *   - each weight element is dequantized in fp32 (Q8_0: d*q; Q4_K:
 *     (d*sc)*q - dmin*m) and rounded to binary16 (RNE);
 *   - the fp32 sum over K is scaled back by 2^-s_m.
 * Error vs the fp64 dequantized reference: relative L2 ~3e-4 on N(0,1)
 * activations and N(0, 0.02^2) weights (gate 2e-3).
 * Determinism: the sum over K may be cut into pieces computed by different
 * SMs (all tiles of a small problem, or only the tiles of a short last wave
 * of a large one); the plan depends only on the shape and the device's SM
 * count, and the pieces are added in a fixed order, so repeated calls give
 * the same bits.
 * Weight range: dequantized weights must lie inside the binary16 range.  A
 * block whose scales admit a value of magnitude >= 65520 -- a Q8_0 block
 * with |d|*127 >= 65520, or a Q4_K sub-block whose code-0 or code-15 value
 * (-dmin*m or 15*d*sc - dmin*m, in fp32) reaches 65520 -- makes the kernel
 * record DSQ_ERR_RANGE in the device status word (read it with
 * dsq_device_status); the outputs that read such a block are inf or NaN.
 * Weights below 2^-14 in magnitude become binary16 subnormals (absolute
 * spacing 2^-24) and keep less relative precision.
 * workspace: device scratch of at least dsq_prefill_workspace_bytes(...)
 * bytes, 256-byte aligned, used only for the duration of the call's kernels
 * on `stream`.  Requires K % 256 == 0 for both types, 1 <= M, N >= 1.
 */
int dsq_gemm_prefill(int type, const void *w, int64_t N, int64_t K,
                     const float *x, int64_t M, float *y,
                     void *workspace, size_t workspace_bytes, void *stream);

size_t dsq_prefill_workspace_bytes(int type, int64_t N, int64_t K, int64_t M);

/*
 * Grouped prefill [ds4-621 consolidated results: the grouped attention-A
 * prefill path, which computes several attention-A projections that read the
 * same input in one launch]: G = 1..DSQ_PREFILL_MAX_GROUP weights of the same
 * type and K (weight g: N[g] rows at w[g]) against ONE activation X [M][K]:
 *   y[g][m][n] = (X * deq(W_g)^T)[m][n],   y[g] row-major [M][N[g]].
 * X is converted to binary16 once and one GEMM launch covers the weight-row
 * tiles of all G weights.  Numerics, layouts, alignment and errors are those
 * of dsq_gemm_prefill for every weight; w, N and y are HOST arrays of G
 * entries (the pointers in them are device pointers).  The split of K (if
 * any) is planned over all G weights' tiles together; whenever it comes out
 * the same as for a weight alone -- in particular when neither splits K --
 * y[g] equals dsq_gemm_prefill's result for that weight bit for bit.
 * workspace: at least dsq_prefill_grouped_workspace_bytes(type, G, N, K, M)
 * bytes, 256-byte aligned.
 */
#define DSQ_PREFILL_MAX_GROUP 4
int dsq_gemm_prefill_grouped(int type, int64_t G, const void *const *w, const int64_t *N,
                             int64_t K, const float *x, int64_t M, float *const *y,
                             void *workspace, size_t workspace_bytes, void *stream);
size_t dsq_prefill_grouped_workspace_bytes(int type, int64_t G, const int64_t *N, int64_t K,
                                           int64_t M);

/*
 * Allocation-free prefill: dsq_gemm_prefill without a workspace argument.
 * The paper has no counterpart; this entry point exists for callers that
 * cannot allocate device memory when they call -- for example code that
 * runs under a fixed device-memory budget reserved up front, a plugin that
 * is handed only its input and output buffers by a host framework with no
 * workspace hook, or a caller inside a region where cudaMalloc is not
 * allowed (such as a global-mode stream capture).
 *
 * Scratch lives in a fixed 32 MiB array in device memory that every device
 * loading libdsq reserves until the process exits.  Problems whose
 * dsq_prefill_workspace_bytes(type, N, K, M) exceeds
 * DSQ_PREFILL_NOALLOC_SCRATCH_BYTES are rejected with DSQ_ERR_WORKSPACE and
 * nothing is launched; otherwise arguments, layout, numerics and errors are
 * those of dsq_gemm_prefill.  No call allocates or frees device memory.
 *
 * The first call on a device performs a one-time set-up (it looks up the
 * device address of the scratch array in the current CUDA context; a new
 * context -- after cudaDeviceReset, or a driver context the caller made
 * current -- repeats it once); make that first call before any stream
 * capture.  All calls on a device share the one scratch array, so
 * calls that may overlap on the GPU (different streams without ordering,
 * or concurrent host threads) race and must be serialized by the caller.
 * Nothing in the array needs to be cleared between calls: each call writes
 * every scratch byte it later reads.
 */
#define DSQ_PREFILL_NOALLOC_SCRATCH_BYTES (32ull * 1024ull * 1024ull)
int dsq_gemm_prefill_noalloc(int type, const void *w, int64_t N, int64_t K,
                             const float *x, int64_t M, float *y, void *stream);

/*
 * Offline weight quantizer (device): fp32 rows x [N][K] -> packed rows in w
 * (N * dsq_row_bytes bytes).  Q8_0: d = fp16(amax/127), q from the fp32
 * scale, round half away from zero.  Q4_K (the pages give no quantizer; a
 * plain min/max rule): per sub-block lo = min(0, min x), hi = max x,
 * s_j = (hi-lo)/15, mm_j = -lo; d = fp16(max s_j / 63), dmin = fp16(max mm_j
 * / 63); sc_j, m_j, q by round half away from zero with clamping.
 * Bit-exact with the CPU oracle.  w needs only 2-byte alignment.
 */
int dsq_quantize_weights(int type, const float *x, int64_t N, int64_t K,
                         void *w, void *stream);

/* Synchronizes `stream`, then returns and clears the device status word of
 * the current device: DSQ_OK; DSQ_ERR_TIMEOUT if a bounded device wait
 * expired since the last read; else DSQ_ERR_RANGE if a prefill kernel met a
 * weight block outside the binary16 range (see dsq_gemm_prefill). */
int dsq_device_status(void *stream);

/* Human-readable description of the last error on this host thread. */
const char *dsq_last_error(void);
const char *dsq_version(void);

/* Number of kernels this library has launched in this process. */
uint64_t dsq_launch_count(void);

#ifdef __cplusplus
}
#endif
#endif /* DSQ_H */
