// quantize.cu -- activation prequantization to Q8 per 32-block (the decode
// step that feeds every quantized projection, "ROCm: restore DeepSeek V4
// Flash decode performance", Summary; quantize_q8_1 in "DeepSeek V4 Flash on
// Strix Halo", "Why I did not keep a ROCm kernel patch"), and the offline
// Q8_0 / Q4_K weight quantizers.
//
// All float steps are single IEEE operations with explicit rounding
// (__fdiv_rn / __fmul_rn / __fadd_rn / __fsub_rn, no contraction) so the
// codes and scales are bit-identical to the CPU oracle's.
#include "act_q8.cuh"
#include "dsq_host.h"

namespace dsq {
namespace {

// One 32-element block is handled by 8 consecutive lanes, 4 elements each
// (one float4 load per lane; a warp covers 4 blocks = 512 contiguous bytes).

__global__ void __launch_bounds__(256) act_q8_kernel(const float4 *__restrict__ x, int64_t nblocks,
                                                     int8_t *__restrict__ xq, float *__restrict__ xd,
                                                     int32_t *__restrict__ xs) {
  if (threadIdx.x == 0) {
    // this CTA's slice of x toward L2 while the previous kernel finishes (a
    // hint: L2 is the point of coherence, so the predecessor's writes win)
    const int64_t f0 = static_cast<int64_t>(blockIdx.x) * blockDim.x;
    const int64_t nf = min(static_cast<int64_t>(blockDim.x), nblocks * 8 - f0);
    if (nf > 0) prefetch_l2(x + f0, static_cast<uint32_t>(nf * 16));
  }
  pdl_trigger();
  pdl_wait();
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t blk = tid >> 3;
  const int sub = threadIdx.x & 7;
  const bool live = blk < nblocks;
  const float4 v = live ? __ldg(&x[blk * 8 + sub]) : make_float4(0.f, 0.f, 0.f, 0.f);
  float d;
  int s;
  const uint32_t packed = q8_block_lanes(v, d, s);
  if (!live) return;
  reinterpret_cast<uint32_t *>(xq)[blk * 8 + sub] = packed;
  if (sub == 0) {
    xd[blk] = d;
    if (xs) xs[blk] = s;
  }
}

// Q8_0 weight blocks: same rule, the stored scale is fp16(d32).  The 34-byte
// block is only 2-byte aligned, so codes are stored as 16-bit pairs.
__global__ void __launch_bounds__(256) weight_q8_0_kernel(const float4 *__restrict__ x, int64_t nblocks,
                                                          uint8_t *__restrict__ w) {
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t blk = tid >> 3;
  const int sub = threadIdx.x & 7;
  const bool live = blk < nblocks;
  float4 v = live ? __ldg(&x[blk * 8 + sub]) : make_float4(0.f, 0.f, 0.f, 0.f);
  float amax = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
#pragma unroll
  for (int o = 4; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if (!live) return;
  const float d = __fdiv_rn(amax, 127.0f);
  const int q0 = static_cast<int>(q8_code(v.x, d));
  const int q1 = static_cast<int>(q8_code(v.y, d));
  const int q2 = static_cast<int>(q8_code(v.z, d));
  const int q3 = static_cast<int>(q8_code(v.w, d));
  uint8_t *b = w + blk * 34;
  uint16_t *q16 = reinterpret_cast<uint16_t *>(b + 2 + 4 * sub);
  q16[0] = static_cast<uint16_t>((q0 & 0xff) | ((q1 & 0xff) << 8));
  q16[1] = static_cast<uint16_t>((q2 & 0xff) | ((q3 & 0xff) << 8));
  if (sub == 0) *reinterpret_cast<uint16_t *>(b) = __half_as_ushort(__float2half_rn(d));
}

__device__ __forceinline__ float clampf(float v, float lo, float hi) { return fminf(fmaxf(v, lo), hi); }

// Q4_K weight super-blocks: one thread per 256 elements, in the order the
// plain min/max rule is stated (offline; simplicity over speed).
__global__ void __launch_bounds__(128) weight_q4_k_kernel(const float *__restrict__ x, int64_t nsb,
                                                          uint8_t *__restrict__ w) {
  const int64_t sbi = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (sbi >= nsb) return;
  const float *xs = x + sbi * 256;
  uint8_t *blk = w + sbi * 144;
  float s[8], mm[8];
  float smax = 0.0f, mmax = 0.0f;
  for (int j = 0; j < 8; ++j) {
    float lo = 0.0f, hi = xs[32 * j];
    for (int l = 0; l < 32; ++l) {
      const float v = xs[32 * j + l];
      lo = v < lo ? v : lo;
      hi = v > hi ? v : hi;
    }
    s[j] = __fdiv_rn(__fsub_rn(hi, lo), 15.0f);
    mm[j] = -lo;
    smax = s[j] > smax ? s[j] : smax;
    mmax = mm[j] > mmax ? mm[j] : mmax;
  }
  const __half dh = __float2half_rn(__fdiv_rn(smax, 63.0f));
  const __half mh = __float2half_rn(__fdiv_rn(mmax, 63.0f));
  const float d = __half2float(dh), dmin = __half2float(mh);
  uint8_t sc_b[12];
  for (int i = 0; i < 12; ++i) sc_b[i] = 0;
  uint8_t qs[128];
  for (int i = 0; i < 128; ++i) qs[i] = 0;
  for (int j = 0; j < 8; ++j) {
    const int sc = d > 0.0f ? static_cast<int>(clampf(roundf(__fdiv_rn(s[j], d)), 0.0f, 63.0f)) : 0;
    const int m = dmin > 0.0f ? static_cast<int>(clampf(roundf(__fdiv_rn(mm[j], dmin)), 0.0f, 63.0f)) : 0;
    if (j < 4) {
      sc_b[j] = static_cast<uint8_t>((sc_b[j] & 0xc0) | sc);
      sc_b[j + 4] = static_cast<uint8_t>((sc_b[j + 4] & 0xc0) | m);
    } else {
      sc_b[j + 4] = static_cast<uint8_t>((sc & 15) | ((m & 15) << 4));
      sc_b[j - 4] = static_cast<uint8_t>((sc_b[j - 4] & 0x3f) | ((sc >> 4) << 6));
      sc_b[j] = static_cast<uint8_t>((sc_b[j] & 0x3f) | ((m >> 4) << 6));
    }
    const float den = __fmul_rn(d, static_cast<float>(sc));
    const float off = __fmul_rn(dmin, static_cast<float>(m));
    for (int l = 0; l < 32; ++l) {
      int q = 0;
      if (den != 0.0f) {
        const float t = __fadd_rn(xs[32 * j + l], off);
        q = static_cast<int>(clampf(roundf(__fdiv_rn(t, den)), 0.0f, 15.0f));
      }
      uint8_t &byte = qs[32 * (j / 2) + l];
      byte = (j & 1) ? static_cast<uint8_t>((byte & 0x0f) | (q << 4)) : static_cast<uint8_t>((byte & 0xf0) | q);
    }
  }
  *reinterpret_cast<uint16_t *>(blk) = __half_as_ushort(dh);
  *reinterpret_cast<uint16_t *>(blk + 2) = __half_as_ushort(mh);
  for (int i = 0; i < 12; ++i) blk[4 + i] = sc_b[i];
  for (int i = 0; i < 128; ++i) blk[16 + i] = qs[i];
}

}  // namespace
}  // namespace dsq

extern "C" int dsq_quantize_act_q8(const float *x, int64_t M, int64_t K, int8_t *xq, float *xd,
                                   int32_t *xs, void *stream) {
  using namespace dsq;
  DSQ_REQUIRE(M >= 0 && K > 0, DSQ_ERR_INVALID_ARG, "dsq_quantize_act_q8: M=%lld K=%lld", (long long)M,
              (long long)K);
  DSQ_REQUIRE(K % 32 == 0, DSQ_ERR_SHAPE, "dsq_quantize_act_q8: K=%lld is not a multiple of 32", (long long)K);
  DSQ_REQUIRE(M <= (int64_t(1) << 31) && K <= (int64_t(1) << 31), DSQ_ERR_SHAPE,
              "dsq_quantize_act_q8: size out of range");
  if (M == 0) return DSQ_OK;
  DSQ_REQUIRE(x && xq && xd, DSQ_ERR_INVALID_ARG, "dsq_quantize_act_q8: null pointer");
  DSQ_REQUIRE(aligned(x, 16) && aligned(xq, 16) && aligned(xd, 16) && (!xs || aligned(xs, 16)),
              DSQ_ERR_ALIGNMENT, "dsq_quantize_act_q8: x/xq/xd/xs must be 16-byte aligned");
  int rc = device_ready(nullptr, nullptr);
  if (rc != DSQ_OK) return rc;
  const int64_t nblocks = M * (K / 32);
  const int64_t threads = nblocks * 8;
  const unsigned grid = static_cast<unsigned>((threads + 255) / 256);
  const cudaError_t e = launch_pdl(act_q8_kernel, dim3(grid), dim3(256), 0, as_stream(stream),
                                   reinterpret_cast<const float4 *>(x), nblocks, xq, xd, xs);
  if (e != cudaSuccess) return fail(DSQ_ERR_LAUNCH, "dsq_quantize_act_q8: %s", cudaGetErrorString(e));
  return after_launch("dsq_quantize_act_q8");
}

extern "C" int dsq_quantize_weights(int type, const float *x, int64_t N, int64_t K, void *w, void *stream) {
  using namespace dsq;
  DSQ_REQUIRE(type == DSQ_Q8_0 || type == DSQ_Q4_K, DSQ_ERR_INVALID_ARG, "dsq_quantize_weights: type %d", type);
  DSQ_REQUIRE(N >= 0 && K > 0, DSQ_ERR_INVALID_ARG, "dsq_quantize_weights: N=%lld K=%lld", (long long)N,
              (long long)K);
  DSQ_REQUIRE(dsq_row_bytes(type, K) != 0, DSQ_ERR_SHAPE, "dsq_quantize_weights: K=%lld does not fit type %d",
              (long long)K, type);
  DSQ_REQUIRE(N <= (int64_t(1) << 31) && K <= (int64_t(1) << 31), DSQ_ERR_SHAPE,
              "dsq_quantize_weights: size out of range");
  if (N == 0) return DSQ_OK;
  DSQ_REQUIRE(x && w, DSQ_ERR_INVALID_ARG, "dsq_quantize_weights: null pointer");
  DSQ_REQUIRE(aligned(x, 16) && aligned(w, 2), DSQ_ERR_ALIGNMENT,
              "dsq_quantize_weights: x must be 16-byte and w 2-byte aligned");
  int rc = device_ready(nullptr, nullptr);
  if (rc != DSQ_OK) return rc;
  if (type == DSQ_Q8_0) {
    const int64_t nblocks = N * (K / 32);
    const unsigned grid = static_cast<unsigned>((nblocks * 8 + 255) / 256);
    weight_q8_0_kernel<<<grid, 256, 0, as_stream(stream)>>>(reinterpret_cast<const float4 *>(x), nblocks,
                                                            static_cast<uint8_t *>(w));
  } else {
    const int64_t nsb = N * (K / 256);
    const unsigned grid = static_cast<unsigned>((nsb + 127) / 128);
    weight_q4_k_kernel<<<grid, 128, 0, as_stream(stream)>>>(x, nsb, static_cast<uint8_t *>(w));
  }
  return after_launch("dsq_quantize_weights");
}
