// act_q8.cuh -- activation prequantization to Q8 per 32-block, as a warp
// building block shared by the stand-alone quantizer and the GEMV that
// quantizes its own activation ("ROCm: restore DeepSeek V4 Flash decode
// performance", Summary: the activation is quantized once and shared by the
// projections that read it).
//
// Rule: d = amax / 127 (IEEE division), q = clamp(round-half-away(x / d),
// -127, 127) using the unrounded fp32 d, q = 0 for an all-zero block; the
// block code sum s = sum q serves the Q4_K min term.  Every float step is a
// single IEEE operation with explicit rounding, so codes and scales are
// bit-identical to the CPU oracle's.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace dsq {

__device__ __forceinline__ float q8_code(float x, float d) {
  if (d == 0.0f) return 0.0f;
  float v = roundf(__fdiv_rn(x, d));   // roundf: half away from zero
  return fminf(fmaxf(v, -127.0f), 127.0f);
}

// One 32-element block per 8 consecutive lanes (lane & 7 = the lane's float4
// within the block), 4 elements per lane in v.  All 32 lanes of the warp must
// call it together (xor shuffles inside aligned groups of 8); a lane with no
// block passes zeros.  Returns the lane's 4 codes packed little-endian; d and
// the block's code sum come back in every lane of the group.
__device__ __forceinline__ uint32_t q8_block_lanes(float4 v, float &d, int &s) {
  float amax = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
#pragma unroll
  for (int o = 4; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  d = __fdiv_rn(amax, 127.0f);
  const int q0 = static_cast<int>(q8_code(v.x, d));
  const int q1 = static_cast<int>(q8_code(v.y, d));
  const int q2 = static_cast<int>(q8_code(v.z, d));
  const int q3 = static_cast<int>(q8_code(v.w, d));
  s = q0 + q1 + q2 + q3;
#pragma unroll
  for (int o = 4; o >= 1; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  return (static_cast<uint32_t>(q0) & 0xffu) | ((static_cast<uint32_t>(q1) & 0xffu) << 8) |
         ((static_cast<uint32_t>(q2) & 0xffu) << 16) | ((static_cast<uint32_t>(q3) & 0xffu) << 24);
}

}  // namespace dsq
