// gemv.cu -- decode GEMV with the activation prequantized to Q8 per 32-block:
// regular, paired (two weights sharing one activation) and grouped low-rank
// attention-output (G independent weight/activation pairs), for Q8_0 and
// Q4_K weights.
//
// Sources: "ROCm: restore DeepSeek V4 Flash decode performance and Q4 SSD
// streaming" (antirez/ds4 PR #623) -- Summary (prequantized Q8 decode for
// regular, paired and low-rank attention-output projections) and the
// per-stage timing comment (matmul_q8_0_tensor, matmul_q8_0_pair_tensor,
// attention_output_low_q8_tensor; the fast kernels run a warp per output
// row, the slow ones a 256-thread block per row); "Support AProjQ4 GGUFs"
// (antirez/ds4 PR #621) for the Q4_K projections; "DeepSeek V4"
// (ggml-org/llama.cpp PR #24162) for the [4096, 1024, 8] grouped layout.
//
// B200 design (HBM-bound weight stream):
//  * A CTA owns a contiguous, balanced range of weight rows.  Each warp runs
//    its own ring of shared-memory slots, filled by cp.async.bulk (one
//    elected lane, completion on an mbarrier, L2 evict-first): deep bytes
//    in flight per SM without register staging, perfectly coalesced.
//  * A row is split into 256-element units (8 Q8_0 blocks = 272 B, or one
//    Q4_K super-block = 144 B, both 16-byte multiples).  G lanes share a row
//    (G = units per row rounded up to a power of two, at most 32), so a warp
//    holds 32/G rows per slot and lane j takes units j, j+G, ...
//  * The lane's 256-element activation slice (xq, xd, xs) is cached in
//    registers for as long as its (group, unit) does not change -- for
//    K <= 8192 that is every row the warp touches.
//  * Per 32-block: 8 dp4a give the exact int32 dot; the block term is
//    (d_w * xd) * isum in fp32; lanes reduce with xor-shuffles; one store
//    per row.  Rows whose byte length is not a multiple of 16 (Q8_0 with
//    K % 256 != 0) take a plain warp-per-row kernel instead.
//  * The *_f32 entry points take the fp32 activation and quantize it inside
//    the GEMV: each CTA starts its weight copies, then its 256 threads
//    quantize every activation row into shared memory (the rule of
//    act_q8.cuh), and the lanes read their slices from there.  Same codes,
//    same dot order -- the outputs equal the two-call path bit for bit --
//    but one launch per call instead of two.
#include "../../include/dsq_test.h"
#include "act_q8.cuh"
#include "dsq_host.h"

// Launch shape (compile-time constants; the defaults are the tuned values).
#ifndef DSQ_GEMV_MAX_WARPS
#define DSQ_GEMV_MAX_WARPS 8
#endif
#ifndef DSQ_GEMV_SMEM_KB
#define DSQ_GEMV_SMEM_KB 220
#endif
#ifndef DSQ_GEMV_MAX_STAGES
#define DSQ_GEMV_MAX_STAGES 2
#endif
#ifndef DSQ_GEMV_CTAS_PER_SM
#define DSQ_GEMV_CTAS_PER_SM 1
#endif
// Long Q4_K matrices: more warps, once every CTA has at least this many
// rows (12 warps of at most 168 registers, 16 of at most 128).
// Single matrices from this many rows up to one 32-row group per SM (one
// token) run the multi-token kernel.
#ifndef DSQ_GEMV_TOK_MIN_ROWS
#define DSQ_GEMV_TOK_MIN_ROWS 2048
#endif
#ifndef DSQ_GEMV_MID_MIN_ROWS
#define DSQ_GEMV_MID_MIN_ROWS 140
#endif
#ifndef DSQ_GEMV_WIDE_MIN_ROWS
#define DSQ_GEMV_WIDE_MIN_ROWS 300
#endif

namespace dsq {
namespace {

struct Seg {
  const uint8_t *w;
  float *y;
  int64_t rows;
};

struct GemvArgs {
  Seg seg[2];
  int64_t rows0;        // rows of seg[0]; seg[1] follows in the virtual row space
  int64_t total_rows;   // rows0 + rows of seg[1]
  int64_t group_rows;   // rows per activation group inside a segment
  const int8_t *xq;
  const float *xd;
  const int32_t *xs;
  int64_t K;
  int64_t row_bytes;
  int nunits;           // K / 256 (fast kernel)
  int warps;            // warps per CTA
  int stages;           // ring slots per warp
  int slot_bytes;       // rows-per-slot * row_bytes
  WaitCtl wait;
  int32_t *isum;        // test hook: per-block int32 sums (NULL in production)
  const float *x32;     // fused mode: fp32 activation rows [act_rows][K], quantized in the kernel
  int64_t act_rows;     // activation rows (1, or the group count)
  int act_off;          // fused mode: byte offset of the activation area in shared memory
};

template <int TYPE> struct Unit;
template <> struct Unit<DSQ_Q8_0> { static constexpr int kBytes = 272; };
template <> struct Unit<DSQ_Q4_K> { static constexpr int kBytes = 144; };

__device__ __forceinline__ float half_lo(uint32_t w) { return __half2float(__ushort_as_half(static_cast<unsigned short>(w & 0xffffu))); }
__device__ __forceinline__ float half_hi(uint32_t w) { return __half2float(__ushort_as_half(static_cast<unsigned short>(w >> 16))); }

// Activation slice of one 256-element unit, held in registers.
struct ActSlice {
  uint32_t q[64];   // 256 int8 codes
  float d[8];       // 8 block scales
  int32_t s[8];     // 8 block code sums (Q4_K only)
};

// The slice of one unit from the prequantized rows in global memory
// (read-only path): codes, scales and sums are contiguous.
template <int TYPE>
__device__ __forceinline__ void load_act(ActSlice &act, const int8_t *xq, const float *xd, const int32_t *xs) {
  const uint4 *q4 = reinterpret_cast<const uint4 *>(xq);
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint4 v = __ldg(q4 + i);
    act.q[4 * i + 0] = v.x; act.q[4 * i + 1] = v.y; act.q[4 * i + 2] = v.z; act.q[4 * i + 3] = v.w;
  }
  const float4 *d4 = reinterpret_cast<const float4 *>(xd);
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float4 v = __ldg(d4 + i);
    act.d[4 * i + 0] = v.x; act.d[4 * i + 1] = v.y; act.d[4 * i + 2] = v.z; act.d[4 * i + 3] = v.w;
  }
  if (TYPE == DSQ_Q4_K) {
    const int4 *s4 = reinterpret_cast<const int4 *>(xs);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int4 v = __ldg(s4 + i);
      act.s[4 * i + 0] = v.x; act.s[4 * i + 1] = v.y; act.s[4 * i + 2] = v.z; act.s[4 * i + 3] = v.w;
    }
  }
}

// Shared-memory activation area (fused and staged modes), per activation
// row: the codes as [16][nunits] 16-byte words (word i of unit u at
// i * nunits + u) and the scales and sums each as [2][nunits] 16-byte words.
// The G lanes of a row read G consecutive units at once, so they touch
// consecutive 16-byte words instead of the same bank 16 times.
__device__ __forceinline__ uint32_t act_q_word(uint32_t w, uint32_t nunits) {   // w: 4-code word of the row
  return (((w & 63u) >> 2) * nunits + (w >> 6)) * 4u + (w & 3u);
}
__device__ __forceinline__ uint32_t act_s_word(uint32_t b, uint32_t nunits) {   // b: 32-block of the row
  return (((b & 7u) >> 2) * nunits + (b >> 3)) * 4u + (b & 3u);
}

template <int TYPE>
__device__ __forceinline__ void load_act_smem(ActSlice &act, const int8_t *qrow, const float *drow,
                                              const int32_t *srow, int u, int nunits) {
  const uint4 *q4 = reinterpret_cast<const uint4 *>(qrow) + u;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint4 v = q4[i * nunits];
    act.q[4 * i + 0] = v.x; act.q[4 * i + 1] = v.y; act.q[4 * i + 2] = v.z; act.q[4 * i + 3] = v.w;
  }
  const float4 *d4 = reinterpret_cast<const float4 *>(drow) + u;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float4 v = d4[i * nunits];
    act.d[4 * i + 0] = v.x; act.d[4 * i + 1] = v.y; act.d[4 * i + 2] = v.z; act.d[4 * i + 3] = v.w;
  }
  if (TYPE == DSQ_Q4_K) {
    const int4 *s4 = reinterpret_cast<const int4 *>(srow) + u;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int4 v = s4[i * nunits];
      act.s[4 * i + 0] = v.x; act.s[4 * i + 1] = v.y; act.s[4 * i + 2] = v.z; act.s[4 * i + 3] = v.w;
    }
  }
}

// Where the dot loop reads its activation slices: global memory (the
// prequantized rows), shared memory quantized by the CTA itself from fp32 (the
// fused entry points), or shared memory copied once from the prequantized
// groups (the grouped form: a warp whose rows cross into the next group then
// reloads its slice from shared memory instead of waiting on L2).
enum : int { kActGlobal = 0, kActFused = 1, kActStaged = 2 };

// Staged mode: the CTA's threads copy prequantized activation groups
// [g0, g0 + rows) into the shared-memory area (at most 64 KB, so 32-bit
// indices suffice).
__device__ __forceinline__ void copy_act_to_smem(const GemvArgs &a, int64_t g0, int64_t rows, int8_t *sq,
                                                 float *sd, int32_t *ss) {
  const uint32_t nunits = static_cast<uint32_t>(a.nunits);
  const uint32_t q_row = nunits * 16u, s_row = nunits * 2u;   // 16-byte words per row: codes, scales
  const uint32_t nq = static_cast<uint32_t>(rows) * q_row, ns = static_cast<uint32_t>(rows) * s_row;
  const uint4 *q = reinterpret_cast<const uint4 *>(a.xq + g0 * a.K);
  for (uint32_t g = threadIdx.x; g < nq; g += blockDim.x) {
    const uint32_t r = g / q_row, gg = g - r * q_row;   // row; word gg = 16 codes of unit gg / 16
    reinterpret_cast<uint4 *>(sq)[r * q_row + (gg & 15u) * nunits + (gg >> 4)] = __ldg(q + g);
  }
  const uint4 *d = reinterpret_cast<const uint4 *>(a.xd + g0 * (a.K / 32));
  const uint4 *x = a.xs ? reinterpret_cast<const uint4 *>(a.xs + g0 * (a.K / 32)) : nullptr;
  for (uint32_t f = threadIdx.x; f < ns; f += blockDim.x) {
    const uint32_t r = f / s_row, ff = f - r * s_row;   // row; word ff = 4 blocks of unit ff / 2
    const uint32_t dst = r * s_row + (ff & 1u) * nunits + (ff >> 1);
    reinterpret_cast<uint4 *>(sd)[dst] = __ldg(d + f);
    if (x) reinterpret_cast<uint4 *>(ss)[dst] = __ldg(x + f);
  }
}

// Fused mode: the CTA's threads quantize activation rows [g0, g0 + rows)
// into shared memory (xq [rows][K] int8, then xd and xs [rows][K/32]).  8 lanes
// per 32-block, 4 elements each.  Each thread issues the loads of 4 float4s
// before quantizing them (one L2 round trip per batch, not per float4), and
// the loop runs the same number of iterations in every thread so each warp's
// shuffles see all 32 lanes.
__device__ __forceinline__ void quantize_act_to_smem(const GemvArgs &a, int64_t g0, int64_t rows, int8_t *sq,
                                                     float *sd, int32_t *ss) {
  constexpr int kBatch = 4;
  const int64_t tasks = rows * a.K / 4;   // float4s
  const uint32_t row_words = static_cast<uint32_t>(a.K / 4), nunits = static_cast<uint32_t>(a.nunits);
  const float4 *x4 = reinterpret_cast<const float4 *>(a.x32 + g0 * a.K);
  const int64_t step = static_cast<int64_t>(blockDim.x) * kBatch;
  for (int64_t base = 0; base < tasks; base += step) {
    float4 v[kBatch];
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const int64_t t = base + i * blockDim.x + threadIdx.x;
      v[i] = t < tasks ? __ldg(x4 + t) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const int64_t t = base + i * blockDim.x + threadIdx.x;
      float d;
      int sum;
      const uint32_t packed = q8_block_lanes(v[i], d, sum);
      if (t < tasks) {
        // the area is at most 64 KB: 32-bit indices
        const uint32_t r = static_cast<uint32_t>(t) / row_words, w = static_cast<uint32_t>(t) - r * row_words;
        reinterpret_cast<uint32_t *>(sq)[r * row_words + act_q_word(w, nunits)] = packed;
        if ((w & 7u) == 0) {
          const uint32_t b = r * (row_words / 8u) + act_s_word(w >> 3, nunits);
          sd[b] = d;
          ss[b] = sum;
        }
      }
    }
  }
}

// One Q8_0 unit (8 blocks, 272 bytes = 68 words) against its activation
// slice.  Block b starts at byte 34b: for even b the scale is the low half of
// word 17b/2 and the codes start two bytes later (realigned with a funnel
// shift); for odd b the scale is the high half of word (17b-1)/2 and the
// codes are word-aligned.
template <bool ISUM>
__device__ __forceinline__ float unit_q8_0(const uint8_t *p, const ActSlice &act, int32_t *isum_out) {
  uint32_t w[68];
  const uint4 *p4 = reinterpret_cast<const uint4 *>(p);
#pragma unroll
  for (int i = 0; i < 17; ++i) {
    const uint4 v = p4[i];
    w[4 * i + 0] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
  }
  float acc = 0.0f;
#pragma unroll
  for (int b = 0; b < 8; ++b) {
    int32_t s = 0;
    float dw;
    if ((b & 1) == 0) {
      const int a = 17 * b / 2;
      dw = half_lo(w[a]);
#pragma unroll
      for (int i = 0; i < 8; ++i) s = __dp4a(static_cast<int>(__funnelshift_r(w[a + i], w[a + i + 1], 16)),
                                             static_cast<int>(act.q[8 * b + i]), s);
    } else {
      const int a = (17 * b - 1) / 2;
      dw = half_hi(w[a]);
#pragma unroll
      for (int i = 0; i < 8; ++i) s = __dp4a(static_cast<int>(w[a + 1 + i]), static_cast<int>(act.q[8 * b + i]), s);
    }
    if (ISUM) isum_out[b] = s;
    acc += __fmul_rn(__fmul_rn(dw, act.d[b]), static_cast<float>(s));
  }
  return acc;
}

// One Q4_K super-block (144 bytes = 36 words): word 0 = d | dmin << 16,
// words 1..3 = the 12 scale bytes, words 4..35 = the 128 nibble bytes.
// Four unsigned bytes of a times four signed bytes of b, added to c.
__device__ __forceinline__ int32_t dp4a_us(uint32_t a, uint32_t b, int32_t c) {
  int32_t d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

template <bool ISUM>
__device__ __forceinline__ float unit_q4_k(const uint8_t *p, const ActSlice &act, int32_t *isum_out) {
  uint32_t w[36];
  const uint4 *p4 = reinterpret_cast<const uint4 *>(p);
#pragma unroll
  for (int i = 0; i < 9; ++i) {
    const uint4 v = p4[i];
    w[4 * i + 0] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
  }
  const float d = half_lo(w[0]), dmin = half_hi(w[0]);
  const uint32_t s0 = w[1], s1 = w[2], s2 = w[3];
  // bytes j of (scA, mA) are (sc_j, m_j) for j < 4; of (scB, mB) for j >= 4
  const uint32_t scA = s0 & 0x3f3f3f3fu;
  const uint32_t mA = s1 & 0x3f3f3f3fu;
  const uint32_t scB = (s2 & 0x0f0f0f0fu) | ((s0 >> 2) & 0x30303030u);
  const uint32_t mB = ((s2 >> 4) & 0x0f0f0f0fu) | ((s1 >> 2) & 0x30303030u);
  float acc = 0.0f;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint32_t scw = j < 4 ? scA : scB, mw = j < 4 ? mA : mB;
    const int sh = 8 * (j & 3);
    const float sc = static_cast<float>((scw >> sh) & 0xffu);
    const float m = static_cast<float>((mw >> sh) & 0xffu);
    // The high nibbles stay in place (16 x the code, an unsigned byte) and
    // the sum is divided by 16 once: Σ 16·q·x is an exact multiple of 16.
    int32_t s = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t byte4 = w[4 + 8 * (j >> 1) + i];
      const uint32_t nib = byte4 & ((j & 1) ? 0xf0f0f0f0u : 0x0f0f0f0fu);
      s = dp4a_us(nib, act.q[8 * j + i], s);
    }
    if (j & 1) s >>= 4;
    if (ISUM) isum_out[j] = s;
    const float t = __fmul_rn(__fmul_rn(d, sc), static_cast<float>(s));
    const float u = __fmul_rn(__fmul_rn(dmin, m), static_cast<float>(act.s[j]));
    acc += __fmul_rn(act.d[j], __fsub_rn(t, u));
  }
  return acc;
}

// Virtual row r -> (segment, row within segment).
__device__ __forceinline__ void locate(const GemvArgs &a, int64_t r, int &seg, int64_t &local) {
  if (r < a.rows0) { seg = 0; local = r; } else { seg = 1; local = r - a.rows0; }
}

// Issue the bulk copy of virtual rows [ra, rb) into a slot (split when the
// range crosses from segment 0 into segment 1).
__device__ __forceinline__ void issue_rows(const GemvArgs &a, int64_t ra, int64_t rb, uint8_t *dst, uint64_t *bar,
                                           uint64_t policy) {
  const uint32_t total = static_cast<uint32_t>((rb - ra) * a.row_bytes);
  mbar_arrive_expect_tx(bar, total);
  if (rb <= a.rows0) {
    bulk_g2s(dst, a.seg[0].w + ra * a.row_bytes, total, bar, policy);
  } else if (ra >= a.rows0) {
    bulk_g2s(dst, a.seg[1].w + (ra - a.rows0) * a.row_bytes, total, bar, policy);
  } else {
    const uint32_t n0 = static_cast<uint32_t>((a.rows0 - ra) * a.row_bytes);
    bulk_g2s(dst, a.seg[0].w + ra * a.row_bytes, n0, bar, policy);
    bulk_g2s(dst + n0, a.seg[1].w, total - n0, bar, policy);
  }
}

// MINB = 2: the overlapped launch.  The CTA fits half an SM (registers and
// shared memory), so the next call's CTA can be resident beside it; it issues
// its first weight slots before its launch-dependency wait and releases its
// own dependents only after that wait.
template <int TYPE, int G, bool ISUM, int ACT, int MAXW, int MINB>
__global__ void __launch_bounds__(32 * MAXW, MINB) gemv_kernel(const __grid_constant__ GemvArgs a) {
  constexpr int RPC = 32 / G;  // rows per slot
  constexpr bool EARLY = MINB > 1;
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int W = a.warps, S = a.stages;
  const int64_t r0 = a.total_rows * blockIdx.x / gridDim.x;
  const int64_t r1 = a.total_rows * (blockIdx.x + 1) / gridDim.x;
  const int64_t nchunks = (r1 - r0 + RPC - 1) / RPC;
  const int64_t mine = nchunks > warp ? (nchunks - warp + W - 1) / W : 0;
  uint8_t *ring = smem + static_cast<size_t>(warp) * S * a.slot_bytes;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + static_cast<size_t>(W) * S * a.slot_bytes) + warp * S;

  // Weights are read-only parameters: start pulling this warp's first slots
  // into L2 while the previous kernel (usually the activation quantizer)
  // finishes, then let the next kernel launch, then wait for our inputs.
  if (lane == 0) {
    for (int64_t k = 0; k < mine && k < S; ++k) {
      const int64_t c = warp + k * W;
      const int64_t ra = r0 + c * RPC, rb = min(ra + RPC, r1);
      if (rb <= a.rows0) {
        prefetch_l2(a.seg[0].w + ra * a.row_bytes, static_cast<uint32_t>((rb - ra) * a.row_bytes));
      } else if (ra >= a.rows0) {
        prefetch_l2(a.seg[1].w + (ra - a.rows0) * a.row_bytes, static_cast<uint32_t>((rb - ra) * a.row_bytes));
      }
    }
  }
  if (ACT != kActFused && threadIdx.x == 0) {
    // the prequantized activation rows this CTA reads (codes, scales, sums)
    // toward L2 as well: a row that the weight stream has pushed out of L2
    // cost 0.7 us per paired call before (12.14 us with the activation in
    // L2, 12.82 from HBM, 12.24 with this prefetch; interleaved A/B on B200)
    int64_t ga = 0, gb = 0;
    if (r1 > r0 && a.act_rows > 1) {
      ga = r0 / a.group_rows;
      gb = (r1 - 1) / a.group_rows;
    }
    const uint32_t nr = static_cast<uint32_t>(gb - ga + 1);
    prefetch_l2(a.xq + ga * a.K, nr * static_cast<uint32_t>(a.K));
    prefetch_l2(a.xd + ga * (a.K / 32), nr * static_cast<uint32_t>(a.K / 32) * 4);
    if (a.xs) prefetch_l2(a.xs + ga * (a.K / 32), nr * static_cast<uint32_t>(a.K / 32) * 4);
  }
  if (ACT == kActFused && threadIdx.x == 0) {
    // the fp32 activation rows this CTA will quantize, toward L2 (a hint:
    // the predecessor's writes still win, L2 being the point of coherence)
    int64_t ga = 0, gb = 0;
    if (r1 > r0 && a.act_rows > 1) {
      ga = r0 / a.group_rows;
      gb = (r1 - 1) / a.group_rows;
    }
    prefetch_l2(a.x32 + ga * a.K, static_cast<uint32_t>((gb - ga + 1) * a.K * 4));
  }
  // Everything that needs nothing from a predecessor is set up before the
  // wait: the slot barriers, the copy policy, and where this lane's first
  // activation slice lives.
  const uint64_t policy = l2_policy_evict_first();
  if (lane == 0 && mine > 0) {
    for (int s = 0; s < S; ++s) mbar_init(&bars[s], 1);
    fence_barrier_init();
  }
  const int sub = lane / G, j = lane % G;
  int64_t first_group = -1, first_key = -1;   // group and (group * nunits + unit) of that slice
  {
    const int64_t row = r0 + static_cast<int64_t>(warp) * RPC + sub;
    if (row < min(r0 + static_cast<int64_t>(warp) * RPC + RPC, r1) && j < a.nunits) {
      int seg;
      int64_t local;
      locate(a, row, seg, local);
      const int64_t group = local < a.group_rows ? 0 : local / a.group_rows;
      first_group = group;
      first_key = group * a.nunits + j;
    }
  }
  auto issue_first = [&]() {
    if (lane == 0 && mine > 0) {
      for (int64_t k = 0; k < mine && k < S; ++k) {
        const int64_t c = warp + k * W;
        const int64_t ra = r0 + c * RPC, rb = min(ra + RPC, r1);
        issue_rows(a, ra, rb, ring + k * a.slot_bytes, &bars[k], policy);
      }
    }
  };
  if constexpr (EARLY) {
    // The weights are read-only for the call, and every kernel of this
    // library that can precede this one releases it only after its own wait
    // or writes no weights, so the first slots load before the wait.
    issue_first();
    pdl_wait();
    pdl_trigger();
  } else {
    pdl_trigger();
    pdl_wait();
    issue_first();
  }
  if (ACT == kActGlobal && mine == 0) return;
  // activation source: global (two-call path) or quantized here, into shared
  // memory, while the first weight copies are in flight
  const int8_t *xq = a.xq;
  const float *xd = a.xd;
  const int32_t *xs = a.xs;
  if (ACT != kActGlobal) {
    // only the activation groups this CTA's rows read: [g0, g1]
    int64_t g0 = 0, g1 = 0;
    if (r1 > r0 && a.act_rows > 1) {
      g0 = r0 / a.group_rows;
      g1 = (r1 - 1) / a.group_rows;
    }
    const int64_t rows = g1 - g0 + 1;
    int8_t *sq = reinterpret_cast<int8_t *>(smem + a.act_off);
    float *sd = reinterpret_cast<float *>(sq + rows * a.K);
    int32_t *ss = reinterpret_cast<int32_t *>(sd + rows * (a.K / 32));
    if (ACT == kActFused) quantize_act_to_smem(a, g0, rows, sq, sd, ss);
    else copy_act_to_smem(a, g0, rows, sq, sd, ss);
    __syncthreads();
    if (mine == 0) return;
    // indexed by absolute group below: shift the bases by g0 rows
    xq = sq - g0 * a.K;
    xd = sd - g0 * (a.K / 32);
    xs = ss - g0 * (a.K / 32);
  }
  __syncwarp();

  // the activation slice of (group, unit u) into registers
  auto fetch_act = [&](ActSlice &dst, int64_t group, int u) {
    if (ACT == kActGlobal) {
      const int64_t e0 = group * a.K + static_cast<int64_t>(u) * 256;
      load_act<TYPE>(dst, xq + e0, xd + e0 / 32, TYPE == DSQ_Q4_K ? xs + e0 / 32 : nullptr);
    } else {
      load_act_smem<TYPE>(dst, xq + group * a.K, xd + group * (a.K / 32), xs + group * (a.K / 32), u, a.nunits);
    }
  };
  ActSlice act;
  int64_t cached = -1;  // (group * nunits + unit) currently in registers
  if (first_group >= 0) {
    // the slice of this lane's first (group, unit), loaded now so its
    // latency overlaps the first weight slot's instead of following it
    fetch_act(act, first_group, j);
    cached = first_key;
  }
  int slot = 0;         // ring position kept incrementally (no division per chunk)
  uint32_t parity = 0;
  for (int64_t k = 0; k < mine; ++k) {
    const bool ok = __all_sync(0xffffffffu, mbar_wait_for(&bars[slot], parity, a.wait.limit_ns));
    if (!ok) {
      if (lane == 0) {
        record_timeout(a.wait);
        for (int64_t kk = k; kk < mine && kk < k + S; ++kk)
          mbar_wait_for(&bars[kk % S], static_cast<uint32_t>((kk / S) & 1), kDrainLimitNs);
      }
      __syncwarp();
      return;
    }
    const int64_t c = warp + k * W;
    const int64_t ra = r0 + c * RPC, rb = min(ra + RPC, r1);
    const int64_t row = ra + sub;
    float acc = 0.0f;
    if (row < rb) {
      int seg;
      int64_t local;
      locate(a, row, seg, local);
      // rows and group sizes are below 2^31 (checked on the host): 32-bit division
      const int64_t group =
          local < a.group_rows ? 0 : static_cast<uint32_t>(local) / static_cast<uint32_t>(a.group_rows);
      const uint8_t *rowp = ring + static_cast<size_t>(slot) * a.slot_bytes + static_cast<size_t>(sub) * a.row_bytes;
      for (int u = j; u < a.nunits; u += G) {
        const int64_t key = group * a.nunits + u;
        if (key != cached) {
          fetch_act(act, group, u);
          cached = key;
        }
        int32_t is[8];
        if (TYPE == DSQ_Q8_0)
          acc += unit_q8_0<ISUM>(rowp + static_cast<size_t>(u) * Unit<TYPE>::kBytes, act, is);
        else
          acc += unit_q4_k<ISUM>(rowp + static_cast<size_t>(u) * Unit<TYPE>::kBytes, act, is);
        if (ISUM) {
#pragma unroll
          for (int b = 0; b < 8; ++b) a.isum[row * (a.K / 32) + u * 8 + b] = is[b];
        }
      }
    }
#pragma unroll
    for (int o = G / 2; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (row < rb && j == 0) {
      int seg;
      int64_t local;
      locate(a, row, seg, local);
      a.seg[seg].y[local] = acc;
    }
    __syncwarp();
    if (lane == 0 && k + S < mine) {
      fence_proxy_async_smem();
      const int64_t c2 = warp + (k + S) * W;
      const int64_t ra2 = r0 + c2 * RPC, rb2 = min(ra2 + RPC, r1);
      issue_rows(a, ra2, rb2, ring + static_cast<size_t>(slot) * a.slot_bytes, &bars[slot], policy);
    }
    if (++slot == S) {
      slot = 0;
      parity ^= 1u;
    }
  }
}

// Rows whose length is not a multiple of 16 bytes (Q8_0, K % 256 != 0): one
// warp per row, lanes over 34-byte blocks read with 16-bit loads.
template <bool ISUM>
__global__ void __launch_bounds__(256) gemv_q8_0_rowwise_kernel(const __grid_constant__ GemvArgs a) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t nb = a.K / 32;
  for (int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5); row < a.total_rows;
       row += static_cast<int64_t>(gridDim.x) * 8) {
    int seg;
    int64_t local;
    locate(a, row, seg, local);
    const int64_t group = local / a.group_rows;
    const uint8_t *rowp = a.seg[seg].w + local * a.row_bytes;
    float acc = 0.0f;
    for (int64_t b = lane; b < nb; b += 32) {
      const uint16_t *h = reinterpret_cast<const uint16_t *>(rowp + b * 34);
      const float dw = __half2float(__ushort_as_half(h[0]));
      const uint32_t *xq = reinterpret_cast<const uint32_t *>(a.xq + group * a.K + b * 32);
      int32_t s = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t qw = static_cast<uint32_t>(h[1 + 2 * i]) | (static_cast<uint32_t>(h[2 + 2 * i]) << 16);
        s = __dp4a(static_cast<int>(qw), static_cast<int>(__ldg(xq + i)), s);
      }
      if (ISUM) a.isum[row * nb + b] = s;
      acc += __fmul_rn(__fmul_rn(dw, __ldg(a.xd + group * nb + b)), static_cast<float>(s));
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) a.seg[seg].y[local] = acc;
  }
}

constexpr int kMaxWarps = DSQ_GEMV_MAX_WARPS;
constexpr size_t kSmemBudget = DSQ_GEMV_SMEM_KB * 1024;
// shared memory of an overlapped-launch CTA: two of them fit one SM
constexpr size_t kOverlapSmem = 110 * 1024;

// Shared memory of the activation area in fused mode: int8 codes plus fp32
// scales and int32 sums per 32-block.
size_t act_smem_bytes(int64_t rows, int64_t K) { return static_cast<size_t>(rows) * (K + 8 * (K / 32)); }

template <int TYPE, int G, bool ISUM, int ACT, int MAXW, int MINB>
int launch_fast(GemvArgs &a, int num_sms, cudaStream_t stream) {
  constexpr int RPC = 32 / G;
  size_t smem = static_cast<size_t>(a.warps) * a.stages * a.slot_bytes +
                static_cast<size_t>(a.warps) * a.stages * sizeof(uint64_t);
  if (ACT != kActGlobal) {
    smem = (smem + 15) / 16 * 16;
    a.act_off = static_cast<int>(smem);
    smem += act_smem_bytes(a.act_rows, a.K);
  }
  auto kern = gemv_kernel<TYPE, G, ISUM, ACT, MAXW, MINB>;
  const int rc = set_smem_once(reinterpret_cast<const void *>(kern), static_cast<int>(smem), "gemv");
  if (rc != DSQ_OK) return rc;
  const int64_t chunks = (a.total_rows + RPC - 1) / RPC;
  const int64_t slots = static_cast<int64_t>(num_sms) * DSQ_GEMV_CTAS_PER_SM;
  const unsigned grid = static_cast<unsigned>(chunks < slots ? chunks : slots);
  const cudaError_t e = launch_pdl(kern, dim3(grid), dim3(a.warps * 32), smem, stream, a);
  if (e != cudaSuccess) return fail(DSQ_ERR_LAUNCH, "gemv: %s", cudaGetErrorString(e));
  return after_launch("gemv");
}

template <int TYPE, bool ISUM, int ACT, int MAXW = DSQ_GEMV_MAX_WARPS, int MINB = DSQ_GEMV_CTAS_PER_SM>
int dispatch_g(GemvArgs &a, int G, int num_sms, cudaStream_t stream) {
  switch (G) {
    case 1: return launch_fast<TYPE, 1, ISUM, ACT, MAXW, MINB>(a, num_sms, stream);
    case 2: return launch_fast<TYPE, 2, ISUM, ACT, MAXW, MINB>(a, num_sms, stream);
    case 4: return launch_fast<TYPE, 4, ISUM, ACT, MAXW, MINB>(a, num_sms, stream);
    case 8: return launch_fast<TYPE, 8, ISUM, ACT, MAXW, MINB>(a, num_sms, stream);
    case 16: return launch_fast<TYPE, 16, ISUM, ACT, MAXW, MINB>(a, num_sms, stream);
    default: return launch_fast<TYPE, 32, ISUM, ACT, MAXW, MINB>(a, num_sms, stream);
  }
}

template <int TYPE, bool ISUM>
int dispatch_act(GemvArgs &a, int G, int act, int num_sms, cudaStream_t stream) {
  if (act == kActFused) return dispatch_g<TYPE, ISUM, kActFused>(a, G, num_sms, stream);
  if (act == kActStaged) return dispatch_g<TYPE, ISUM, kActStaged>(a, G, num_sms, stream);
  return dispatch_g<TYPE, ISUM, kActGlobal>(a, G, num_sms, stream);
}

// Largest activation area the fused mode keeps in shared memory (e.g. 8 rows
// of K = 4096, or one row of K = 49152).
constexpr size_t kMaxActSmem = 64 * 1024;

// Validates and launches one GEMV over up to two segments.  x32 != NULL
// selects the fused mode (fp32 activation rows quantized inside the kernel;
// xq/xd/xs unused).
int run_gemv(const char *name, int type, Seg s0, Seg s1, int64_t group_rows, int64_t groups, int64_t K,
             const int8_t *xq, const float *xd, const int32_t *xs, int32_t *isum, cudaStream_t stream,
             const float *x32 = nullptr) {
  DSQ_REQUIRE(type == DSQ_Q8_0 || type == DSQ_Q4_K, DSQ_ERR_INVALID_ARG, "%s: unsupported type %d", name, type);
  DSQ_REQUIRE(K > 0 && s0.rows >= 0 && s1.rows >= 0, DSQ_ERR_INVALID_ARG, "%s: negative size", name);
  const size_t rb = dsq_row_bytes(type, K);
  DSQ_REQUIRE(rb != 0, DSQ_ERR_SHAPE, "%s: K=%lld is not a multiple of %d", name, (long long)K,
              type == DSQ_Q8_0 ? 32 : 256);
  DSQ_REQUIRE(K <= (int64_t(1) << 20) && s0.rows + s1.rows <= (int64_t(1) << 31), DSQ_ERR_SHAPE,
              "%s: size out of range (K <= 2^20, rows <= 2^31)", name);
  const int64_t total = s0.rows + s1.rows;
  if (total == 0) return DSQ_OK;
  if (x32) {
    DSQ_REQUIRE(aligned(x32, 16), DSQ_ERR_ALIGNMENT, "%s: x must be 16-byte aligned", name);
    DSQ_REQUIRE(rb % 16 == 0, DSQ_ERR_SHAPE, "%s: K=%lld: the fused form needs K %% 256 == 0", name, (long long)K);
    DSQ_REQUIRE(act_smem_bytes(groups, K) <= kMaxActSmem, DSQ_ERR_SHAPE,
                "%s: %lld activation rows of K=%lld exceed the fused form's %zu bytes of shared memory", name,
                (long long)groups, (long long)K, kMaxActSmem);
  } else {
    DSQ_REQUIRE(xq && xd && (type == DSQ_Q8_0 || xs), DSQ_ERR_INVALID_ARG, "%s: null activation pointer", name);
  }
  DSQ_REQUIRE((s0.rows == 0 || (s0.w && s0.y)) && (s1.rows == 0 || (s1.w && s1.y)), DSQ_ERR_INVALID_ARG,
              "%s: null weight/output pointer", name);
  DSQ_REQUIRE(x32 || (aligned(xq, 16) && aligned(xd, 16) && (!xs || aligned(xs, 16))), DSQ_ERR_ALIGNMENT,
              "%s: xq/xd/xs must be 16-byte aligned", name);
  DSQ_REQUIRE((s0.rows == 0 || (aligned(s0.w, 16) && aligned(s0.y, 4))) &&
                  (s1.rows == 0 || (aligned(s1.w, 16) && aligned(s1.y, 4))),
              DSQ_ERR_ALIGNMENT, "%s: weights must be 16-byte and outputs 4-byte aligned", name);
  WaitCtl ctl;
  int num_sms = 0;
  int rc = wait_ctl(&ctl, &num_sms);
  if (rc != DSQ_OK) return rc;

  GemvArgs a{};
  a.seg[0] = s0;
  a.seg[1] = s1;
  a.rows0 = s0.rows;
  a.total_rows = total;
  a.group_rows = group_rows;
  a.xq = xq;
  a.xd = xd;
  a.xs = xs;
  a.K = K;
  a.row_bytes = static_cast<int64_t>(rb);
  a.wait = ctl;
  a.isum = isum;
  a.x32 = x32;
  a.act_rows = groups;

  // Mid-length single matrices on one token: the multi-token kernel (one CTA
  // per 32-row group, warps over 256-element units, bit-identical outputs)
  // is faster while its row groups fill at most one wave of SMs.
  // Interleaved A/B on B200, K = 4096, this kernel against it: Q4_K 2048 /
  // 3072 / 4096 rows 3.57 / 4.53 / 4.67 against 3.49 / 3.92 / 4.14 us, Q8_0
  // 2048 / 4096 rows 3.81 / 6.21 against 3.65 / 4.99 us; past one wave
  // (Q4_K 5120 rows) 5.47 against 5.82 us.
  // (K <= 32768 keeps one token's activation inside that kernel's 64 KB area.)
  if (s1.rows == 0 && groups == 1 && !isum && !x32 && K % 256 == 0 && K <= 32768 && total >= DSQ_GEMV_TOK_MIN_ROWS &&
      (total + 31) / 32 <= num_sms)
    return gemv_one_token(name, type, s0.w, s0.rows, K, xq, xd, xs, s0.y, stream);
  if (rb % 16 != 0) {  // Q8_0 with K % 256 != 0
    const int64_t blocks = (total + 7) / 8;
    const unsigned grid = static_cast<unsigned>(blocks < 4 * num_sms ? blocks : 4 * num_sms);
    const cudaError_t e = isum ? launch_pdl(gemv_q8_0_rowwise_kernel<true>, dim3(grid), dim3(256), 0, stream, a)
                               : launch_pdl(gemv_q8_0_rowwise_kernel<false>, dim3(grid), dim3(256), 0, stream, a);
    if (e != cudaSuccess) return fail(DSQ_ERR_LAUNCH, "%s: %s", name, cudaGetErrorString(e));
    return after_launch(name);
  }
  a.nunits = static_cast<int>(K / 256);
  int G = 1;
  while (G < a.nunits && G < 32) G <<= 1;
  a.slot_bytes = static_cast<int>((32 / G) * rb);
  // the grouped form copies its CTA's activation groups into shared memory
  // when they fit; the ring gets the shared memory the activation area leaves
  const int act = x32 ? kActFused : (groups > 1 && act_smem_bytes(groups, K) <= kMaxActSmem ? kActStaged : kActGlobal);
  const size_t budget = kSmemBudget - (act != kActGlobal ? act_smem_bytes(groups, K) + 16 : 0);
  a.warps = kMaxWarps;
  while (a.warps > 1 && static_cast<size_t>(a.warps) * 2 * a.slot_bytes > budget) a.warps >>= 1;
  DSQ_REQUIRE(static_cast<size_t>(a.warps) * 2 * a.slot_bytes <= budget, DSQ_ERR_SHAPE,
              "%s: K=%lld rows do not fit the shared-memory pipeline", name, (long long)K);
  a.stages = static_cast<int>(budget / (static_cast<size_t>(a.warps) * a.slot_bytes));
  if (a.stages > DSQ_GEMV_MAX_STAGES) a.stages = DSQ_GEMV_MAX_STAGES;
  // A long Q4_K matrix is bound by how much unpacking is in flight, not by
  // its loads (a deeper ring measured slower): more warps, each with the
  // same 2-slot ring.  Shorter matrices keep 8 warps, which start faster.
  // Interleaved A/B on B200, K = 4096, rows per CTA in brackets, 8 / 12 / 16
  // warps: 16,384 rows (110) 10.1 / 10.6 / 11.8 us; 24,576 (166) 13.3 /
  // 12.8 / 14.0; 32,768 (221) 16.7 / 15.5 / 16.1; 65,536 (443) 29.7 / 26.7 /
  // 26.2-26.6.
  if (type == DSQ_Q4_K && act == kActGlobal && !isum && a.warps == kMaxWarps) {
    const int64_t per_cta = total / (static_cast<int64_t>(num_sms) * DSQ_GEMV_CTAS_PER_SM);
    if (per_cta >= DSQ_GEMV_WIDE_MIN_ROWS && size_t(16) * 2 * a.slot_bytes <= budget) {
      a.warps = 16;
      a.stages = 2;
      return dispatch_g<DSQ_Q4_K, false, kActGlobal, 16>(a, G, num_sms, stream);
    }
    if (per_cta >= DSQ_GEMV_MID_MIN_ROWS && size_t(12) * 2 * a.slot_bytes <= budget) {
      a.warps = 12;
      a.stages = 2;
      return dispatch_g<DSQ_Q4_K, false, kActGlobal, 12>(a, G, num_sms, stream);
    }
    // Shorter Q4_K matrices: the overlapped launch, when 8 warps with 2 slots
    // each fit half an SM's shared memory (Q4_K slots are 4.6 KB at K = 4096).
    // The next call's first weight slots then load while this call drains
    // (interleaved A/B on B200: 4096 x 4096 5.57 -> 4.67 us, 16,384 x 4096
    // 10.0 -> 9.5 us).  Q8_0's 8.7 KB slots would need fewer warps, which
    // cost more than the overlap gives (8192 x 4096: 8.0 -> 8.7 us).
    if (a.stages == 2 && size_t(kMaxWarps) * 2 * (a.slot_bytes + sizeof(uint64_t)) <= kOverlapSmem)
      return dispatch_g<DSQ_Q4_K, false, kActGlobal, DSQ_GEMV_MAX_WARPS, 2>(a, G, num_sms, stream);
  }
  // Short Q8_0 matrices whose CTAs hold at most two slots per warp even with
  // the fewer warps that fit half an SM take the overlapped launch too
  // (1024 x 1024: 2.09 -> 1.98 us, interleaved A/B on B200).
  if (type == DSQ_Q8_0 && act == kActGlobal && !isum && a.stages == 2) {
    const int64_t chunks = (total + (32 / G) - 1) / (32 / G);
    const int64_t slots = static_cast<int64_t>(num_sms) * DSQ_GEMV_CTAS_PER_SM;
    const int64_t per_cta_chunks = (chunks + (chunks < slots ? chunks : slots) - 1) / (chunks < slots ? chunks : slots);
    int64_t w_fit = static_cast<int64_t>(kOverlapSmem / (2 * (static_cast<size_t>(a.slot_bytes) + sizeof(uint64_t))));
    if (w_fit > kMaxWarps) w_fit = kMaxWarps;
    if (w_fit >= 1 && per_cta_chunks <= 2 * w_fit) {
      a.warps = static_cast<int>(w_fit);
      return dispatch_g<DSQ_Q8_0, false, kActGlobal, DSQ_GEMV_MAX_WARPS, 2>(a, G, num_sms, stream);
    }
  }
  if (type == DSQ_Q8_0)
    return isum ? dispatch_act<DSQ_Q8_0, true>(a, G, act, num_sms, stream)
                : dispatch_act<DSQ_Q8_0, false>(a, G, act, num_sms, stream);
  return isum ? dispatch_act<DSQ_Q4_K, true>(a, G, act, num_sms, stream)
              : dispatch_act<DSQ_Q4_K, false>(a, G, act, num_sms, stream);
}

constexpr int64_t kOneGroup = int64_t(1) << 62;

}  // namespace
}  // namespace dsq

extern "C" {

int dsq_gemv_q8_0(const void *w, int64_t N, int64_t K, const int8_t *xq, const float *xd, float *y, void *stream) {
  using namespace dsq;
  return run_gemv("dsq_gemv_q8_0", DSQ_Q8_0, Seg{static_cast<const uint8_t *>(w), y, N}, Seg{nullptr, nullptr, 0},
                  kOneGroup, 1, K, xq, xd, nullptr, nullptr, as_stream(stream));
}

int dsq_gemv_q4_k(const void *w, int64_t N, int64_t K, const int8_t *xq, const float *xd, const int32_t *xs,
                  float *y, void *stream) {
  using namespace dsq;
  return run_gemv("dsq_gemv_q4_k", DSQ_Q4_K, Seg{static_cast<const uint8_t *>(w), y, N}, Seg{nullptr, nullptr, 0},
                  kOneGroup, 1, K, xq, xd, xs, nullptr, as_stream(stream));
}

int dsq_gemv_paired(int type, const void *w0, int64_t N0, const void *w1, int64_t N1, int64_t K, const int8_t *xq,
                    const float *xd, const int32_t *xs, float *y0, float *y1, void *stream) {
  using namespace dsq;
  return run_gemv("dsq_gemv_paired", type, Seg{static_cast<const uint8_t *>(w0), y0, N0},
                  Seg{static_cast<const uint8_t *>(w1), y1, N1}, kOneGroup, 1, K, xq, xd, xs, nullptr,
                  as_stream(stream));
}

int dsq_gemv_grouped(int type, const void *w, int64_t G, int64_t N, int64_t K, const int8_t *xq, const float *xd,
                     const int32_t *xs, float *y, void *stream) {
  using namespace dsq;
  DSQ_REQUIRE(G >= 0 && N >= 0, DSQ_ERR_INVALID_ARG, "dsq_gemv_grouped: G=%lld N=%lld", (long long)G, (long long)N);
  DSQ_REQUIRE(G <= (int64_t(1) << 20), DSQ_ERR_SHAPE, "dsq_gemv_grouped: G out of range");
  if (G == 0 || N == 0) return dsq::run_gemv("dsq_gemv_grouped", type, Seg{nullptr, nullptr, 0}, Seg{nullptr, nullptr, 0},
                                             1, 0, K, xq, xd, xs, nullptr, as_stream(stream));
  return run_gemv("dsq_gemv_grouped", type, Seg{static_cast<const uint8_t *>(w), y, G * N}, Seg{nullptr, nullptr, 0}, N,
                  G, K, xq, xd, xs, nullptr, as_stream(stream));
}

int dsq_gemv_f32(int type, const void *w, int64_t N, int64_t K, const float *x, float *y, void *stream) {
  using namespace dsq;
  return run_gemv("dsq_gemv_f32", type, Seg{static_cast<const uint8_t *>(w), y, N}, Seg{nullptr, nullptr, 0},
                  kOneGroup, 1, K, nullptr, nullptr, nullptr, nullptr, as_stream(stream), x);
}

int dsq_gemv_paired_f32(int type, const void *w0, int64_t N0, const void *w1, int64_t N1, int64_t K, const float *x,
                        float *y0, float *y1, void *stream) {
  using namespace dsq;
  return run_gemv("dsq_gemv_paired_f32", type, Seg{static_cast<const uint8_t *>(w0), y0, N0},
                  Seg{static_cast<const uint8_t *>(w1), y1, N1}, kOneGroup, 1, K, nullptr, nullptr, nullptr, nullptr,
                  as_stream(stream), x);
}

int dsq_gemv_grouped_f32(int type, const void *w, int64_t G, int64_t N, int64_t K, const float *x, float *y,
                         void *stream) {
  using namespace dsq;
  DSQ_REQUIRE(G >= 0 && N >= 0, DSQ_ERR_INVALID_ARG, "dsq_gemv_grouped_f32: G=%lld N=%lld", (long long)G,
              (long long)N);
  DSQ_REQUIRE(G <= (int64_t(1) << 20), DSQ_ERR_SHAPE, "dsq_gemv_grouped_f32: G out of range");
  if (G == 0 || N == 0)
    return run_gemv("dsq_gemv_grouped_f32", type, Seg{nullptr, nullptr, 0}, Seg{nullptr, nullptr, 0}, 1, 0, K,
                    nullptr, nullptr, nullptr, nullptr, as_stream(stream), x);
  return run_gemv("dsq_gemv_grouped_f32", type, Seg{static_cast<const uint8_t *>(w), y, G * N},
                  Seg{nullptr, nullptr, 0}, N, G, K, nullptr, nullptr, nullptr, nullptr, as_stream(stream), x);
}

int dsq_test_block_sums(int type, const void *w, int64_t N, int64_t K, const int8_t *xq, const float *xd,
                        const int32_t *xs, float *y, int32_t *isum, void *stream) {
  using namespace dsq;
  DSQ_REQUIRE(isum != nullptr || N == 0, DSQ_ERR_INVALID_ARG, "dsq_test_block_sums: null isum");
  DSQ_REQUIRE(aligned(isum, 4), DSQ_ERR_ALIGNMENT, "dsq_test_block_sums: isum alignment");
  return run_gemv("dsq_test_block_sums", type, Seg{static_cast<const uint8_t *>(w), y, N}, Seg{nullptr, nullptr, 0},
                  kOneGroup, 1, K, xq, xd, xs, isum, as_stream(stream));
}

}  // extern "C"
