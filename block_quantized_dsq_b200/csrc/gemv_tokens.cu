// gemv_tokens.cu -- multi-token decode GEMV: M = 1..8 prequantized activation
// rows against one block-quantized weight, or against two weights that share
// the same input (the paired Q / KV projections), reading every weight byte
// once for all M tokens.
//
// Sources: "Support AProjQ4 GGUFs: Q4_K dense attention projections"
// (antirez/ds4 PR #621), GB10 test report: short multi-token batches of up to
// 8 tokens (the grouped-tok8 and QKV-pair decode paths) are worth a path of
// their own only if they keep decode consistent and cost nothing; "ROCm:
// restore DeepSeek V4 Flash decode performance" (antirez/ds4 PR #623),
// Summary: the activation is prequantized to Q8 once and shared by the
// projections that read it.
//
// Numerics: each token's output equals, bit for bit, what the single-token
// entry points (dsq_gemv_q8_0 / dsq_gemv_q4_k / dsq_gemv_paired) give for that
// token alone.  The block terms, the per-unit partial sums and the order in
// which they are added are the single-token kernel's, so decoding M tokens
// in one call is indistinguishable from M decode steps.
//
// B200 design (HBM-bound weight stream, M tokens per weight byte):
//  * lane = weight row.  A warp handles a group of 32 consecutive rows of one
//    weight, one 256-element unit at a time: the unit arrives as one 2-D TMA
//    box (32 rows x 272 B for Q8_0, x 144 B for Q4_K) in the warp's ring of
//    shared-memory slots.
//  * All 32 lanes read the same activation bytes at the same moment, so the
//    M tokens' codes and scales come out of shared memory as broadcasts:
//    per unit and token, 20 16-byte reads for the whole warp.
//  * A row is split into units the way the single-token kernel splits it
//    across the lanes of a row: virtual lane j (j < G, G = units per row
//    rounded up to a power of two, at most 32) owns units j, j+G, ...  The
//    CTA's warps take virtual lanes j = warp + W*i.  Each virtual lane keeps
//    its partial sum per token; the partials meet in the single-token
//    kernel's butterfly order -- inside the warp for the strides >= W, then
//    across warps through shared memory.
//  * Persistent CTAs (one per SM) step through the row groups of both
//    weights; weights are read once, activations stay in shared memory.
#include <cudaTypedefs.h>

#include "../../include/dsq_test.h"
#include "dsq_host.h"

namespace dsq {
namespace {

constexpr int kTokMaxM = 8;
constexpr int kTokWarps = 8;          // warps per CTA
constexpr int kTokRows = 32;          // rows per group (lane = row)
constexpr int kTokMaxStages = 4;      // ring slots per warp
constexpr size_t kTokSmemLimit = 227 * 1024;
constexpr size_t kTokMaxActSmem = 64 * 1024;

template <int TYPE> __host__ __device__ constexpr int tok_unit_bytes() { return TYPE == DSQ_Q8_0 ? 272 : 144; }

struct TokArgs {
  float *y[2];            // outputs [M][n[s]] of each weight
  int64_t n[2];           // rows of each weight
  int64_t groups0;        // 32-row groups of weight 0 (weight 1's follow)
  int64_t total_groups;
  int64_t K;
  int nunits;             // K / 256
  int G;                  // virtual lanes per row (power of two, <= 32)
  int W;                  // warps with virtual lanes: min(8, G)
  int stages;             // ring slots per warp
  uint32_t box_bytes;     // one TMA box: 32 rows x one unit
  uint32_t q_bytes, d_bytes, s_bytes;   // activation areas in shared memory
  uint32_t ring_off, bar_off, red_off;  // shared-memory offsets
  uint32_t sc_off;        // tensor-core form, Q4_K: per-warp scale scratch
  const int8_t *xq;       // [M][K]
  const float *xd;        // [M][K/32]
  const int32_t *xs;      // [M][K/32] (Q4_K)
  int32_t *isum;          // test hook: [M][n0 + n1][K/32] block sums, or NULL
  WaitCtl wait;
};

__device__ __forceinline__ float tok_half_lo(uint32_t w) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(w & 0xffffu)));
}
__device__ __forceinline__ float tok_half_hi(uint32_t w) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(w >> 16)));
}

// One Q8_0 unit (8 blocks, 272 bytes at p) of this lane's row against unit u
// of the M tokens.  Block b starts at byte 34b: even b has its scale in the
// low half of word 17b/2 and its codes two bytes later (realigned with a
// funnel shift), odd b its scale in the high half of word (17b-1)/2 and its
// codes word-aligned.  part[m] = sum over the 8 blocks, in block order from
// 0, of (d_w * xd) * isum: the single-token kernel's unit partial.
template <int M>
__device__ __forceinline__ void tok_unit_q8_0(const uint8_t *p, const int8_t *sq, const float *sd, int64_t K, int u,
                                              float (&part)[M], int32_t *isum, int64_t isum_tok_stride) {
  uint32_t w[68];
  const uint4 *p4 = reinterpret_cast<const uint4 *>(p);
#pragma unroll
  for (int i = 0; i < 17; ++i) {
    const uint4 v = p4[i];
    w[4 * i + 0] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
  }
#pragma unroll
  for (int m = 0; m < M; ++m) part[m] = 0.0f;
  const int64_t nb = K / 32;
#pragma unroll
  for (int b = 0; b < 8; ++b) {
    uint32_t c[8];
    float dw;
    if ((b & 1) == 0) {
      const int a0 = 17 * b / 2;
      dw = tok_half_lo(w[a0]);
#pragma unroll
      for (int i = 0; i < 8; ++i) c[i] = __funnelshift_r(w[a0 + i], w[a0 + i + 1], 16);
    } else {
      const int a0 = (17 * b - 1) / 2;
      dw = tok_half_hi(w[a0]);
#pragma unroll
      for (int i = 0; i < 8; ++i) c[i] = w[a0 + 1 + i];
    }
#pragma unroll
    for (int m = 0; m < M; ++m) {
      const uint4 *x4 = reinterpret_cast<const uint4 *>(sq + m * K + u * 256 + b * 32);
      const uint4 x0 = x4[0], x1 = x4[1];
      int32_t s = 0;
      s = __dp4a(static_cast<int>(c[0]), static_cast<int>(x0.x), s);
      s = __dp4a(static_cast<int>(c[1]), static_cast<int>(x0.y), s);
      s = __dp4a(static_cast<int>(c[2]), static_cast<int>(x0.z), s);
      s = __dp4a(static_cast<int>(c[3]), static_cast<int>(x0.w), s);
      s = __dp4a(static_cast<int>(c[4]), static_cast<int>(x1.x), s);
      s = __dp4a(static_cast<int>(c[5]), static_cast<int>(x1.y), s);
      s = __dp4a(static_cast<int>(c[6]), static_cast<int>(x1.z), s);
      s = __dp4a(static_cast<int>(c[7]), static_cast<int>(x1.w), s);
      if (isum) isum[m * isum_tok_stride + u * 8 + b] = s;
      part[m] += __fmul_rn(__fmul_rn(dw, sd[m * nb + u * 8 + b]), static_cast<float>(s));
    }
  }
}

// One Q4_K super-block (144 bytes at p: word 0 = d | dmin << 16, words 1..3
// the packed 6-bit scales and mins, words 4..35 the nibbles) against unit u of
// the M tokens: part[m] = sum over sub-blocks j, in order from 0, of
// xd * ((d*sc_j)*isum_j - (dmin*m_j)*xs_j).
template <int M>
__device__ __forceinline__ void tok_unit_q4_k(const uint8_t *p, const int8_t *sq, const float *sd,
                                              const int32_t *ss, int64_t K, int u, float (&part)[M],
                                              int32_t *isum, int64_t isum_tok_stride) {
  uint32_t w[36];
  const uint4 *p4 = reinterpret_cast<const uint4 *>(p);
#pragma unroll
  for (int i = 0; i < 9; ++i) {
    const uint4 v = p4[i];
    w[4 * i + 0] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
  }
  const float d = tok_half_lo(w[0]), dmin = tok_half_hi(w[0]);
  const uint32_t s0 = w[1], s1 = w[2], s2 = w[3];
  const uint32_t scA = s0 & 0x3f3f3f3fu;
  const uint32_t mA = s1 & 0x3f3f3f3fu;
  const uint32_t scB = (s2 & 0x0f0f0f0fu) | ((s0 >> 2) & 0x30303030u);
  const uint32_t mB = ((s2 >> 4) & 0x0f0f0f0fu) | ((s1 >> 2) & 0x30303030u);
#pragma unroll
  for (int m = 0; m < M; ++m) part[m] = 0.0f;
  const int64_t nb = K / 32;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint32_t scw = j < 4 ? scA : scB, mw = j < 4 ? mA : mB;
    const int sh = 8 * (j & 3);
    const float dsc = __fmul_rn(d, static_cast<float>((scw >> sh) & 0xffu));
    const float dmm = __fmul_rn(dmin, static_cast<float>((mw >> sh) & 0xffu));
    uint32_t c[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t byte4 = w[4 + 8 * (j >> 1) + i];
      c[i] = (j & 1) ? ((byte4 >> 4) & 0x0f0f0f0fu) : (byte4 & 0x0f0f0f0fu);
    }
#pragma unroll
    for (int m = 0; m < M; ++m) {
      const uint4 *x4 = reinterpret_cast<const uint4 *>(sq + m * K + u * 256 + j * 32);
      const uint4 x0 = x4[0], x1 = x4[1];
      int32_t s = 0;
      s = __dp4a(static_cast<int>(c[0]), static_cast<int>(x0.x), s);
      s = __dp4a(static_cast<int>(c[1]), static_cast<int>(x0.y), s);
      s = __dp4a(static_cast<int>(c[2]), static_cast<int>(x0.z), s);
      s = __dp4a(static_cast<int>(c[3]), static_cast<int>(x0.w), s);
      s = __dp4a(static_cast<int>(c[4]), static_cast<int>(x1.x), s);
      s = __dp4a(static_cast<int>(c[5]), static_cast<int>(x1.y), s);
      s = __dp4a(static_cast<int>(c[6]), static_cast<int>(x1.z), s);
      s = __dp4a(static_cast<int>(c[7]), static_cast<int>(x1.w), s);
      if (isum) isum[m * isum_tok_stride + u * 8 + j] = s;
      const int64_t bi = m * nb + u * 8 + j;
      const float t = __fmul_rn(dsc, static_cast<float>(s));
      const float v = __fmul_rn(dmm, static_cast<float>(ss[bi]));
      part[m] += __fmul_rn(sd[bi], __fsub_rn(t, v));
    }
  }
}

// Position of a warp's work: row group g, virtual-lane slot i (virtual lane
// v = warp + W*i), unit u (v, v+G, ...).  next() steps in consumption order.
struct TokCursor {
  int64_t g;
  int i, u;
  __device__ __forceinline__ void first(const TokArgs &a, int warp, int vpw) {
    g = blockIdx.x;
    i = 0;
    u = warp;
    if (vpw == 0 || u >= a.nunits) g = a.total_groups;   // this warp has no units
  }
  __device__ __forceinline__ void next(const TokArgs &a, int warp, int vpw) {
    u += a.G;
    if (u >= a.nunits) {
      ++i;
      u = warp + a.W * i;
      if (i >= vpw || u >= a.nunits) {
        g += gridDim.x;
        i = 0;
        u = warp;
      }
    }
  }
  __device__ __forceinline__ bool valid(const TokArgs &a) const { return g < a.total_groups; }
};

template <int UB>
__device__ __forceinline__ void tok_issue(const CUtensorMap *map0, const CUtensorMap *map1, const TokArgs &a,
                                          const TokCursor &c, uint8_t *dst, uint64_t *bar) {
  const bool second = c.g >= a.groups0;
  const int32_t row0 = static_cast<int32_t>((second ? c.g - a.groups0 : c.g) * kTokRows);
  mbar_arrive_expect_tx(bar, a.box_bytes);
  tma_load_2d(dst, second ? map1 : map0, c.u * (UB / 4), row0, bar);
}

template <int TYPE, int M>
__global__ void __launch_bounds__(kTokWarps * 32, 1)
    gemv_tokens_kernel(const __grid_constant__ CUtensorMap map0, const __grid_constant__ CUtensorMap map1,
                       const __grid_constant__ TokArgs a) {
  constexpr int UB = tok_unit_bytes<TYPE>();
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int W = a.W, S = a.stages;
  const int vpw = warp < W ? a.G / W : 0;   // virtual lanes of this warp
  const int8_t *sq = reinterpret_cast<const int8_t *>(base);
  const float *sd = reinterpret_cast<const float *>(base + a.q_bytes);
  const int32_t *ss = reinterpret_cast<const int32_t *>(base + a.q_bytes + a.d_bytes);
  uint8_t *ring = base + a.ring_off + static_cast<size_t>(warp) * S * a.box_bytes;
  uint64_t *act_bar = reinterpret_cast<uint64_t *>(base + a.bar_off);
  uint64_t *bars = act_bar + 1 + warp * kTokMaxStages;
  float *red = reinterpret_cast<float *>(base + a.red_off);   // [2][8 warps][M][32 rows]
  volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(act_bar + 1 + kTokWarps * kTokMaxStages);

  if (threadIdx.x == 0) {
    mbar_init(act_bar, 1);
    *abort_flag = 0u;
    prefetch_tensormap(&map0);
    prefetch_tensormap(&map1);
  }
  if (lane == 0)
    for (int s = 0; s < S; ++s) mbar_init(&bars[s], 1);
  fence_barrier_init();
  // weights are read-only: bring this warp's first boxes toward L2 while the
  // kernel before us (usually the activation quantizer) finishes
  TokCursor issue;
  issue.first(a, warp, vpw);
  if (lane == 0) {
    TokCursor c = issue;
    for (int s = 0; s < S && c.valid(a); ++s, c.next(a, warp, vpw)) {
      const bool second = c.g >= a.groups0;
      prefetch_l2_tile_2d(second ? &map1 : &map0, c.u * (UB / 4),
                          static_cast<int32_t>((second ? c.g - a.groups0 : c.g) * kTokRows));
    }
  }
  __syncthreads();
  pdl_trigger();
  pdl_wait();

  if (threadIdx.x == 0) {
    // the M tokens' prequantized activations, once, into shared memory
    const uint64_t keep = l2_policy_evict_last();
    mbar_arrive_expect_tx(act_bar, a.q_bytes + a.d_bytes + a.s_bytes);
    bulk_g2s(base, a.xq, a.q_bytes, act_bar, keep);
    bulk_g2s(base + a.q_bytes, a.xd, a.d_bytes, act_bar, keep);
    if (a.s_bytes) bulk_g2s(base + a.q_bytes + a.d_bytes, a.xs, a.s_bytes, act_bar, keep);
  }
  int64_t n_issued = 0, n_waited = 0;
  if (lane == 0) {
    for (int s = 0; s < S && issue.valid(a); ++s, issue.next(a, warp, vpw), ++n_issued)
      tok_issue<UB>(&map0, &map1, a, issue, ring + static_cast<size_t>(s) * a.box_bytes, &bars[s]);
  }
  bool ok = __all_sync(0xffffffffu, mbar_wait_for(act_bar, 0, a.wait.limit_ns));
  if (!ok && lane == 0) {
    *abort_flag = 1u;
    record_timeout(a.wait);
  }

  int slot = 0;
  uint32_t parity = 0;
  int buf = 0;
  const int64_t nb = a.K / 32;
  const int64_t rows_total = a.n[0] + a.n[1];
  for (int64_t g = blockIdx.x; g < a.total_groups; g += gridDim.x, buf ^= 1) {
    const bool second = g >= a.groups0;
    const int64_t rloc = (second ? g - a.groups0 : g) * kTokRows + lane;   // this lane's row in its weight
    const int64_t vrow = (second ? a.n[0] : 0) + rloc;                   // in [weight 0 rows, weight 1 rows]
    float acc[4][M];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int m = 0; m < M; ++m) acc[i][m] = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (i >= vpw) break;
      for (int u = warp + W * i; u < a.nunits; u += a.G) {
        ok = ok && *abort_flag == 0u;
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait_for(&bars[slot], parity, a.wait.limit_ns));
        if (!ok) {
          if (lane == 0 && *abort_flag == 0u) {
            *abort_flag = 1u;
            record_timeout(a.wait);
          }
        } else {
          ++n_waited;
          float part[M];
          const uint8_t *rowp = ring + static_cast<size_t>(slot) * a.box_bytes + static_cast<size_t>(lane) * UB;
          int32_t *isum = (a.isum && rloc < a.n[second ? 1 : 0]) ? a.isum + vrow * nb : nullptr;
          if constexpr (TYPE == DSQ_Q8_0)
            tok_unit_q8_0<M>(rowp, sq, sd, a.K, u, part, isum, rows_total * nb);
          else
            tok_unit_q4_k<M>(rowp, sq, sd, ss, a.K, u, part, isum, rows_total * nb);
#pragma unroll
          for (int m = 0; m < M; ++m) acc[i][m] += part[m];
          __syncwarp();
          if (lane == 0 && issue.valid(a)) {
            fence_proxy_async_smem();
            tok_issue<UB>(&map0, &map1, a, issue, ring + static_cast<size_t>(slot) * a.box_bytes, &bars[slot]);
            issue.next(a, warp, vpw);
            ++n_issued;
          }
        }
        if (++slot == S) {
          slot = 0;
          parity ^= 1u;
        }
      }
    }
    // butterfly strides >= W stay inside the warp: virtual lane j = warp + W*i
    // meets j ^ (W * st) = warp + W * (i ^ st)
    float mine[M];
#pragma unroll
    for (int m = 0; m < M; ++m) {
      if (vpw == 4) mine[m] = (acc[0][m] + acc[2][m]) + (acc[1][m] + acc[3][m]);
      else if (vpw == 2) mine[m] = acc[0][m] + acc[1][m];
      else mine[m] = acc[0][m];
    }
    float *rb = red + static_cast<size_t>(buf) * kTokWarps * M * 32;
#pragma unroll
    for (int m = 0; m < M; ++m) rb[(warp * M + m) * 32 + lane] = mine[m];
    __syncthreads();
    // strides < W cross warps: ((r0+r4)+(r2+r6)) + ((r1+r5)+(r3+r7)) for W = 8
    for (int m = warp; m < M; m += kTokWarps) {
      float r[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) r[k] = k < W ? rb[(k * M + m) * 32 + lane] : 0.0f;
      float v;
      if (W == 8) v = ((r[0] + r[4]) + (r[2] + r[6])) + ((r[1] + r[5]) + (r[3] + r[7]));
      else if (W == 4) v = (r[0] + r[2]) + (r[1] + r[3]);
      else if (W == 2) v = r[0] + r[1];
      else v = r[0];
      const int sgi = second ? 1 : 0;
      if (rloc < a.n[sgi] && *abort_flag == 0u) a.y[sgi][m * a.n[sgi] + rloc] = v;
    }
  }
  // after an abort: let this warp's copies still in flight land before exit
  if (lane == 0) {
    for (int64_t k = n_waited; k < n_issued; ++k)
      mbar_wait_for(&bars[k % S], static_cast<uint32_t>((k / S) & 1), kDrainLimitNs);
  }
  if (threadIdx.x == 0 && !ok) mbar_wait_for(act_bar, 0, kDrainLimitNs);
}

// ------------------------------------------------------- 4 to 8 tokens ---
// From 4 (Q8_0) or 5 (Q4_K) tokens on, the block dots run on the tensor cores: one
// mma.sync.m16n8k32 (int8 x int8 -> int32) gives the exact block sums of one
// 32-element block for 16 weight rows x 8 tokens.  Integer sums are exact
// whoever forms them, and the lanes then form each fp32 block term and add
// it in the single-token kernel's order, so every output stays bit-identical
// to the single-token entry points; only the lane that computes a term
// changes.  Per block a warp issues two MMAs (rows 0..15, 16..31) where the
// CUDA-core form issues 64 dp4a per lane, and no lane holds a whole row.
//
// Fragments of m16n8k32 (lane = 4 grp + t): A rows grp and grp + 8, codes
// 4t..4t+3 and 16+4t..16+4t+3 of the block; B token grp, the same codes; D
// rows grp and grp + 8, tokens 2t and 2t + 1.
//
// Activations in shared memory (tokens padded to 8 with zeros):
//   codes as 32-bit words [unit][block][chunk kc][token] -- lane (grp, t)
//   reads chunk t (and t + 4) of token grp: 32 consecutive words;
//   scales and sums as [unit * 8 + block][token] -- lane reads tokens 2t, 2t+1.
// The tensor-core form does the work of 8 tokens whatever M is, so it pays
// only from a type-dependent token count on (interleaved A/B on one B200:
// paired 2 x 8192 x 4096 Q8_0 takes 18.6 us at any M against 15.8 / 20.3 /
// 26.7 / 33.9 us for 2 / 4 / 6 / 8 tokens on the CUDA cores; Q4_K 4096 x 4096
// 7.3 us against 7.0 / 8.7 / 10.4 us for 4 / 6 / 8 tokens).
constexpr int kTokMmaMinM = 4;   // the smallest count any type takes it at
__host__ __device__ constexpr int tok_mma_min_m(int type) { return type == DSQ_Q8_0 ? 4 : 5; }
constexpr int kTokScStride = 18;   // words per row of the Q4_K scale scratch (8 pairs + pad)

__device__ __forceinline__ void mma_s8_m16n8k32(int32_t (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                                uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t lds32(const uint8_t *p) { return *reinterpret_cast<const uint32_t *>(p); }

// Value v of a lane's 8 (row, token) terms: m-tile mt = v / 4, row half h =
// (v / 2) % 2, token e = v % 2 -> row grp + 8h + 16mt, token 2t + e.
__device__ __forceinline__ int mma_row(int v, int grp) { return grp + 8 * ((v >> 1) & 1) + 16 * (v >> 2); }
__device__ __forceinline__ int mma_tok(int v, int t) { return 2 * t + (v & 1); }

// One Q8_0 unit of the warp's 32-row box against unit u of the tokens:
// part[v] = sum over the 8 blocks, in order, of (d_w * xd) * isum.
template <int M, bool ISUM>
__device__ __forceinline__ void tok_mma_q8_0(const uint8_t *box, const uint32_t *qt, const float *dt, int u,
                                             int lane, float (&part)[8], int32_t *isum, int64_t isum_row,
                                             int64_t isum_tok, int64_t rows_left) {
  const int grp = lane >> 2, t = lane & 3;
#pragma unroll
  for (int v = 0; v < 8; ++v) part[v] = 0.0f;
#pragma unroll
  for (int b = 0; b < 8; ++b) {
    uint32_t A[2][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
          const uint8_t *p = box + (grp + 8 * h + 16 * mt) * 272 + 34 * b + 2 + 4 * t + 16 * kk;
          // codes of even blocks sit 2 bytes past a word boundary
          A[mt][h + 2 * kk] = (b & 1) ? lds32(p) : __funnelshift_r(lds32(p - 2), lds32(p + 2), 16);
        }
    const uint32_t *q = qt + (u * 8 + b) * 64;
    const uint32_t b0 = q[t * 8 + grp], b1 = q[(t + 4) * 8 + grp];
    int32_t D[2][4] = {{0, 0, 0, 0}, {0, 0, 0, 0}};
    mma_s8_m16n8k32(D[0], A[0], b0, b1);
    mma_s8_m16n8k32(D[1], A[1], b0, b1);
    const float2 x = *reinterpret_cast<const float2 *>(dt + (u * 8 + b) * 8 + 2 * t);
    float dw[4];   // rows grp, grp + 8, grp + 16, grp + 24
#pragma unroll
    for (int r = 0; r < 4; ++r)
      dw[r] = __half2float(*reinterpret_cast<const __half *>(box + (grp + 8 * r) * 272 + 34 * b));
#pragma unroll
    for (int v = 0; v < 8; ++v) {
      const int32_t sum = D[v >> 2][v & 3];
      if (ISUM && mma_row(v, grp) < rows_left && mma_tok(v, t) < M)
        isum[mma_tok(v, t) * isum_tok + mma_row(v, grp) * isum_row + u * 8 + b] = sum;
      part[v] += __fmul_rn(__fmul_rn(dw[v >> 1], (v & 1) ? x.y : x.x), static_cast<float>(sum));
    }
  }
}

// One Q4_K super-block of the warp's box against unit u: part[v] = sum over
// sub-blocks j, in order, of xd * ((d*sc_j)*isum_j - (dmin*m_j)*xs_j).  The
// lanes first decode their own row's eight (d*sc_j, dmin*m_j) into the warp's
// scratch (lane = row), then read the pairs of the rows they hold.
template <int M, bool ISUM>
__device__ __forceinline__ void tok_mma_q4_k(const uint8_t *box, const uint32_t *qt, const float *dt,
                                             const int32_t *st, float *scr, int u, int lane, float (&part)[8],
                                             int32_t *isum, int64_t isum_row, int64_t isum_tok,
                                             int64_t rows_left) {
  const int grp = lane >> 2, t = lane & 3;
  {
    const uint4 hdr = *reinterpret_cast<const uint4 *>(box + lane * 144);
    const float d = tok_half_lo(hdr.x), dmin = tok_half_hi(hdr.x);
    const uint32_t scA = hdr.y & 0x3f3f3f3fu, mA = hdr.z & 0x3f3f3f3fu;
    const uint32_t scB = (hdr.w & 0x0f0f0f0fu) | ((hdr.y >> 2) & 0x30303030u);
    const uint32_t mB = ((hdr.w >> 4) & 0x0f0f0f0fu) | ((hdr.z >> 2) & 0x30303030u);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t scw = j < 4 ? scA : scB, mw = j < 4 ? mA : mB;
      const int sh = 8 * (j & 3);
      *reinterpret_cast<float2 *>(scr + lane * kTokScStride + 2 * j) =
          make_float2(__fmul_rn(d, static_cast<float>((scw >> sh) & 0xffu)),
                      __fmul_rn(dmin, static_cast<float>((mw >> sh) & 0xffu)));
    }
  }
  __syncwarp();
#pragma unroll
  for (int v = 0; v < 8; ++v) part[v] = 0.0f;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    uint32_t A[2][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
          const uint32_t w = lds32(box + (grp + 8 * h + 16 * mt) * 144 + 16 + 32 * (j >> 1) + 4 * t + 16 * kk);
          A[mt][h + 2 * kk] = (j & 1) ? ((w >> 4) & 0x0f0f0f0fu) : (w & 0x0f0f0f0fu);
        }
    const uint32_t *q = qt + (u * 8 + j) * 64;
    const uint32_t b0 = q[t * 8 + grp], b1 = q[(t + 4) * 8 + grp];
    int32_t D[2][4] = {{0, 0, 0, 0}, {0, 0, 0, 0}};
    mma_s8_m16n8k32(D[0], A[0], b0, b1);
    mma_s8_m16n8k32(D[1], A[1], b0, b1);
    const float2 x = *reinterpret_cast<const float2 *>(dt + (u * 8 + j) * 8 + 2 * t);
    const int2 xs = *reinterpret_cast<const int2 *>(st + (u * 8 + j) * 8 + 2 * t);
#pragma unroll
    for (int v = 0; v < 8; ++v) {
      const int row = mma_row(v, grp);
      const float2 sc = *reinterpret_cast<const float2 *>(scr + row * kTokScStride + 2 * j);
      const int32_t sum = D[v >> 2][v & 3];
      if (ISUM && row < rows_left && mma_tok(v, t) < M)
        isum[mma_tok(v, t) * isum_tok + row * isum_row + u * 8 + j] = sum;
      const float tv = __fmul_rn(sc.x, static_cast<float>(sum));
      const float vv = __fmul_rn(sc.y, static_cast<float>((v & 1) ? xs.y : xs.x));
      part[v] += __fmul_rn((v & 1) ? x.y : x.x, __fsub_rn(tv, vv));
    }
  }
  __syncwarp();   // the scratch is rewritten by the next unit
}

template <int TYPE, int M, bool ISUM>
__global__ void __launch_bounds__(kTokWarps * 32, 1)
    gemv_tokens_mma_kernel(const __grid_constant__ CUtensorMap map0, const __grid_constant__ CUtensorMap map1,
                           const __grid_constant__ TokArgs a) {
  constexpr int UB = tok_unit_bytes<TYPE>();
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = lane >> 2, t = lane & 3;
  const int W = a.W, S = a.stages;
  const int vpw = warp < W ? a.G / W : 0;   // virtual lanes of this warp
  uint32_t *qt = reinterpret_cast<uint32_t *>(base);
  float *dt = reinterpret_cast<float *>(base + a.q_bytes);
  int32_t *st = reinterpret_cast<int32_t *>(base + a.q_bytes + a.d_bytes);
  uint8_t *ring = base + a.ring_off + static_cast<size_t>(warp) * S * a.box_bytes;
  uint64_t *bars = reinterpret_cast<uint64_t *>(base + a.bar_off) + 1 + warp * kTokMaxStages;
  float *red = reinterpret_cast<float *>(base + a.red_off);   // [2][8 warps][M][32 rows]
  float *scr = reinterpret_cast<float *>(base + a.sc_off) + warp * kTokRows * kTokScStride;
  volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(
      reinterpret_cast<uint64_t *>(base + a.bar_off) + 1 + kTokWarps * kTokMaxStages);

  if (threadIdx.x == 0) {
    *abort_flag = 0u;
    prefetch_tensormap(&map0);
    prefetch_tensormap(&map1);
  }
  if (lane == 0)
    for (int s = 0; s < S; ++s) mbar_init(&bars[s], 1);
  fence_barrier_init();
  TokCursor issue;
  issue.first(a, warp, vpw);
  if (lane == 0) {
    TokCursor c = issue;
    for (int s = 0; s < S && c.valid(a); ++s, c.next(a, warp, vpw)) {
      const bool second = c.g >= a.groups0;
      prefetch_l2_tile_2d(second ? &map1 : &map0, c.u * (UB / 4),
                          static_cast<int32_t>((second ? c.g - a.groups0 : c.g) * kTokRows));
    }
  }
  __syncthreads();
  pdl_trigger();
  pdl_wait();

  int64_t n_issued = 0, n_waited = 0;
  if (lane == 0) {
    for (int s = 0; s < S && issue.valid(a); ++s, issue.next(a, warp, vpw), ++n_issued)
      tok_issue<UB>(&map0, &map1, a, issue, ring + static_cast<size_t>(s) * a.box_bytes, &bars[s]);
  }
  {
    // the M tokens' prequantized activations, once, into the layout above
    // (tokens M..7 zero), while the first weight boxes are in flight.  A
    // thread takes one 4-code word of every token (coalesced across the
    // warp) and stores them as two 16-byte words; its loads for four words
    // are all in flight before it stores.
    const uint32_t words = static_cast<uint32_t>(a.K / 4), nb = static_cast<uint32_t>(a.K / 32);
    const uint32_t *xq32 = reinterpret_cast<const uint32_t *>(a.xq);
#pragma unroll 4
    for (uint32_t w = threadIdx.x; w < words; w += blockDim.x) {
      uint32_t v[8];
#pragma unroll
      for (int tok = 0; tok < 8; ++tok) v[tok] = tok < M ? __ldg(xq32 + tok * words + w) : 0u;
      uint4 *dst = reinterpret_cast<uint4 *>(qt + w * 8);
      dst[0] = make_uint4(v[0], v[1], v[2], v[3]);
      dst[1] = make_uint4(v[4], v[5], v[6], v[7]);
    }
    for (uint32_t blk = threadIdx.x; blk < nb; blk += blockDim.x) {
      float d[8];
      int32_t sm[8];
#pragma unroll
      for (int tok = 0; tok < 8; ++tok) {
        d[tok] = tok < M ? __ldg(a.xd + tok * nb + blk) : 0.0f;
        sm[tok] = (TYPE == DSQ_Q4_K && tok < M) ? __ldg(a.xs + tok * nb + blk) : 0;
      }
      float4 *dd = reinterpret_cast<float4 *>(dt + blk * 8);
      dd[0] = make_float4(d[0], d[1], d[2], d[3]);
      dd[1] = make_float4(d[4], d[5], d[6], d[7]);
      if (TYPE == DSQ_Q4_K) {
        int4 *ds = reinterpret_cast<int4 *>(st + blk * 8);
        ds[0] = make_int4(sm[0], sm[1], sm[2], sm[3]);
        ds[1] = make_int4(sm[4], sm[5], sm[6], sm[7]);
      }
    }
  }
  __syncthreads();

  bool ok = true;
  int slot = 0;
  uint32_t parity = 0;
  int buf = 0;
  const int64_t nb = a.K / 32;
  const int64_t rows_total = a.n[0] + a.n[1];
  for (int64_t g = blockIdx.x; g < a.total_groups; g += gridDim.x, buf ^= 1) {
    const bool second = g >= a.groups0;
    const int sgi = second ? 1 : 0;
    const int64_t rbase = (second ? g - a.groups0 : g) * kTokRows;   // first row of the group in its weight
    const int64_t vbase = (second ? a.n[0] : 0) + rbase;               // in [weight 0 rows, weight 1 rows]
    float acc[4][8];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int v = 0; v < 8; ++v) acc[i][v] = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (i >= vpw) break;
      for (int u = warp + W * i; u < a.nunits; u += a.G) {
        ok = ok && *abort_flag == 0u;
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait_for(&bars[slot], parity, a.wait.limit_ns));
        if (!ok) {
          if (lane == 0 && *abort_flag == 0u) {
            *abort_flag = 1u;
            record_timeout(a.wait);
          }
        } else {
          ++n_waited;
          float part[8];
          const uint8_t *box = ring + static_cast<size_t>(slot) * a.box_bytes;
          int32_t *isum = a.isum ? a.isum + vbase * nb : nullptr;
          const int64_t rows_left = a.n[sgi] - rbase;
          if constexpr (TYPE == DSQ_Q8_0)
            tok_mma_q8_0<M, ISUM>(box, qt, dt, u, lane, part, isum, nb, rows_total * nb, rows_left);
          else
            tok_mma_q4_k<M, ISUM>(box, qt, dt, st, scr, u, lane, part, isum, nb, rows_total * nb, rows_left);
#pragma unroll
          for (int v = 0; v < 8; ++v) acc[i][v] += part[v];
          __syncwarp();
          if (lane == 0 && issue.valid(a)) {
            fence_proxy_async_smem();
            tok_issue<UB>(&map0, &map1, a, issue, ring + static_cast<size_t>(slot) * a.box_bytes, &bars[slot]);
            issue.next(a, warp, vpw);
            ++n_issued;
          }
        }
        if (++slot == S) {
          slot = 0;
          parity ^= 1u;
        }
      }
    }
    // butterfly strides >= W inside the warp, as in the CUDA-core form
    float *rb = red + static_cast<size_t>(buf) * kTokWarps * M * 32;
#pragma unroll
    for (int v = 0; v < 8; ++v) {
      float mine;
      if (vpw == 4) mine = (acc[0][v] + acc[2][v]) + (acc[1][v] + acc[3][v]);
      else if (vpw == 2) mine = acc[0][v] + acc[1][v];
      else mine = acc[0][v];
      const int tok = mma_tok(v, t);
      if (tok < M) rb[(warp * M + tok) * 32 + mma_row(v, grp)] = mine;
    }
    __syncthreads();
    // strides < W cross warps: ((r0+r4)+(r2+r6)) + ((r1+r5)+(r3+r7)) for W = 8
    for (int m = warp; m < M; m += kTokWarps) {
      float r[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) r[k] = k < W ? rb[(k * M + m) * 32 + lane] : 0.0f;
      float v;
      if (W == 8) v = ((r[0] + r[4]) + (r[2] + r[6])) + ((r[1] + r[5]) + (r[3] + r[7]));
      else if (W == 4) v = (r[0] + r[2]) + (r[1] + r[3]);
      else if (W == 2) v = r[0] + r[1];
      else v = r[0];
      const int64_t rloc = rbase + lane;
      if (rloc < a.n[sgi] && *abort_flag == 0u) a.y[sgi][m * a.n[sgi] + rloc] = v;
    }
  }
  if (lane == 0) {
    for (int64_t k = n_waited; k < n_issued; ++k)
      mbar_wait_for(&bars[k % S], static_cast<uint32_t>((k / S) & 1), kDrainLimitNs);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 tok_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// The weight rows viewed as uint32 [N][row_bytes / 4]; a box is one
// 256-element unit (68 or 36 words) of 32 rows; rows past N read as zero.
int tok_map(CUtensorMap *map, const void *w, int type, int64_t N, int64_t K, const char *name) {
  auto enc = tok_encode_fn();
  DSQ_REQUIRE(enc != nullptr, DSQ_ERR_CUDA, "%s: cuTensorMapEncodeTiled unavailable", name);
  const int64_t rb = static_cast<int64_t>(dsq_row_bytes(type, K));
  const cuuint64_t gdim[2] = {static_cast<cuuint64_t>(rb / 4), static_cast<cuuint64_t>(N)};
  const cuuint64_t gstride[1] = {static_cast<cuuint64_t>(rb)};
  const cuuint32_t box[2] = {type == DSQ_Q8_0 ? 68u : 36u, static_cast<cuuint32_t>(kTokRows)};
  const cuuint32_t estride[2] = {1u, 1u};
  const CUresult cr = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void *>(w), gdim, gstride, box, estride,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  DSQ_REQUIRE(cr == CUDA_SUCCESS, DSQ_ERR_CUDA, "%s: weight tensor map (%d)", name, (int)cr);
  return DSQ_OK;
}

// The CUDA-core kernel below tok_mma_min_m(type) tokens; from there on the
// tensor-core one, whenever its padded activation layout fits.
template <int TYPE, int M>
const void *tok_kernel_m(bool mma, bool isum) {
  if constexpr (M >= kTokMmaMinM)
    if (mma)
      return isum ? reinterpret_cast<const void *>(gemv_tokens_mma_kernel<TYPE, M, true>)
                  : reinterpret_cast<const void *>(gemv_tokens_mma_kernel<TYPE, M, false>);
  return reinterpret_cast<const void *>(gemv_tokens_kernel<TYPE, M>);
}

template <int TYPE, int M>
cudaError_t tok_launch(bool mma, const CUtensorMap &m0, const CUtensorMap &m1, const TokArgs &a, unsigned grid,
                       size_t smem, cudaStream_t st) {
  if constexpr (M >= kTokMmaMinM)
    if (mma)
      return a.isum ? launch_pdl(gemv_tokens_mma_kernel<TYPE, M, true>, dim3(grid), dim3(kTokWarps * 32), smem, st,
                                 m0, m1, a)
                    : launch_pdl(gemv_tokens_mma_kernel<TYPE, M, false>, dim3(grid), dim3(kTokWarps * 32), smem, st,
                                 m0, m1, a);
  return launch_pdl(gemv_tokens_kernel<TYPE, M>, dim3(grid), dim3(kTokWarps * 32), smem, st, m0, m1, a);
}

template <int TYPE>
const void *tok_kernel(int M, bool mma, bool isum) {
  switch (M) {
    case 1: return tok_kernel_m<TYPE, 1>(mma, isum);
    case 2: return tok_kernel_m<TYPE, 2>(mma, isum);
    case 3: return tok_kernel_m<TYPE, 3>(mma, isum);
    case 4: return tok_kernel_m<TYPE, 4>(mma, isum);
    case 5: return tok_kernel_m<TYPE, 5>(mma, isum);
    case 6: return tok_kernel_m<TYPE, 6>(mma, isum);
    case 7: return tok_kernel_m<TYPE, 7>(mma, isum);
    default: return tok_kernel_m<TYPE, 8>(mma, isum);
  }
}

template <int TYPE>
cudaError_t tok_dispatch(int M, bool mma, const CUtensorMap &m0, const CUtensorMap &m1, const TokArgs &a,
                         unsigned grid, size_t smem, cudaStream_t st) {
  switch (M) {
    case 1: return tok_launch<TYPE, 1>(mma, m0, m1, a, grid, smem, st);
    case 2: return tok_launch<TYPE, 2>(mma, m0, m1, a, grid, smem, st);
    case 3: return tok_launch<TYPE, 3>(mma, m0, m1, a, grid, smem, st);
    case 4: return tok_launch<TYPE, 4>(mma, m0, m1, a, grid, smem, st);
    case 5: return tok_launch<TYPE, 5>(mma, m0, m1, a, grid, smem, st);
    case 6: return tok_launch<TYPE, 6>(mma, m0, m1, a, grid, smem, st);
    case 7: return tok_launch<TYPE, 7>(mma, m0, m1, a, grid, smem, st);
    default: return tok_launch<TYPE, 8>(mma, m0, m1, a, grid, smem, st);
  }
}

size_t tok_align(size_t v, size_t a) { return (v + a - 1) / a * a; }

int run_tokens(const char *name, int type, const void *w0, int64_t N0, const void *w1, int64_t N1, int64_t K,
               int64_t M, const int8_t *xq, const float *xd, const int32_t *xs, float *y0, float *y1,
               int32_t *isum, cudaStream_t stream) {
  DSQ_REQUIRE(type == DSQ_Q8_0 || type == DSQ_Q4_K, DSQ_ERR_INVALID_ARG, "%s: unsupported type %d", name, type);
  DSQ_REQUIRE(K > 0 && N0 >= 0 && N1 >= 0, DSQ_ERR_INVALID_ARG, "%s: negative size", name);
  DSQ_REQUIRE(M >= 1 && M <= kTokMaxM, DSQ_ERR_SHAPE, "%s: M=%lld tokens (1..%d supported)", name, (long long)M,
              kTokMaxM);
  DSQ_REQUIRE(K % 256 == 0, DSQ_ERR_SHAPE, "%s: K=%lld must be a multiple of 256", name, (long long)K);
  DSQ_REQUIRE(N0 + N1 <= (int64_t(1) << 31), DSQ_ERR_SHAPE, "%s: too many rows", name);
  // the tensor-core form keeps 8 (padded) tokens in its own layout; where
  // that does not fit, the CUDA-core kernel takes the call
  const size_t per_token = static_cast<size_t>(K) + (K / 32) * 4 * (type == DSQ_Q4_K ? 2 : 1);
  const bool mma = M >= tok_mma_min_m(type) && 8 * per_token <= kTokMaxActSmem;
  const int64_t Mk = mma ? 8 : M;
  const size_t q_bytes = static_cast<size_t>(Mk) * K;
  const size_t d_bytes = static_cast<size_t>(Mk) * (K / 32) * 4;
  const size_t s_bytes = type == DSQ_Q4_K ? d_bytes : 0;
  DSQ_REQUIRE(q_bytes + d_bytes + s_bytes <= kTokMaxActSmem, DSQ_ERR_SHAPE,
              "%s: %lld tokens of K=%lld exceed the %zu bytes of shared memory kept for activations", name,
              (long long)M, (long long)K, kTokMaxActSmem);
  if (N0 + N1 == 0) return DSQ_OK;
  DSQ_REQUIRE(xq && xd && (type == DSQ_Q8_0 || xs), DSQ_ERR_INVALID_ARG, "%s: null activation pointer", name);
  DSQ_REQUIRE((N0 == 0 || (w0 && y0)) && (N1 == 0 || (w1 && y1)), DSQ_ERR_INVALID_ARG,
              "%s: null weight/output pointer", name);
  DSQ_REQUIRE(aligned(xq, 16) && aligned(xd, 16) && (type == DSQ_Q8_0 || aligned(xs, 16)), DSQ_ERR_ALIGNMENT,
              "%s: xq/xd/xs must be 16-byte aligned", name);
  DSQ_REQUIRE((N0 == 0 || (aligned(w0, 16) && aligned(y0, 4))) && (N1 == 0 || (aligned(w1, 16) && aligned(y1, 4))),
              DSQ_ERR_ALIGNMENT, "%s: weights must be 16-byte and outputs 4-byte aligned", name);
  WaitCtl ctl;
  int sms = 0;
  int rc = wait_ctl(&ctl, &sms);
  if (rc != DSQ_OK) return rc;

  TokArgs a{};
  a.y[0] = y0;
  a.y[1] = y1;
  a.n[0] = N0;
  a.n[1] = N1;
  a.groups0 = (N0 + kTokRows - 1) / kTokRows;
  a.total_groups = a.groups0 + (N1 + kTokRows - 1) / kTokRows;
  a.K = K;
  a.nunits = static_cast<int>(K / 256);
  a.G = 1;
  while (a.G < a.nunits && a.G < 32) a.G <<= 1;
  a.W = a.G < kTokWarps ? a.G : kTokWarps;
  a.box_bytes = static_cast<uint32_t>(kTokRows * (type == DSQ_Q8_0 ? 272 : 144));
  a.q_bytes = static_cast<uint32_t>(q_bytes);
  a.d_bytes = static_cast<uint32_t>(d_bytes);
  a.s_bytes = static_cast<uint32_t>(s_bytes);
  a.xq = xq;
  a.xd = xd;
  a.xs = xs;
  a.isum = isum;
  a.wait = ctl;
  // shared memory: activations | ring (W warps x stages x box) | barriers |
  // reduction | Q4_K scale scratch of the tensor-core form
  const size_t act = tok_align(q_bytes + d_bytes + s_bytes, 1024);
  const size_t bars = (1 + kTokWarps * kTokMaxStages + 1) * sizeof(uint64_t);
  const size_t red = 2 * static_cast<size_t>(kTokWarps) * M * 32 * sizeof(float);
  const size_t scr = (mma && type == DSQ_Q4_K) ? static_cast<size_t>(kTokWarps) * kTokRows * kTokScStride * 4 : 0;
  const size_t fixed = 1024 + act + tok_align(bars, 16) + red + scr;
  const size_t per_stage = static_cast<size_t>(kTokWarps) * a.box_bytes;
  int stages = static_cast<int>((kTokSmemLimit - fixed) / per_stage);
  if (stages > kTokMaxStages) stages = kTokMaxStages;
  DSQ_REQUIRE(stages >= 2, DSQ_ERR_SHAPE, "%s: no pipeline fits next to %lld tokens of K=%lld", name, (long long)M,
              (long long)K);
  a.stages = stages;
  a.ring_off = static_cast<uint32_t>(act);
  a.bar_off = static_cast<uint32_t>(act + per_stage * stages);
  a.red_off = static_cast<uint32_t>(a.bar_off + tok_align(bars, 16));
  a.sc_off = static_cast<uint32_t>(a.red_off + red);
  const size_t smem = 1024 + a.sc_off + scr;

  CUtensorMap m0, m1;
  const void *wa = N0 > 0 ? w0 : w1;
  rc = tok_map(&m0, wa, type, N0 > 0 ? N0 : N1, K, name);
  if (rc != DSQ_OK) return rc;
  if (N1 > 0) {
    rc = tok_map(&m1, w1, type, N1, K, name);
    if (rc != DSQ_OK) return rc;
  } else {
    m1 = m0;
  }
  const int64_t slots = sms;
  const unsigned grid = static_cast<unsigned>(a.total_groups < slots ? a.total_groups : slots);
  const int mi = static_cast<int>(M);
  rc = set_smem_once(type == DSQ_Q8_0 ? tok_kernel<DSQ_Q8_0>(mi, mma, isum != nullptr)
                                     : tok_kernel<DSQ_Q4_K>(mi, mma, isum != nullptr),
                     static_cast<int>(smem), name);
  if (rc != DSQ_OK) return rc;
  const cudaError_t e = type == DSQ_Q8_0 ? tok_dispatch<DSQ_Q8_0>(mi, mma, m0, m1, a, grid, smem, stream)
                                         : tok_dispatch<DSQ_Q4_K>(mi, mma, m0, m1, a, grid, smem, stream);
  if (e != cudaSuccess) return fail(DSQ_ERR_LAUNCH, "%s: %s", name, cudaGetErrorString(e));
  return after_launch(name);
}

}  // namespace

// One token through the multi-token kernel, with the caller's name in any
// error message (the decode GEMV entry points route mid-length matrices here).
int gemv_one_token(const char *name, int type, const void *w, int64_t N, int64_t K, const int8_t *xq,
                   const float *xd, const int32_t *xs, float *y, cudaStream_t stream) {
  return run_tokens(name, type, w, N, nullptr, 0, K, 1, xq, xd, xs, y, nullptr, nullptr, stream);
}
}  // namespace dsq

extern "C" {

int dsq_gemv_tokens(int type, const void *w0, int64_t N0, const void *w1, int64_t N1, int64_t K, int64_t M,
                    const int8_t *xq, const float *xd, const int32_t *xs, float *y0, float *y1, void *stream) {
  using namespace dsq;
  return run_tokens("dsq_gemv_tokens", type, w0, N0, w1, N1, K, M, xq, xd, xs, y0, y1, nullptr, as_stream(stream));
}

int dsq_test_block_sums_tokens(int type, const void *w, int64_t N, int64_t K, int64_t M, const int8_t *xq,
                               const float *xd, const int32_t *xs, float *y, int32_t *isum, void *stream) {
  using namespace dsq;
  DSQ_REQUIRE(isum != nullptr || N == 0, DSQ_ERR_INVALID_ARG, "dsq_test_block_sums_tokens: null isum");
  DSQ_REQUIRE(aligned(isum, 4), DSQ_ERR_ALIGNMENT, "dsq_test_block_sums_tokens: isum alignment");
  return run_tokens("dsq_test_block_sums_tokens", type, w, N, nullptr, 0, K, M, xq, xd, xs, y, nullptr, isum,
                    as_stream(stream));
}

}  // extern "C"
