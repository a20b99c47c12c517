// prefill.cu -- prefill projection: dequantize Q8_0 / Q4_K weights into a
// dense tensor-core GEMM, Y[M][N] = X[M][K] * deq(W)^T.
//
// Source: "Support AProjQ4 GGUFs: Q4_K dense attention projections"
// (antirez/ds4 PR #621), GB10 test report (Q4_K prefill fell to 54.6 t/s
// until a dequant + GEMM prefill path existed; the tester calls that path
// the deciding factor) and the consolidated results (grouped attention-A
// prefill).  The pages give no kernel; this is a B200-first design.
//
// Numerics: 16-bit float operands, fp32 accumulation.  Each activation row
// is scaled by an exact power of two 2^s_m (its largest magnitude lands in
// [2^14, 2^15)) and rounded to binary16; each weight element is dequantized
// in fp32 ((d*q) for Q8_0, (d*sc)*q - dmin*m for Q4_K) and rounded to
// binary16; the fp32 dot is scaled back by 2^-s_m.  binary16 (10 explicit
// mantissa bits) keeps the operand rounding at ~3e-4 relative L2 on this
// workload; bfloat16 operands would give ~2.3e-3, above the 2e-3 bar.
//
// Kernel (one CTA per 128 weight rows x TN tokens x K-split):
//  * the weight tile is the MMA's A operand (M = 128 rows of W), the
//    activation tile its B operand (N = TN tokens) -- "swap AB", so small
//    token counts still use a full 128-row MMA and the weight stream stays
//    HBM-efficient down to one token;
//  * warp 0: TMA producer of the activation tiles (fp16, 128-byte swizzle);
//  * warp 1: allocates TMEM and issues tcgen05.mma (kind::f16, fp32
//    accumulate in TMEM), releasing smem stages with tcgen05.commit;
//  * warps 2-5: each thread owns one weight row: it streams the row's raw
//    blocks from global memory (one 256-element unit ahead), dequantizes 64
//    elements per stage into the 128-byte-swizzled K-major layout the MMA
//    reads, then runs the epilogue (tcgen05.ld -> scale by 2^-s_m -> global,
//    coalesced across the 32 rows of a warp);
//  * every wait is bounded; an expired wait records a timeout, stops every
//    role, drains copies and MMAs in flight, frees TMEM and returns.
#include <cudaTypedefs.h>
#include <mutex>

#include "../../include/dsq_test.h"
#include "dsq_host.h"

namespace dsq {
namespace {

constexpr int kBM = 128;          // weight rows per MMA (the MMA's M)
constexpr int kHalves = 2;        // a CTA tile holds 2 x 128 weight rows sharing each activation stage
constexpr int kTileN = kBM * kHalves;   // weight rows per CTA tile
constexpr int kBK = 64;           // K elements per pipeline stage
constexpr int kAColsHalf = kBK / 2;     // TMEM columns of one half's A stage (2 fp16 per column)
constexpr int kAColsStage = kHalves * kAColsHalf;   // 64
constexpr int kTmemCols = 512;    // the CTA owns all of TMEM (1 CTA per SM)
// warp roles
constexpr int kWarpX = 0;         // bulk-copy producer: fp16 activation stages
constexpr int kWarpMma = 1;       // TMEM owner, tcgen05.mma issuer
constexpr int kWarpConv0 = 2;     // warps 2..9: one weight row per thread, dequantize into TMEM
constexpr int kConvWarps = 8;
constexpr int kWarpEpi0 = kWarpConv0 + kConvWarps;   // warps 10..13: TMEM -> global epilogue
constexpr int kWarpW = kWarpEpi0 + 4;                 // warp 14: TMA producer of raw weight units
constexpr int kThreads = (kWarpW + 1) * 32;

struct PrefillArgs {
  const uint8_t *w;       // packed weight rows
  int64_t row_bytes;
  int64_t N, K, M;
  const __half *x16;      // fp16 activations, tile-major and swizzled (see x_to_f16_kernel)
  const int32_t *shift;   // [M] activation row shifts
  float *y;               // [M][N], or [splits][M][N] partials
  int units_per_split;    // 256-element units of K per split
  int splits;
  int tn;                 // tokens per tile (MMA N): 32..256, multiple of 32
  int groups_b;           // activation slots in shared memory (one 256-element unit of K each)
  int raw_slots;          // raw weight unit slots in shared memory (256 rows x unit bytes each)
  int stages_a;           // dequantized weight stages in TMEM
  int64_t tiles_m, tiles_n, total_tiles;
  WaitCtl wait;
};

// ---------------------------------------------------------------- dequant --
// 256-element unit of one weight row in registers: Q8_0 = 8 blocks (272 B),
// Q4_K = one super-block (144 B).
template <int TYPE> struct RawUnit;
template <> struct RawUnit<DSQ_Q8_0> { static constexpr int kVecs = 17; uint4 v[17]; };
template <> struct RawUnit<DSQ_Q4_K> { static constexpr int kVecs = 9; uint4 v[9]; };
template <int TYPE> __host__ __device__ constexpr int unit_bytes() { return TYPE == DSQ_Q8_0 ? 272 : 144; }

template <int TYPE>
__device__ __forceinline__ void load_unit(RawUnit<TYPE> &u, const uint8_t *p) {
  const uint4 *p4 = reinterpret_cast<const uint4 *>(p);
#pragma unroll
  for (int i = 0; i < RawUnit<TYPE>::kVecs; ++i) u.v[i] = __ldg(p4 + i);
}

template <int TYPE>
__device__ __forceinline__ uint32_t word_of(const RawUnit<TYPE> &u, int i) {
  const uint4 &v = u.v[i >> 2];
  return (i & 3) == 0 ? v.x : (i & 3) == 1 ? v.y : (i & 3) == 2 ? v.z : v.w;
}

__device__ __forceinline__ uint32_t h2_bits(__half2 h) { return *reinterpret_cast<uint32_t *>(&h); }
__device__ __forceinline__ __half2 bits_h2(uint32_t b) { return *reinterpret_cast<__half2 *>(&b); }

// 4 int8 codes (one word) times an fp16 scale -> 4 binary16 values (2 words).
// A biased byte u = q + 128 placed under exponent byte 0x64 is the half
// 1024 + u; subtracting 1152 gives q exactly; the product d*q (exact in
// fp32: 11 x 7 significant bits) is then rounded once to binary16 by the
// half multiply -- the same value as fp16_rne(float(d) * q).
__device__ __forceinline__ void q8x4_to_h(uint32_t qw, __half2 d2, uint32_t &o0, uint32_t &o1) {
  const uint32_t b = qw ^ 0x80808080u;
  const __half2 bias = __half2half2(__ushort_as_half(0x6480));   // 1152.0
  const __half2 lo = __hsub2(bits_h2(__byte_perm(b, 0x64646464u, 0x5140)), bias);
  const __half2 hi = __hsub2(bits_h2(__byte_perm(b, 0x64646464u, 0x7362)), bias);
  o0 = h2_bits(__hmul2_rn(lo, d2));
  o1 = h2_bits(__hmul2_rn(hi, d2));
}

// Q8_0: piece p (64 elements = blocks 2p, 2p+1) as 8 chunks of 8 halves.
__device__ __forceinline__ void piece_q8_0(const RawUnit<DSQ_Q8_0> &u, int p, uint32_t (&out)[32]) {
#pragma unroll
  for (int half_ = 0; half_ < 2; ++half_) {
    const int b = 2 * p + half_;
    // block b starts at byte 34b; see gemv.cu for the word alignment rule
    uint32_t qwd[8];
    __half dh;
    if ((b & 1) == 0) {
      const int a = 17 * b / 2;
      dh = __ushort_as_half(static_cast<unsigned short>(word_of(u, a) & 0xffffu));
#pragma unroll
      for (int i = 0; i < 8; ++i) qwd[i] = __funnelshift_r(word_of(u, a + i), word_of(u, a + i + 1), 16);
    } else {
      const int a = (17 * b - 1) / 2;
      dh = __ushort_as_half(static_cast<unsigned short>(word_of(u, a) >> 16));
#pragma unroll
      for (int i = 0; i < 8; ++i) qwd[i] = word_of(u, a + 1 + i);
    }
    const __half2 d2 = __half2half2(dh);
#pragma unroll
    for (int i = 0; i < 8; ++i) q8x4_to_h(qwd[i], d2, out[16 * half_ + 2 * i], out[16 * half_ + 2 * i + 1]);
  }
}

// Q4_K: piece p (64 elements = sub-blocks 2p (low nibbles) and 2p+1 (high
// nibbles) of bytes qs[32p .. 32p+31]).  Each value is fp32 (d*sc)*q - dmin*m
// (one rounding: (d*sc)*q and dmin*m are exact), then binary16 RNE.
__device__ __forceinline__ void piece_q4_k(const RawUnit<DSQ_Q4_K> &u, int p, uint32_t (&out)[32]) {
  const uint32_t w0 = word_of(u, 0);
  const float d = __half2float(__ushort_as_half(static_cast<unsigned short>(w0 & 0xffffu)));
  const float dmin = __half2float(__ushort_as_half(static_cast<unsigned short>(w0 >> 16)));
  const uint32_t s0 = word_of(u, 1), s1 = word_of(u, 2), s2 = word_of(u, 3);
#pragma unroll
  for (int half_ = 0; half_ < 2; ++half_) {
    const int j = 2 * p + half_;
    uint32_t scw, mw;
    if (j < 4) {
      scw = s0 & 0x3f3f3f3fu;
      mw = s1 & 0x3f3f3f3fu;
    } else {
      scw = (s2 & 0x0f0f0f0fu) | ((s0 >> 2) & 0x30303030u);
      mw = ((s2 >> 4) & 0x0f0f0f0fu) | ((s1 >> 2) & 0x30303030u);
    }
    const int sh = 8 * (j & 3);
    const float a = __fmul_rn(d, static_cast<float>((scw >> sh) & 0xffu));
    const float nb = -__fmul_rn(dmin, static_cast<float>((mw >> sh) & 0xffu));
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t byte4 = word_of(u, 4 + 8 * p + i);
      const uint32_t nib = half_ ? ((byte4 >> 4) & 0x0f0f0f0fu) : (byte4 & 0x0f0f0f0fu);
      float v[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        // 0x4B000000 | q is the float 2^23 + q; subtracting 2^23 is exact
        const float f = __uint_as_float(__byte_perm(nib, 0x4B000000u, 0x7540 + e));
        v[e] = __fmaf_rn(__fsub_rn(f, 8388608.0f), a, nb);
      }
      out[16 * half_ + 2 * i] = h2_bits(__floats2half2_rn(v[0], v[1]));
      out[16 * half_ + 2 * i + 1] = h2_bits(__floats2half2_rn(v[2], v[3]));
    }
  }
}

template <int TYPE>
__device__ __forceinline__ void dequant_piece(const RawUnit<TYPE> &u, int p, uint32_t (&out)[32]) {
  if constexpr (TYPE == DSQ_Q8_0) piece_q8_0(u, p, out);
  else piece_q4_k(u, p, out);
}


// ------------------------------------------------------------------ GEMM ---
// TMEM map (512 columns x 128 lanes): [0, 2*tn) the fp32 accumulators of the
// two halves (half h at h*tn); then stages_a dequantized-weight stages of
// 64 columns each (half h at +32h), lane = row of the half, each column two
// consecutive fp16 K elements.  The MMA reads A from TMEM and B (the
// activation tile) from shared memory, so shared memory carries only the
// activation stream.
struct Smem {
  uint8_t *b;          // groups_b x 4 x tn*128: activation tiles of one K unit each (MMA B)
  uint64_t *bfull;     // activation unit landed (1 + tx)
  uint64_t *bempty;    // MMA finished reading an activation unit (commit)
  uint64_t *afull;     // converters stored a TMEM weight stage (count 8 warps)
  uint64_t *aempty;    // MMA finished reading a TMEM weight stage (commit)
  uint8_t *raw;        // raw_slots x 256 rows x unit bytes: raw weight units (TMA)
  uint64_t *rfull;     // raw unit landed (1 + tx)
  uint64_t *rempty;    // converters copied a raw unit into registers (count 8 warps)
  uint64_t *accfull;   // accumulators complete (commit)
  uint64_t *accempty;  // epilogue drained the accumulators (count 4)
  uint64_t *drain;     // MMA drain after an abort
  uint32_t *tmem;      // TMEM base address
  volatile int *abort;
};

__device__ __forceinline__ Smem carve(uint8_t *base, int groups_b, int stages_a, int tn, int raw_slots, int raw_bytes) {
  Smem s;
  s.b = base;
  s.raw = s.b + static_cast<size_t>(groups_b) * 4 * tn * 128;
  uint64_t *p = reinterpret_cast<uint64_t *>(s.raw + static_cast<size_t>(raw_slots) * raw_bytes);
  s.bfull = p;
  s.bempty = s.bfull + groups_b;
  s.afull = s.bempty + groups_b;
  s.aempty = s.afull + stages_a;
  s.rfull = s.aempty + stages_a;
  s.rempty = s.rfull + raw_slots;
  s.accfull = s.rempty + raw_slots;
  s.accempty = s.accfull + 1;
  s.drain = s.accempty + 1;
  s.tmem = reinterpret_cast<uint32_t *>(s.drain + 1);
  s.abort = reinterpret_cast<volatile int *>(s.tmem + 1);
  return s;
}

__device__ __forceinline__ bool aborted(const Smem &s) { return *s.abort != 0; }
__device__ __forceinline__ void set_abort(const Smem &s, const WaitCtl &w) {
  *s.abort = 1;
  record_timeout(w);
}

// One thread's bounded wait; on expiry (or an abort raised elsewhere) it
// raises the CTA abort flag and returns false.  sleep_ns: poll back-off for
// waiters off the critical path.
__device__ __forceinline__ bool wait_or_abort(const Smem &s, uint64_t *bar, uint32_t parity, const WaitCtl &w,
                                              uint32_t sleep_ns = 0) {
  if (aborted(s)) return false;
  if (mbar_wait_for(bar, parity, w.limit_ns, sleep_ns)) return true;
  set_abort(s, w);
  return false;
}

// Tile t -> (first token, first weight row, K split); consecutive tiles
// share a weight tile, so CTAs running side by side reuse it from L2.
struct Tile {
  int64_t m0, n0;
  int u0, u1;
  int split;
};
__device__ __forceinline__ Tile tile_of(const PrefillArgs &a, int64_t t) {
  Tile tl;
  const int64_t m = t % a.tiles_m;
  const int64_t rest = t / a.tiles_m;
  tl.split = static_cast<int>(rest % a.splits);
  tl.m0 = m * a.tn;
  tl.n0 = (rest / a.splits) * kTileN;
  tl.u0 = tl.split * a.units_per_split;
  tl.u1 = min(tl.u0 + a.units_per_split, static_cast<int>(a.K / 256));
  return tl;
}

// Persistent CTA over tiles of 256 weight rows x tn tokens x one K split:
// tiles blockIdx.x, blockIdx.x + gridDim.x, ...  Each 64-K stage holds the
// activation tile once (shared memory) and the two 128-row weight halves
// (TMEM); the MMA warp issues both halves against the same activation tile.
template <int TYPE>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ PrefillArgs a) {
  constexpr int UB = unit_bytes<TYPE>();
  constexpr int RAW_BYTES = kTileN * UB;   // one unit of the tile's 256 rows
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const Smem s = carve(base, a.groups_b, a.stages_a, a.tn, a.raw_slots, RAW_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int SB = a.groups_b, SA = a.stages_a, SR = a.raw_slots;
  const uint32_t stage_b_bytes = static_cast<uint32_t>(a.tn) * 128u;   // one 64-K activation tile
  const uint32_t group_b_bytes = 4u * stage_b_bytes;                    // one 256-K unit
  const int units = static_cast<int>(a.K / 256);

  if (threadIdx.x == 0) {
    for (int i = 0; i < SB; ++i) {
      mbar_init(&s.bfull[i], 1);
      mbar_init(&s.bempty[i], 1);
    }
    for (int i = 0; i < SA; ++i) {
      mbar_init(&s.afull[i], kConvWarps);
      mbar_init(&s.aempty[i], 1);
    }
    for (int i = 0; i < SR; ++i) {
      mbar_init(&s.rfull[i], 1);
      mbar_init(&s.rempty[i], kConvWarps);
    }
    mbar_init(s.accfull, 1);
    mbar_init(s.accempty, 4);
    mbar_init(s.drain, 1);
    *s.abort = 0;
    fence_barrier_init();
    prefetch_tensormap(&tmap_w);
  }
  const int conv = (warp >= kWarpConv0 && warp < kWarpEpi0) ? warp - kWarpConv0 : -1;
  // converter warp c: half c / 4, TMEM lane quadrant warp % 4 (a warp may only
  // touch its own quadrant), so its row within the half is 32 * (warp % 4) + lane
  const int conv_half = conv / 4, conv_rr = 32 * (warp & 3) + lane;
  if (warp == kWarpW && lane == 0 && blockIdx.x < a.total_tiles) {
    // weights are read-only: start the first units toward L2 while the
    // activation-rounding kernel before us finishes
    const Tile tl = tile_of(a, blockIdx.x);
    for (int u = tl.u0; u < tl.u1 && u < tl.u0 + 2; ++u)
      for (int h = 0; h < kHalves; ++h)
        prefetch_l2_tile_2d(&tmap_w, u * (UB / 4), static_cast<int32_t>(tl.n0 + h * kBM));
  }
  if (warp == kWarpMma) {
    tmem_alloc(s.tmem, static_cast<uint32_t>(kTmemCols));
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  pdl_trigger();
  pdl_wait();
  const uint32_t tmem_base = *s.tmem;
  const uint32_t a_col0 = static_cast<uint32_t>(kHalves * a.tn);   // first weight-stage column

  if (warp == kWarpX) {
    // ---------------------------------------- activation stages (bulk copy)
    if (lane == 0) {
      const uint64_t keep = l2_policy_evict_last();   // every weight tile re-reads these
      // One bulk copy per 256-element K unit: the activation tile of the
      // unit is contiguous in the tile-major layout.  Ring position kept
      // incrementally (no integer division on this path): slot sb of round
      // rnd; round r >= 1 first waits for the MMA's release from round r - 1.
      int64_t gs = 0;
      int sb = 0;
      uint32_t rnd = 0;
      for (int64_t t = blockIdx.x; t < a.total_tiles && !aborted(s); t += gridDim.x) {
        const Tile tl = tile_of(a, t);
        const int64_t mt = tl.m0 / a.tn;
        for (int u = tl.u0; u < tl.u1; ++u, ++gs) {
          if (rnd > 0 && !wait_or_abort(s, &s.bempty[sb], (rnd - 1) & 1u, a.wait, 64)) break;
          mbar_arrive_expect_tx(&s.bfull[sb], group_b_bytes);
          bulk_g2s(s.b + static_cast<size_t>(sb) * group_b_bytes,
                   reinterpret_cast<const uint8_t *>(a.x16) + (mt * units + u) * static_cast<int64_t>(group_b_bytes),
                   group_b_bytes, &s.bfull[sb], keep);
          if (++sb == SB) {
            sb = 0;
            ++rnd;
          }
        }
      }
      if (aborted(s))
        for (int64_t g = (gs > SB ? gs - SB : 0); g < gs; ++g)
          mbar_wait_for(&s.bfull[g % SB], static_cast<uint32_t>((g / SB) & 1), kDrainLimitNs);
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_f16(kBM, static_cast<uint32_t>(a.tn), 0);
      const uint32_t b_base = smem_u32(s.b);
      int64_t i = 0;
      int sb = 0, sa = 0;
      uint32_t pb = 0, pa = 0;   // phase parity of the current round of each ring
      bool ok = true;
      for (int64_t t = blockIdx.x; t < a.total_tiles && ok; t += gridDim.x, ++i) {
        const Tile tl = tile_of(a, t);
        if (i >= 1 && !wait_or_abort(s, s.accempty, static_cast<uint32_t>((i - 1) & 1), a.wait)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        for (int u = tl.u0; u < tl.u1 && ok; ++u) {
          if (!wait_or_abort(s, &s.bfull[sb], pb, a.wait)) {
            ok = false;
            break;
          }
          for (int kb4 = 0; kb4 < 4; ++kb4) {
            if (!wait_or_abort(s, &s.afull[sa], pa, a.wait)) {
              ok = false;
              break;
            }
            tc_fence_after_sync();
            const uint32_t b_addr = b_base + static_cast<uint32_t>(sb) * group_b_bytes + static_cast<uint32_t>(kb4) * stage_b_bytes;
            const uint32_t a_tmem = tmem_base + a_col0 + static_cast<uint32_t>(sa * kAColsStage);
            const bool first = (u == tl.u0 && kb4 == 0);
#pragma unroll
            for (int k = 0; k < kBK / 16; ++k) {
              const uint64_t bdesc = umma_desc_sw128(b_addr + 32 * k);
#pragma unroll
              for (int h = 0; h < kHalves; ++h)
                umma_f16_ts(tmem_base + static_cast<uint32_t>(h * a.tn),
                            a_tmem + static_cast<uint32_t>(h * kAColsHalf + 8 * k), bdesc, idesc,
                            (!first || k > 0) ? 1u : 0u);
            }
            umma_commit(&s.aempty[sa]);
            if (++sa == SA) {
              sa = 0;
              pa ^= 1u;
            }
          }
          if (!ok) break;
          umma_commit(&s.bempty[sb]);
          if (++sb == SB) {
            sb = 0;
            pb ^= 1u;
          }
        }
        if (ok) umma_commit(s.accfull);
      }
      if (!ok) {
        umma_commit(s.drain);
        mbar_wait_for(s.drain, 0, kDrainLimitNs);
      }
    }
  } else if (warp == kWarpW) {
    // ------------------------------------------- raw weight units (TMA)
    if (lane == 0) {
      int64_t gu = 0;
      int rs = 0;
      uint32_t rnd = 0;
      for (int64_t t = blockIdx.x; t < a.total_tiles && !aborted(s); t += gridDim.x) {
        const Tile tl = tile_of(a, t);
        for (int u = tl.u0; u < tl.u1; ++u, ++gu) {
          if (rnd > 0 && !wait_or_abort(s, &s.rempty[rs], (rnd - 1) & 1u, a.wait, 64)) break;
          mbar_arrive_expect_tx(&s.rfull[rs], static_cast<uint32_t>(RAW_BYTES));
          for (int h = 0; h < kHalves; ++h)
            tma_load_2d(s.raw + static_cast<size_t>(rs) * RAW_BYTES + static_cast<size_t>(h) * kBM * UB, &tmap_w,
                        u * (UB / 4), static_cast<int32_t>(tl.n0 + h * kBM), &s.rfull[rs]);
          if (++rs == SR) {
            rs = 0;
            ++rnd;
          }
        }
      }
      if (aborted(s))
        for (int64_t g = (gu > SR ? gu - SR : 0); g < gu; ++g)
          mbar_wait_for(&s.rfull[g % SR], static_cast<uint32_t>((g / SR) & 1), kDrainLimitNs);
    }
  } else if (conv >= 0) {
    // ------------------------------------------ converters (dequantize)
    // Thread (half h, row rr) owns weight row 128h + rr of the tile.  It
    // reads the row's raw 256-element units from global memory (the next
    // unit is prefetched into L2 while this one is converted) and writes 64
    // dequantized fp16 per stage into its TMEM lane with one store.
    const int h = conv_half, rr = conv_rr;
    const uint32_t lane_addr = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    int sa = 0;
    uint32_t rnd = 0;   // ring round; round r >= 1 waits for the release from round r - 1
    int rs = 0;         // raw unit slot and its phase parity
    uint32_t rpar = 0;
    bool ok = true;
    for (int64_t t = blockIdx.x; t < a.total_tiles && ok; t += gridDim.x) {
      const Tile tl = tile_of(a, t);
      for (int u = tl.u0; u < tl.u1 && ok; ++u) {
        const bool got = wait_or_abort(s, &s.rfull[rs], rpar, a.wait);
        if (__any_sync(0xffffffffu, !got)) {
          ok = false;
          break;
        }
        RawUnit<TYPE> ru;
        const uint4 *src = reinterpret_cast<const uint4 *>(s.raw + static_cast<size_t>(rs) * RAW_BYTES +
                                                           static_cast<size_t>(h * kBM + rr) * UB);
#pragma unroll
        for (int v = 0; v < RawUnit<TYPE>::kVecs; ++v) ru.v[v] = src[v];
        __syncwarp();
        if (lane == 0) mbar_arrive(&s.rempty[rs]);
        if (++rs == SR) {
          rs = 0;
          rpar ^= 1u;
        }
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          if (rnd > 0) {
            const bool free_ = wait_or_abort(s, &s.aempty[sa], (rnd - 1) & 1u, a.wait, 32);
            if (__any_sync(0xffffffffu, !free_)) {
              ok = false;
              break;
            }
          }
          uint32_t v[32];
          dequant_piece<TYPE>(ru, p, v);   // rows past N arrive as zero blocks: zeros
          tc_fence_after_sync();
          tmem_st_32cols(tmem_base + lane_addr + a_col0 + static_cast<uint32_t>(sa * kAColsStage + h * kAColsHalf), v);
          tmem_st_wait();
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive(&s.afull[sa]);
          if (++sa == SA) {
            sa = 0;
            ++rnd;
          }
        }
      }
    }
  } else if (warp >= kWarpEpi0) {
    // ------------------------------- epilogue: TMEM -> y * 2^-s_m
    const int q = warp & 3;                 // TMEM lane quadrant of this warp
    const int r = 32 * q + lane;            // row within each 128-row half
    int64_t i = 0;
    for (int64_t t = blockIdx.x; t < a.total_tiles; t += gridDim.x, ++i) {
      const Tile tl = tile_of(a, t);
      const bool got = wait_or_abort(s, s.accfull, static_cast<uint32_t>(i & 1), a.wait, 256);
      if (__any_sync(0xffffffffu, !got)) break;
      tc_fence_after_sync();
      float *y = a.y + static_cast<int64_t>(tl.split) * a.M * a.N;
      for (int hh = 0; hh < kHalves; ++hh) {
        const int64_t n = tl.n0 + hh * kBM + r;
        for (int c = 0; c < a.tn / 32; ++c) {
          uint32_t v[32];
          tmem_ld_32cols(tmem_base + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(hh * a.tn + 32 * c),
                         v);
          tmem_ld_wait();
          if (hh == kHalves - 1 && c == a.tn / 32 - 1) {
            // every accumulator column is in registers: let the next tile start
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(s.accempty);
          }
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int64_t m = tl.m0 + 32 * c + j;
            if (m < a.M && n < a.N) {
              const int sft = __ldg(a.shift + m);
              const float scale = __int_as_float((127 - sft) << 23);   // 2^-s, s in [-64, 64]
              y[m * a.N + n] = __fmul_rn(__uint_as_float(v[j]), scale);
            }
          }
        }
      }
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, static_cast<uint32_t>(kTmemCols));
  }
}

// --------------------------------------------------- activation rounding --
// One CTA per activation row: row max -> shift s (max |x| * 2^s in
// [2^14, 2^15), 0 for a zero row, clamped to [-64, 64]) -> binary16 RNE of
// x * 2^s (an exact scaling unless the product is an fp32 subnormal).
// BLOCKED = true writes the tile-major layout the MMA reads, so the
// activations of one token tile for one 256-element unit of K are a single
// contiguous block (one bulk copy): for token tile mt = m / tn, unit ub and
// 64-element sub-block kb4, the 128 bytes of row m start at
//   (((mt * units + ub) * 4 + kb4) * tn + m % tn) * 128,
// and inside them the 16-byte chunk c sits at position c ^ (m & 7) (the
// 128-byte swizzle).  BLOCKED = false writes plain row-major [M][K].  Rows
// m >= M (padding up to whole token tiles) are written as zeros.
template <bool BLOCKED>
__global__ void __launch_bounds__(256) x_to_f16_kernel(const float *__restrict__ x, int64_t M, int64_t K,
                                                       int64_t tn, __half *__restrict__ x16,
                                                       int32_t *__restrict__ shift) {
  __shared__ float red[8];
  pdl_trigger();
  pdl_wait();
  const int64_t m = blockIdx.x;
  const int64_t nchunks = K / 8;   // 16-byte chunks of 8 halves per row
  const int64_t units = K / 256;
  auto chunk_ptr = [&](int64_t c) -> uint4 * {
    if (BLOCKED) {
      const int64_t kb = c / 8, cc = c % 8;
      const int64_t off = ((((m / tn) * units + kb / 4) * 4 + kb % 4) * tn + m % tn) * 128 + ((cc ^ (m & 7)) << 4);
      return reinterpret_cast<uint4 *>(reinterpret_cast<uint8_t *>(x16) + off);
    }
    return reinterpret_cast<uint4 *>(x16 + m * K) + c;
  };
  if (m >= M) {
    for (int64_t c = threadIdx.x; c < nchunks; c += blockDim.x) *chunk_ptr(c) = make_uint4(0u, 0u, 0u, 0u);
    if (threadIdx.x == 0) shift[m] = 0;
    return;
  }
  const float4 *row = reinterpret_cast<const float4 *>(x + m * K);
  const int64_t nv = K / 4;
  float amax = 0.0f;
  for (int64_t i = threadIdx.x; i < nv; i += blockDim.x) {
    const float4 v = __ldg(row + i);
    amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) amax = fmaxf(amax, red[i]);
  int s = 0;
  if (amax > 0.0f && !isinf(amax)) {
    int e;
    frexpf(amax, &e);
    s = min(64, max(-64, 15 - e));
  }
  const float scale = __int_as_float((127 + s) << 23);
  if (threadIdx.x == 0) shift[m] = s;
  for (int64_t c = threadIdx.x; c < nchunks; c += blockDim.x) {
    const float4 a = __ldg(row + 2 * c), b = __ldg(row + 2 * c + 1);
    const __half2 h0 = __floats2half2_rn(__fmul_rn(a.x, scale), __fmul_rn(a.y, scale));
    const __half2 h1 = __floats2half2_rn(__fmul_rn(a.z, scale), __fmul_rn(a.w, scale));
    const __half2 h2 = __floats2half2_rn(__fmul_rn(b.x, scale), __fmul_rn(b.y, scale));
    const __half2 h3 = __floats2half2_rn(__fmul_rn(b.z, scale), __fmul_rn(b.w, scale));
    *chunk_ptr(c) = make_uint4(h2_bits(h0), h2_bits(h1), h2_bits(h2), h2_bits(h3));
  }
}

// Split-K partials -> output, summed in split order (deterministic).
__global__ void __launch_bounds__(256) splitk_reduce_kernel(const float *__restrict__ part, int64_t total, int splits,
                                                            float *__restrict__ y) {
  pdl_trigger();
  pdl_wait();
  const int64_t n4 = total / 4;
  const float4 *p4 = reinterpret_cast<const float4 *>(part);
  float4 *y4 = reinterpret_cast<float4 *>(y);
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4; i += stride) {
    float4 acc = __ldg(p4 + i);
    for (int s = 1; s < splits; ++s) {
      const float4 v = __ldg(p4 + static_cast<int64_t>(s) * n4 + i);
      acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
    y4[i] = acc;
  }
  for (int64_t i = 4 * n4 + static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride) {
    float acc = part[i];
    for (int s = 1; s < splits; ++s) acc += part[static_cast<int64_t>(s) * total + i];
    y[i] = acc;
  }
}

// Test hook: the whole dequantized weight matrix in binary16, produced by the
// same device functions as the GEMM's converter warps.
template <int TYPE>
__global__ void __launch_bounds__(128) w_to_f16_kernel(const uint8_t *__restrict__ w, int64_t N, int64_t K,
                                                       int64_t row_bytes, uint16_t *__restrict__ w16) {
  const int64_t units = K / 256;
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= N * units) return;
  const int64_t n = idx / units, u = idx % units;
  RawUnit<TYPE> ru;
  load_unit<TYPE>(ru, w + n * row_bytes + u * (TYPE == DSQ_Q8_0 ? 272 : 144));
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    uint32_t v[32];
    dequant_piece<TYPE>(ru, p, v);
    uint4 *dst = reinterpret_cast<uint4 *>(w16 + n * K + u * 256 + p * 64);
#pragma unroll
    for (int c = 0; c < 8; ++c) dst[c] = make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
  }
}

// ------------------------------------------------------------------- host --
struct Plan {
  int tn, groups_b, stages_a, raw_slots, splits, units_per_split;
  int64_t tiles_m, tiles_n, total_tiles, m_pad;
  unsigned grid;
  size_t smem, x16_bytes, shift_off, part_off, total;
};

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

constexpr size_t kSmemLimit = 227 * 1024;

Plan make_plan(int type, int64_t N, int64_t K, int64_t M, int num_sms) {
  Plan p{};
  const int64_t tiles_n = (N + kTileN - 1) / kTileN;
  // tokens per tile: the smallest multiple of 32 that covers M, at most 128
  // (TMEM holds 2 x tn accumulator columns plus the weight stages, so tn <= 128)
  p.tn = M <= 128 ? static_cast<int>((M + 31) / 32 * 32) : 128;
  p.tiles_m = (M + p.tn - 1) / p.tn;
  p.tiles_n = tiles_n;
  const int units = static_cast<int>(K / 256);
  const int64_t tiles = p.tiles_m * p.tiles_n;
  // split K only when the tiles leave more than half the SMs idle
  p.splits = 1;
  while (tiles * p.splits * 2 <= num_sms && p.splits * 2 <= 16 && p.splits * 2 <= units) p.splits *= 2;
  p.units_per_split = (units + p.splits - 1) / p.splits;
  p.splits = (units + p.units_per_split - 1) / p.units_per_split;
  p.total_tiles = tiles * p.splits;
  p.grid = static_cast<unsigned>(p.total_tiles < num_sms ? p.total_tiles : num_sms);
  // TMEM: the accumulators (2 halves x tn fp32 columns), then as many
  // 64-column weight stages as fit (at most 6)
  p.stages_a = (kTmemCols - kHalves * p.tn) / kAColsStage;
  if (p.stages_a > 6) p.stages_a = 6;
  // shared memory: raw weight slots (one 256-element unit of the tile's 256
  // rows each; two when they fit, else one) and activation slots (one unit
  // of K each; two or more)
  const int group_bytes = 4 * p.tn * 128;
  const int raw_bytes = kTileN * (type == DSQ_Q8_0 ? 272 : 144);
  const size_t fixed = 1024 + 512;
  p.raw_slots = (fixed + 2 * static_cast<size_t>(raw_bytes) + 2 * group_bytes <= kSmemLimit) ? 2 : 1;
  p.groups_b = static_cast<int>((kSmemLimit - fixed - static_cast<size_t>(p.raw_slots) * raw_bytes) / group_bytes);
  if (p.groups_b > 6) p.groups_b = 6;
  p.smem = 1024 + static_cast<size_t>(p.groups_b) * group_bytes + static_cast<size_t>(p.raw_slots) * raw_bytes +
           (2 * p.groups_b + 2 * p.stages_a + 2 * p.raw_slots + 3) * sizeof(uint64_t) + 16;
  // the fp16 activation buffer is padded with zero rows to whole token tiles
  p.m_pad = p.tiles_m * p.tn;
  p.x16_bytes = align_up(static_cast<size_t>(p.m_pad) * K * 2, 1024);
  p.shift_off = p.x16_bytes;
  p.part_off = align_up(p.shift_off + static_cast<size_t>(p.m_pad) * 4, 1024);
  p.total = p.part_off + (p.splits > 1 ? static_cast<size_t>(p.splits) * M * N * 4 : 0);
  return p;
}

int validate(const char *name, int type, const void *w, int64_t N, int64_t K, const float *x, int64_t M) {
  DSQ_REQUIRE(type == DSQ_Q8_0 || type == DSQ_Q4_K, DSQ_ERR_INVALID_ARG, "%s: unsupported type %d", name, type);
  DSQ_REQUIRE(N >= 1 && M >= 1 && K >= 1, DSQ_ERR_INVALID_ARG, "%s: N, M, K must be >= 1", name);
  DSQ_REQUIRE(K % 256 == 0, DSQ_ERR_SHAPE, "%s: K=%lld must be a multiple of 256", name, (long long)K);
  DSQ_REQUIRE(K <= 65536 && N <= (int64_t(1) << 24) && M <= (int64_t(1) << 24), DSQ_ERR_SHAPE,
              "%s: size out of range (K <= 65536, M, N <= 2^24)", name);
  DSQ_REQUIRE(w && x, DSQ_ERR_INVALID_ARG, "%s: null pointer", name);
  DSQ_REQUIRE(aligned(w, 16) && aligned(x, 16), DSQ_ERR_ALIGNMENT, "%s: w and x must be 16-byte aligned", name);
  return DSQ_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

template <int TYPE>
int launch_gemm(const CUtensorMap &map_w, const PrefillArgs &args, const Plan &p, cudaStream_t stream) {
  auto kern = prefill_kernel<TYPE>;
  const int rc = set_smem_once(reinterpret_cast<const void *>(kern), static_cast<int>(p.smem), "prefill");
  if (rc != DSQ_OK) return rc;
  // ask for no more shared-memory carveout than the kernel uses: the rest is L1
  const int carve = static_cast<int>((p.smem * 100 + 228 * 1024 - 1) / (228 * 1024));
  cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, carve);
  const cudaError_t e = launch_pdl(kern, dim3(p.grid), dim3(kThreads), p.smem, stream, map_w, args);
  if (e != cudaSuccess) return fail(DSQ_ERR_LAUNCH, "dsq_gemm_prefill: gemm: %s", cudaGetErrorString(e));
  return after_launch("dsq_gemm_prefill: gemm");
}

}  // namespace
}  // namespace dsq

extern "C" size_t dsq_prefill_workspace_bytes(int type, int64_t N, int64_t K, int64_t M) {
  using namespace dsq;
  if ((type != DSQ_Q8_0 && type != DSQ_Q4_K) || N < 1 || M < 1 || K < 256 || K % 256 != 0) return 0;
  int sms = 148;
  if (device_ready(nullptr, &sms) != DSQ_OK) sms = 148;
  return make_plan(type, N, K, M, sms).total;
}

extern "C" int dsq_gemm_prefill(int type, const void *w, int64_t N, int64_t K, const float *x, int64_t M, float *y,
                                void *workspace, size_t workspace_bytes, void *stream) {
  using namespace dsq;
  int rc = validate("dsq_gemm_prefill", type, w, N, K, x, M);
  if (rc != DSQ_OK) return rc;
  DSQ_REQUIRE(y != nullptr, DSQ_ERR_INVALID_ARG, "dsq_gemm_prefill: null output");
  DSQ_REQUIRE(aligned(y, 16), DSQ_ERR_ALIGNMENT, "dsq_gemm_prefill: y must be 16-byte aligned");
  WaitCtl ctl;
  int sms = 0;
  rc = wait_ctl(&ctl, &sms);
  if (rc != DSQ_OK) return rc;
  const Plan p = make_plan(type, N, K, M, sms);
  DSQ_REQUIRE(workspace != nullptr && workspace_bytes >= p.total, DSQ_ERR_WORKSPACE,
              "dsq_gemm_prefill: workspace of %zu bytes needed, %zu given", p.total, workspace_bytes);
  DSQ_REQUIRE(aligned(workspace, 256), DSQ_ERR_ALIGNMENT, "dsq_gemm_prefill: workspace must be 256-byte aligned");
  DSQ_REQUIRE(p.smem <= kSmemLimit && p.groups_b >= 2 && p.stages_a >= 2 && p.raw_slots >= 1, DSQ_ERR_SHAPE,
              "dsq_gemm_prefill: no pipeline fits");

  uint8_t *ws = static_cast<uint8_t *>(workspace);
  __half *x16 = reinterpret_cast<__half *>(ws);
  int32_t *shift = reinterpret_cast<int32_t *>(ws + p.shift_off);
  float *part = reinterpret_cast<float *>(ws + p.part_off);

  // raw weight units: the packed rows viewed as uint32 [N][row_bytes/4], one
  // 256-element unit (68 or 36 words) x 128 rows per box; rows past N read as
  // zero (a zero block dequantizes to zero)
  auto enc = encode_fn();
  DSQ_REQUIRE(enc != nullptr, DSQ_ERR_CUDA, "dsq_gemm_prefill: cuTensorMapEncodeTiled unavailable");
  CUtensorMap map_w;
  {
    const int64_t rb = static_cast<int64_t>(dsq_row_bytes(type, K));
    const cuuint32_t unit_words = type == DSQ_Q8_0 ? 68u : 36u;
    const cuuint64_t gdim[2] = {static_cast<cuuint64_t>(rb / 4), static_cast<cuuint64_t>(N)};
    const cuuint64_t gstride[1] = {static_cast<cuuint64_t>(rb)};
    const cuuint32_t box[2] = {unit_words, static_cast<cuuint32_t>(kBM)};
    const cuuint32_t estride[2] = {1u, 1u};
    const CUresult cr = enc(&map_w, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void *>(w), gdim, gstride, box,
                            estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    DSQ_REQUIRE(cr == CUDA_SUCCESS, DSQ_ERR_CUDA, "dsq_gemm_prefill: weight tensor map (%d)", (int)cr);
  }
  cudaStream_t st = as_stream(stream);
  cudaError_t e = launch_pdl(x_to_f16_kernel<true>, dim3(static_cast<unsigned>(p.m_pad)), dim3(256), 0, st, x, M, K,
                             static_cast<int64_t>(p.tn), x16, shift);
  if (e != cudaSuccess) return fail(DSQ_ERR_LAUNCH, "dsq_gemm_prefill: x_to_f16: %s", cudaGetErrorString(e));
  rc = after_launch("dsq_gemm_prefill: x_to_f16");
  if (rc != DSQ_OK) return rc;

  PrefillArgs args{};
  args.w = static_cast<const uint8_t *>(w);
  args.row_bytes = static_cast<int64_t>(dsq_row_bytes(type, K));
  args.N = N;
  args.K = K;
  args.M = M;
  args.x16 = x16;
  args.shift = shift;
  args.y = p.splits > 1 ? part : y;
  args.units_per_split = p.units_per_split;
  args.splits = p.splits;
  args.tn = p.tn;
  args.groups_b = p.groups_b;
  args.raw_slots = p.raw_slots;
  args.stages_a = p.stages_a;
  args.tiles_m = p.tiles_m;
  args.tiles_n = p.tiles_n;
  args.total_tiles = p.total_tiles;
  args.wait = ctl;
  rc = type == DSQ_Q8_0 ? launch_gemm<DSQ_Q8_0>(map_w, args, p, st) : launch_gemm<DSQ_Q4_K>(map_w, args, p, st);
  if (rc != DSQ_OK) return rc;
  if (p.splits > 1) {
    const int64_t total = M * N;
    const int64_t blocks = (total / 4 + 255) / 256 + 1;
    const unsigned grid = static_cast<unsigned>(blocks < 8 * sms ? blocks : 8 * sms);
    e = launch_pdl(splitk_reduce_kernel, dim3(grid), dim3(256), 0, st, static_cast<const float *>(part), total,
                   p.splits, y);
    if (e != cudaSuccess) return fail(DSQ_ERR_LAUNCH, "dsq_gemm_prefill: reduce: %s", cudaGetErrorString(e));
    rc = after_launch("dsq_gemm_prefill: split-k reduce");
  }
  return rc;
}

extern "C" int dsq_test_prefill_operands(int type, const void *w, int64_t N, int64_t K, const float *x, int64_t M,
                                         uint16_t *x16, int32_t *shift, uint16_t *w16, void *stream) {
  using namespace dsq;
  int rc = validate("dsq_test_prefill_operands", type, w, N, K, x, M);
  if (rc != DSQ_OK) return rc;
  DSQ_REQUIRE(x16 && shift && w16, DSQ_ERR_INVALID_ARG, "dsq_test_prefill_operands: null output");
  DSQ_REQUIRE(aligned(x16, 16) && aligned(w16, 16) && aligned(shift, 4), DSQ_ERR_ALIGNMENT,
              "dsq_test_prefill_operands: output alignment");
  rc = device_ready(nullptr, nullptr);
  if (rc != DSQ_OK) return rc;
  cudaStream_t st = as_stream(stream);
  x_to_f16_kernel<false><<<static_cast<unsigned>(M), 256, 0, st>>>(x, M, K, M, reinterpret_cast<__half *>(x16), shift);
  rc = after_launch("dsq_test_prefill_operands: x");
  if (rc != DSQ_OK) return rc;
  const int64_t work = N * (K / 256);
  const unsigned grid = static_cast<unsigned>((work + 127) / 128);
  const int64_t rb = static_cast<int64_t>(dsq_row_bytes(type, K));
  if (type == DSQ_Q8_0)
    w_to_f16_kernel<DSQ_Q8_0><<<grid, 128, 0, st>>>(static_cast<const uint8_t *>(w), N, K, rb, w16);
  else
    w_to_f16_kernel<DSQ_Q4_K><<<grid, 128, 0, st>>>(static_cast<const uint8_t *>(w), N, K, rb, w16);
  return after_launch("dsq_test_prefill_operands: w");
}

// ------------------------------------------------ allocation-free variant --
// Scratch for dsq_gemm_prefill_noalloc: a fixed array in device global
// memory, reserved once per device when the module loads (every device that
// loads the library holds these 32 MiB until the process exits).  The
// prefill kernels write every byte of it they later read in the same call,
// so nothing has to be cleared between calls.
static __device__ __align__(256) uint8_t g_prefill_scratch[DSQ_PREFILL_NOALLOC_SCRATCH_BYTES];

namespace dsq {
namespace {
std::mutex g_scratch_mu;
void *g_scratch_addr[64] = {};   // device address of g_prefill_scratch, per device
}  // namespace
}  // namespace dsq

extern "C" int dsq_gemm_prefill_noalloc(int type, const void *w, int64_t N, int64_t K, const float *x, int64_t M,
                                        float *y, void *stream) {
  using namespace dsq;
  const size_t need = dsq_prefill_workspace_bytes(type, N, K, M);
  if (need == 0)  // invalid type or shape: let the regular entry point name it
    return dsq_gemm_prefill(type, w, N, K, x, M, y, nullptr, 0, stream);
  DSQ_REQUIRE(need <= DSQ_PREFILL_NOALLOC_SCRATCH_BYTES, DSQ_ERR_WORKSPACE,
              "dsq_gemm_prefill_noalloc: this problem needs %zu bytes of scratch but the built-in scratch holds "
              "%llu bytes (M x K x 2 bytes of fp16 activations plus split-K partials must fit); use "
              "dsq_gemm_prefill with a caller-provided workspace",
              need, (unsigned long long)DSQ_PREFILL_NOALLOC_SCRATCH_BYTES);
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  DSQ_REQUIRE(e == cudaSuccess && dev >= 0 && dev < 64, DSQ_ERR_CUDA, "dsq_gemm_prefill_noalloc: no current device");
  void *scratch = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (g_scratch_addr[dev] == nullptr) {
      // One-time set-up on this device (the device is current): the host
      // name of the array is only a stand-in, so fetch its device address.
      void *p = nullptr;
      e = cudaGetSymbolAddress(&p, g_prefill_scratch);
      DSQ_REQUIRE(e == cudaSuccess && p != nullptr, DSQ_ERR_CUDA,
                  "dsq_gemm_prefill_noalloc: cudaGetSymbolAddress of the scratch failed: %s", cudaGetErrorString(e));
      g_scratch_addr[dev] = p;
    }
    scratch = g_scratch_addr[dev];
  }
  return dsq_gemm_prefill(type, w, N, K, x, M, y, scratch, static_cast<size_t>(DSQ_PREFILL_NOALLOC_SCRATCH_BYTES),
                          stream);
}
