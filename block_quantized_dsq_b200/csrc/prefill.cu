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
// GEMM kernel: persistent clusters of two CTAs (one per SM) sharing one
// tcgen05 MMA of M = 256 weight rows (cta_group::2).  A pair tile is 256
// weight rows x tn tokens x one K split; CTA r of the pair owns weight rows
// 128r..128r+127 and holds tokens r*tn/2 .. r*tn/2 + tn/2 - 1 of the tile:
//  * the dequantized weights are the MMA's A operand and live in TMEM (each
//    CTA's 128 lanes = its 128 rows), the activations are the B operand in
//    shared memory (each CTA holds half of the N = tn columns);  "swap AB"
//    keeps small token counts on full 128-lane MMAs;
//  * the pipeline runs in slots of one stage pair (2 x 64 K): per CTA, warp 0
//    copies the slot's activations (one bulk copy of a tile-major fp16
//    layout), warp 14 streams raw weight units (TMA, 128 rows x 256 K), warps
//    2-9 dequantize (thread = weight row; warps 2-5 the first stage pair of
//    each unit, 6-9 the second) into the slot's TMEM columns, warps 10-13
//    drain the fp32 accumulators (tcgen05.ld -> scale by 2^-s_m -> global);
//  * warp 1 of the even CTA issues the pair MMAs: one wait on the slot's
//    ready barrier and one multicast tcgen05.commit to both CTAs' consumed
//    barrier per 8 MMAs (the tcgen05 issue queue is shallow); warp 1 of the
//    odd CTA forwards "activation slot landed" to the even CTA;
//  * every wait is bounded; an expired wait records a timeout, raises the
//    abort flag of both CTAs, drains copies and MMAs in flight, and the pair
//    meets at a final cluster barrier before TMEM is freed.
#include <cudaTypedefs.h>
#include <mutex>

#include "../../include/dsq_test.h"
#include "dsq_host.h"

namespace dsq {
namespace {

constexpr int kRows = 128;          // weight rows per CTA (TMEM lanes)
constexpr int kTileN = 2 * kRows;   // weight rows per pair tile (the MMA's M)
constexpr int kBK = 64;             // K elements per pipeline stage
constexpr int kAColsStage = kBK / 2;   // TMEM columns of one A stage (2 fp16 per column)
constexpr int kAColsSlot = 2 * kAColsStage;   // an A slot holds 2 consecutive stages
constexpr int kTmemCols = 512;      // the CTA owns all of TMEM (1 CTA per SM)
constexpr int kMaxSlots = 6;
// warp roles
constexpr int kWarpX = 0;         // bulk-copy producer: fp16 activation stages
constexpr int kWarpMma = 1;       // TMEM owner; MMA issuer (even CTA) / activation relay (odd CTA)
constexpr int kWarpConv0 = 2;     // warps 2..9: dequantize into TMEM
constexpr int kConvWarps = 8;
constexpr int kWarpEpi0 = kWarpConv0 + kConvWarps;   // warps 10..13: TMEM -> global epilogue
constexpr int kWarpW = kWarpEpi0 + 4;                 // warp 14: TMA producer of raw weight units
constexpr int kThreads = (kWarpW + 1) * 32;
constexpr int kMaxGroup = DSQ_PREFILL_MAX_GROUP;   // weights sharing X in one launch

// The weights' tensor maps (one per weight; unused entries repeat entry 0).
struct WeightMaps {
  CUtensorMap m[kMaxGroup];
};

struct PrefillArgs {
  int64_t K, M;
  int G;                  // weights that share X
  int64_t N[kMaxGroup];   // rows of each weight
  float *y[kMaxGroup];    // [M][N_g] outputs, or [splits] x split_stride partials
  int64_t split_stride[kMaxGroup];   // floats between two splits' partials (a multiple of 4)
  int64_t tile_n0[kMaxGroup + 1];    // first 256-row tile of each weight in the tile order
  const __half *x16;      // fp16 activations, tile-major and swizzled (see x_to_f16_kernel)
  const int32_t *shift;   // [M] activation row shifts
  int units_per_split;    // 256-element units of K per split
  int splits;
  // Last-wave split: when the pair tiles fill whole waves and a short last
  // one, that last wave's tail_tiles tiles are split tail_splits ways in K
  // (tail_ups units each) into pieces that follow the head_tiles unsplit
  // tiles; piece j + s * tail_tiles (split s of tail tile j) writes its
  // partial to tail_part + (j + s * tail_tiles) * tn * 256, token-major
  // (token * 256 + row), and tail_reduce_kernel sums the splits in order.
  // head_tiles = total_tiles when nothing is split this way.
  int64_t head_tiles;
  int tail_tiles, tail_splits, tail_ups;
  float *tail_part;
  int tn;                 // tokens per pair tile (MMA N): 32..256, multiple of 32
  int slots;              // pipeline slots: one stage pair each, activations in shared memory
                          // (2 x 64 K x tn/2 tokens) and dequantized weights in TMEM (64 columns); even
  int slots_raw;          // raw weight unit slots in shared memory (128 rows x 256 K each)
  int64_t tiles_m, tiles_n, total_tiles;
  WaitCtl wait;
};

// ---------------------------------------------------------------- dequant --
template <int TYPE> __host__ __device__ constexpr int unit_bytes() { return TYPE == DSQ_Q8_0 ? 272 : 144; }

__device__ __forceinline__ uint32_t h2_bits(__half2 h) { return *reinterpret_cast<uint32_t *>(&h); }
__device__ __forceinline__ __half2 bits_h2(uint32_t b) { return *reinterpret_cast<__half2 *>(&b); }

__device__ __forceinline__ uint32_t word4(const uint4 &v, int i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

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

// Q8_0: one 64-element piece = two blocks = 68 bytes = 17 words starting
// word-aligned (a piece starts at byte 68p of its 256-element unit).
// word(i), i = 0..16, returns the piece's i-th word.  Block 0: fp16 d in the
// low half of word 0, codes in bytes 2..33; block 1: d in the high half of
// word 8, codes in words 9..16.  Output: 8 chunks of 8 halves.
template <class Word>
__device__ __forceinline__ void piece_q8_0(Word word, uint32_t (&out)[32]) {
  {
    const __half2 d2 = __half2half2(__ushort_as_half(static_cast<unsigned short>(word(0) & 0xffffu)));
#pragma unroll
    for (int i = 0; i < 8; ++i)
      q8x4_to_h(__funnelshift_r(word(i), word(i + 1), 16), d2, out[2 * i], out[2 * i + 1]);
  }
  {
    const __half2 d2 = __half2half2(__ushort_as_half(static_cast<unsigned short>(word(8) >> 16)));
#pragma unroll
    for (int i = 0; i < 8; ++i) q8x4_to_h(word(9 + i), d2, out[16 + 2 * i], out[16 + 2 * i + 1]);
  }
}

// Q4_K: piece P (64 elements = sub-blocks 2P (low nibbles) and 2P+1 (high
// nibbles) of bytes qs[32P .. 32P+31]).  hdr = the super-block's first 16
// bytes (fp16 d, fp16 dmin, 12 bytes of packed 6-bit scales and mins);
// nib(i), i = 0..7, returns word i of qs[32P ..].  Each value is fp32
// (d*sc)*q - dmin*m (one rounding: (d*sc)*q and dmin*m are exact), then
// binary16 RNE.
// Paired fp32 arithmetic (sm_100): two independent IEEE single operations per
// instruction, lane 0 in the low 32 bits.
__device__ __forceinline__ uint64_t pack2(float lo, float hi) {
  return static_cast<uint64_t>(__float_as_uint(lo)) | (static_cast<uint64_t>(__float_as_uint(hi)) << 32);
}
__device__ __forceinline__ float lo_of(uint64_t v) { return __uint_as_float(static_cast<uint32_t>(v)); }
__device__ __forceinline__ float hi_of(uint64_t v) { return __uint_as_float(static_cast<uint32_t>(v >> 32)); }
__device__ __forceinline__ uint64_t sub2_rn(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t fma2_rn(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
constexpr uint64_t kMagic2 = 0x4B0000004B000000ull;   // (2^23, 2^23)

template <int P, class Nib>
__device__ __forceinline__ void piece_q4_k(const uint4 &hdr, Nib nib, uint32_t (&out)[32]) {
  const float d = __half2float(__ushort_as_half(static_cast<unsigned short>(hdr.x & 0xffffu)));
  const float dmin = __half2float(__ushort_as_half(static_cast<unsigned short>(hdr.x >> 16)));
  const uint32_t s0 = hdr.y, s1 = hdr.z, s2 = hdr.w;
#pragma unroll
  for (int half_ = 0; half_ < 2; ++half_) {
    const int j = 2 * P + half_;
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
    const uint64_t a2 = pack2(a, a), nb2 = pack2(nb, nb);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t byte4 = nib(i);
      const uint32_t q4 = half_ ? ((byte4 >> 4) & 0x0f0f0f0fu) : (byte4 & 0x0f0f0f0fu);
#pragma unroll
      for (int e = 0; e < 4; e += 2) {
        // 0x4B000000 | q is the float 2^23 + q; subtracting 2^23 is exact.
        // Two elements per paired-fp32 instruction, each rounded as its
        // own __fsub_rn / __fmaf_rn would be.
        const uint64_t f2 = pack2(__uint_as_float(__byte_perm(q4, 0x4B000000u, 0x7540 + e)),
                                  __uint_as_float(__byte_perm(q4, 0x4B000000u, 0x7540 + e + 1)));
        const uint64_t v2 = fma2_rn(sub2_rn(f2, kMagic2), a2, nb2);
        out[16 * half_ + 2 * i + e / 2] = h2_bits(__floats2half2_rn(lo_of(v2), hi_of(v2)));
      }
    }
  }
}

// The registers a converter thread loads for stage pair J of a unit
// (stages 2J and 2J+1 = pieces 2J, 2J+1; uint4 granules of the row's
// 256-element unit) and the dequantization of piece 2J + i from them.
// Q8_0: granules 8J .. 8J+8 (144 bytes covering the pair's 136, piece P
// starting at word 17P - 32J of them).  Q4_K: granule 0 (header) and
// 1+4J .. 4+4J (the pair's 64 nibble bytes).
template <int TYPE> struct PairRegs;
template <> struct PairRegs<DSQ_Q8_0> { uint4 v[9]; };
template <> struct PairRegs<DSQ_Q4_K> { uint4 hdr, v[4]; };

template <int TYPE, int J>
__device__ __forceinline__ void load_pair(PairRegs<TYPE> &r, const uint4 *unit) {
  if constexpr (TYPE == DSQ_Q8_0) {
#pragma unroll
    for (int i = 0; i < 9; ++i) r.v[i] = unit[8 * J + i];
  } else {
    r.hdr = unit[0];
#pragma unroll
    for (int i = 0; i < 4; ++i) r.v[i] = unit[1 + 4 * J + i];
  }
}

template <int TYPE, int J, int I>
__device__ __forceinline__ void dequant_pair_piece(const PairRegs<TYPE> &r, uint32_t (&out)[32]) {
  constexpr int P = 2 * J + I;
  if constexpr (TYPE == DSQ_Q8_0) {
    constexpr int o = 17 * P - 32 * J;
    piece_q8_0([&](int i) { return word4(r.v[(o + i) >> 2], (o + i) & 3); }, out);
  } else {
    piece_q4_k<P>(r.hdr, [&](int i) { return word4(r.v[2 * I + (i >> 2)], i & 3); }, out);
  }
}

// Range guard of the binary16 weight operand: false when a block this thread
// dequantizes for stage pair J admits a value of magnitude >= 65520, which
// rounds to +-inf in binary16.  Q8_0 (blocks 4J .. 4J+3 of the unit): |d| *
// 127 >= 65520, i.e. |d| >= 516 (binary16 bits 0x6008), or a non-finite d.
// Q4_K (sub-blocks 4J .. 4J+3): the dequantized value is a line in the code
// q, so its extremes are the codes 0 and 15: -dmin*m and 15*(d*sc) - dmin*m,
// formed in fp32 exactly as the converter forms them.  A cheap bound on the
// whole super-block (|d|*63*15 + |dmin|*63 < 65520) settles almost every
// block before the per-sub-block test.
template <int TYPE, int J>
__device__ __forceinline__ bool pair_in_range(const PairRegs<TYPE> &r) {
  if constexpr (TYPE == DSQ_Q8_0) {
    uint32_t worst = 0;
#pragma unroll
    for (int I = 0; I < 2; ++I) {
      const int o = 17 * (2 * J + I) - 32 * J;   // first word of piece 2J + I
      const uint32_t d0 = word4(r.v[o >> 2], o & 3) & 0x7fffu;
      const uint32_t d1 = (word4(r.v[(o + 8) >> 2], (o + 8) & 3) >> 16) & 0x7fffu;
      worst = max(worst, max(d0, d1));
    }
    return worst < 0x6008u;
  } else {
    const float d = fabsf(__half2float(__ushort_as_half(static_cast<unsigned short>(r.hdr.x & 0xffffu))));
    const float dmin = fabsf(__half2float(__ushort_as_half(static_cast<unsigned short>(r.hdr.x >> 16))));
    if (__fadd_rn(__fmul_rn(d, 945.0f), __fmul_rn(dmin, 63.0f)) < 65520.0f) return true;
    const float ds = __half2float(__ushort_as_half(static_cast<unsigned short>(r.hdr.x & 0xffffu)));
    const float dm = __half2float(__ushort_as_half(static_cast<unsigned short>(r.hdr.x >> 16)));
    bool ok = true;
#pragma unroll
    for (int j = 4 * J; j < 4 * J + 4; ++j) {
      uint32_t scw, mw;
      if (j < 4) {
        scw = r.hdr.y & 0x3f3f3f3fu;
        mw = r.hdr.z & 0x3f3f3f3fu;
      } else {
        scw = (r.hdr.w & 0x0f0f0f0fu) | ((r.hdr.y >> 2) & 0x30303030u);
        mw = ((r.hdr.w >> 4) & 0x0f0f0f0fu) | ((r.hdr.z >> 2) & 0x30303030u);
      }
      const int sh = 8 * (j & 3);
      const float a = __fmul_rn(ds, static_cast<float>((scw >> sh) & 0xffu));
      const float b = __fmul_rn(dm, static_cast<float>((mw >> sh) & 0xffu));
      const float v15 = __fmaf_rn(15.0f, a, -b);
      ok = ok && fabsf(b) < 65520.0f && fabsf(v15) < 65520.0f;
    }
    return ok;
  }
}

__device__ __forceinline__ void record_range(uint32_t *status) { atomicOr(status, kStatusRange); }

// ------------------------------------------------------------------ GEMM ---
// TMEM map of each CTA (512 columns x 128 lanes): [0, tn) the fp32
// accumulators (lane = weight row of this CTA, column = token of the pair
// tile); then the dequantized-weight halves of the pipeline slots, 2 stages = 64 columns each (lane =
// weight row, each column two consecutive fp16 K elements).
struct Smem {
  uint8_t *b;          // slots x 2 stages x (tn/2 rows x 128 B): activation stages (MMA B, this CTA's half)
  uint8_t *raw;        // slots_raw x 128 rows x unit bytes: raw weight units (TMA)
  uint64_t *ready;     // slot filled.  Even CTA: its activation copy (1 + tx), the odd CTA's forwarded
                       // copy arrival (1) and the 4 converter warps of the slot in each CTA (8).
                       // Odd CTA: its activation copy only (1 + tx), forwarded by its warp 1.
  uint64_t *consumed;  // pair MMAs finished reading a slot (multicast commit to both CTAs)
  uint64_t *rfull;     // raw unit landed (1 + tx)
  uint64_t *rempty;    // converters copied a raw unit into registers (8 warps)
  uint64_t *accfull;   // accumulators complete (multicast commit)
  uint64_t *accempty;  // even CTA: both epilogues drained the accumulators (8 warp arrivals)
  uint64_t *drain;     // even CTA: MMA drain after an abort
  uint32_t *tmem;      // TMEM base address
  volatile uint32_t *abort;
};

__device__ __forceinline__ Smem carve(uint8_t *base, int slots, uint32_t slot_b_bytes, int slots_raw,
                                      uint32_t raw_bytes) {
  Smem s;
  s.b = base;
  s.raw = s.b + static_cast<size_t>(slots) * slot_b_bytes;
  uint64_t *p = reinterpret_cast<uint64_t *>(s.raw + static_cast<size_t>(slots_raw) * raw_bytes);
  s.ready = p;
  s.consumed = s.ready + slots;
  s.rfull = s.consumed + slots;
  s.rempty = s.rfull + slots_raw;
  s.accfull = s.rempty + slots_raw;
  s.accempty = s.accfull + 1;
  s.drain = s.accempty + 1;
  s.tmem = reinterpret_cast<uint32_t *>(s.drain + 1);
  s.abort = reinterpret_cast<volatile uint32_t *>(s.tmem + 1);
  return s;
}
__host__ __device__ constexpr size_t barrier_bytes(int slots, int slots_raw) {
  return (2 * static_cast<size_t>(slots) + 2 * slots_raw + 3) * sizeof(uint64_t) + 16;
}

__device__ __forceinline__ bool aborted(const Smem &s) { return *s.abort != 0; }
// Raise the abort flag of both CTAs of the pair.
__device__ __forceinline__ void set_abort(const Smem &s, const WaitCtl &w) {
  *s.abort = 1u;
  st_shared_remote_u32(mapa_shared(smem_u32(const_cast<uint32_t *>(s.abort)), cluster_ctarank() ^ 1u), 1u);
  record_timeout(w);
}

// One thread's bounded wait; on expiry (or an abort raised elsewhere) it
// raises the pair's abort flag and returns false.
// sleep_ns: poll back-off for waiters off the critical path.
__device__ __forceinline__ bool wait_or_abort(const Smem &s, uint64_t *bar, uint32_t parity, const WaitCtl &w,
                                              uint32_t sleep_ns = 0) {
  if (mbar_try_wait(bar, parity)) return true;   // fast path: already complete
  if (aborted(s)) return false;
  if (mbar_wait_for(bar, parity, w.limit_ns, sleep_ns)) return true;
  set_abort(s, w);
  return false;
}

// Pair tile t -> (token tile, first weight row, K split); consecutive tiles
// share a weight tile, so pairs running side by side reuse it from L2.  The
// tile walks its K units [u0, u1) cyclically from u0 + rot: pairs that run
// at the same time on the same activation tile (other weight rows) or the
// same weight tile (other tokens) then read different units instead of the
// same lines at the same moment.
// The weight-row tiles of the G weights follow one another in the tile
// order; g is the tile's weight and n0 its first row within that weight.  The
// K rotation depends only on the tile's place within its own weight, so a
// weight computed inside a group gets exactly the sums it gets alone when
// the split plan is the same.
struct Tile {
  int64_t mt, n0;
  int u0, u1, rot;
  int split, g;
  int piece;   // index of a last-wave piece, -1 for a tile that is not one
};
// Every tile index, count and divisor here fits in 32 bits (the host refuses
// a plan of 2^31 tiles or more), and 32-bit division costs a fraction of
// 64-bit division, which sits at the start of every role's tile.
template <bool TAIL>
__device__ __forceinline__ Tile tile_of(const PrefillArgs &a, int64_t t) {
  Tile tl;
  const uint32_t t32 = static_cast<uint32_t>(t);
  const uint32_t tm = static_cast<uint32_t>(a.tiles_m);
  const uint32_t head = static_cast<uint32_t>(a.head_tiles);
  uint32_t mt, nt, ups;
  if (!TAIL || t32 < head) {
    const uint32_t sp = static_cast<uint32_t>(a.splits);
    const uint32_t rest = t32 / tm;
    mt = t32 - rest * tm;
    nt = rest / sp;
    tl.split = static_cast<int>(rest - nt * sp);
    ups = static_cast<uint32_t>(a.units_per_split);
    tl.piece = -1;
  } else {
    // last-wave piece: split s of the (head + j)-th tile in the unsplit order
    const uint32_t tt = t32 - head, nt_tail = static_cast<uint32_t>(a.tail_tiles);
    const uint32_t sidx = tt / nt_tail;
    const uint32_t ut = head + (tt - sidx * nt_tail);
    nt = ut / tm;
    mt = ut - nt * tm;
    tl.split = static_cast<int>(sidx);
    ups = static_cast<uint32_t>(a.tail_ups);
    tl.piece = static_cast<int>(tt);
  }
  tl.mt = mt;
  int g = 0;
  while (g + 1 < a.G && nt >= static_cast<uint32_t>(a.tile_n0[g + 1])) ++g;
  tl.g = g;
  const uint32_t ntl = nt - static_cast<uint32_t>(a.tile_n0[g]);
  tl.n0 = static_cast<int64_t>(ntl) * kTileN;
  tl.u0 = tl.split * static_cast<int>(ups);
  tl.u1 = min(tl.u0 + static_cast<int>(ups), static_cast<int>(a.K / 256));
  tl.rot = static_cast<int>((ntl + 7u * mt) % static_cast<uint32_t>(tl.u1 - tl.u0));
  return tl;
}

// Converter warp of stage pair J (J = 0: stages 0 and 1 of every unit, J =
// 1: stages 2 and 3): thread = weight row rr of this CTA.  Per unit it copies
// the granules of its two pieces out of the raw slot, releases the slot,
// waits for a free TMEM slot, dequantizes both stages (64 elements each) into
// its lane with two tcgen05.st, and one lane per warp arrives on the even
// CTA's ready barrier of the slot.  The warps of J = 0 fill slots 0, 2, 4, ...
// of the ring, those of J = 1 slots 1, 3, 5, ...
template <int TYPE, int J, bool TAIL>
__device__ __forceinline__ void convert_role(const Smem &s, const PrefillArgs &a, uint32_t tmem_slot0, int rr,
                                             uint32_t ready_even) {
  constexpr uint32_t RAW_BYTES = kRows * unit_bytes<TYPE>();
  const int lane = threadIdx.x & 31;
  const int SA = a.slots, SR = a.slots_raw;
  const int64_t npairs = gridDim.x / 2;
  int sa = J;            // TMEM slot of this warp's next pair (every other slot)
  uint32_t rnd = 0;      // its ring round; round r >= 1 waits for the MMA release of round r - 1
  int rs = 0;            // raw unit slot and its phase parity
  uint32_t rpar = 0;
  for (int64_t t = blockIdx.x / 2; t < a.total_tiles; t += npairs) {
    const Tile tl = tile_of<TAIL>(a, t);
    for (int u = tl.u0; u < tl.u1; ++u) {
      const bool got = wait_or_abort(s, &s.rfull[rs], rpar, a.wait);
      if (__any_sync(0xffffffffu, !got)) return;
      const uint4 *unit = reinterpret_cast<const uint4 *>(s.raw + static_cast<size_t>(rs) * RAW_BYTES +
                                                          static_cast<size_t>(rr) * unit_bytes<TYPE>());
      PairRegs<TYPE> r;
      load_pair<TYPE, J>(r, unit);
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.rempty[rs]);
      if (!pair_in_range<TYPE, J>(r)) record_range(a.wait.status);
      if (++rs == SR) {
        rs = 0;
        rpar ^= 1u;
      }
      if (rnd > 0) {
        const bool free_ = wait_or_abort(s, &s.consumed[sa], (rnd - 1) & 1u, a.wait, 32);
        if (__any_sync(0xffffffffu, !free_)) return;
      }
      tc_fence_after_sync();
      {
        uint32_t v[32];
        dequant_pair_piece<TYPE, J, 0>(r, v);
        tmem_st_32cols(tmem_slot0 + static_cast<uint32_t>(sa * kAColsSlot), v);
      }
      {
        uint32_t v[32];
        dequant_pair_piece<TYPE, J, 1>(r, v);
        tmem_st_32cols(tmem_slot0 + static_cast<uint32_t>(sa * kAColsSlot + kAColsStage), v);
      }
      tmem_st_wait();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(ready_even + static_cast<uint32_t>(sa) * 8u);
      sa += 2;
      if (sa >= SA) {
        sa -= SA;
        ++rnd;
      }
    }
  }
}

// Persistent CTA pair over pair tiles (pair index blockIdx.x / 2, stepping
// by the number of pairs); rank r = this CTA's rank in the cluster.
// TAIL: the plan splits its last wave in K (head_tiles < total_tiles); the
// instantiation without it carries none of the piece handling.
template <int TYPE, bool TAIL>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ WeightMaps maps, const __grid_constant__ PrefillArgs a) {
  constexpr int UB = unit_bytes<TYPE>();
  constexpr uint32_t RAW_BYTES = kRows * UB;   // one unit of this CTA's 128 rows
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tnc = a.tn / 2;                                        // tokens of this CTA
  const uint32_t stage_b_bytes = static_cast<uint32_t>(tnc) * 128u;   // one 64-K activation stage
  const uint32_t slot_b_bytes = 2u * stage_b_bytes;                    // one activation copy: a stage pair
  const Smem s = carve(base, a.slots, slot_b_bytes, a.slots_raw, RAW_BYTES);
  const uint32_t rank = cluster_ctarank();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int SQ = a.slots, SR = a.slots_raw;
  const int64_t pair = blockIdx.x / 2, npairs = gridDim.x / 2;
  const int units = static_cast<int>(a.K / 256);

  if (threadIdx.x == 0) {
    for (int i = 0; i < SQ; ++i) {
      // even CTA: its copy, the forwarded odd copy, 4 converter warps of each
      // CTA -- one wait per slot covers all inputs of 8 MMAs
      mbar_init(&s.ready[i], rank == 0 ? 2 + 2 * 4 : 1);
      mbar_init(&s.consumed[i], 1);
    }
    for (int i = 0; i < SR; ++i) {
      mbar_init(&s.rfull[i], 1);
      mbar_init(&s.rempty[i], kConvWarps);
    }
    mbar_init(s.accfull, 1);
    mbar_init(s.accempty, 2 * 4);      // 4 epilogue warps in each CTA
    mbar_init(s.drain, 1);
    *s.abort = 0u;
    fence_barrier_init();
    for (int g = 0; g < a.G; ++g) prefetch_tensormap(&maps.m[g]);
  }
  if (warp == kWarpW && lane == 0 && pair < a.total_tiles) {
    // weights are read-only: start this CTA's first units toward L2 while
    // the activation-rounding kernel before us finishes
    const Tile tl = tile_of<TAIL>(a, pair);
    for (int k = 0; k < 2 && k < tl.u1 - tl.u0; ++k) {
      const int u = tl.u0 + (tl.rot + k) % (tl.u1 - tl.u0);
      prefetch_l2_tile_2d(&maps.m[tl.g], u * (UB / 4), static_cast<int32_t>(tl.n0 + kRows * rank));
    }
  }
  if (warp == kWarpMma) {
    tmem_alloc_pair(s.tmem, static_cast<uint32_t>(kTmemCols));
    tmem_relinquish_pair();
  }
  __syncwarp();
  tc_fence_before_sync();
  cluster_sync();   // barriers of both CTAs initialised, TMEM allocated
  tc_fence_after_sync();
  pdl_trigger();
  // The launch-dependency wait sits in each role, just before its first read
  // of memory a predecessor may write (the activation and weight copies, the
  // row shifts) or its first write of the outputs; the converters and the
  // MMA issuer touch only shared and tensor memory and never wait.  All the
  // set-up before a role's first copy then overlaps the previous kernel.
  const uint32_t tmem_base = *s.tmem;
  const uint32_t a_col0 = static_cast<uint32_t>(a.tn);   // first weight-stage column

  if (warp == kWarpX) {
    // ---------------------------------------- activation stages (bulk copy)
    if (lane == 0) {
      const uint64_t keep = l2_policy_evict_last();   // every weight tile re-reads these
      // One copy per slot: the stage pair of one K unit, contiguous in the
      // tile-major layout (32 KB for 128 tokens: the copy engine's cost is
      // mostly per copy).  Ring position kept incrementally; round r >= 1
      // first waits for the MMA release of round r - 1.
      int64_t gs = 0;
      int sq = 0;
      uint32_t rnd = 0;
      bool ok = true;
      for (int64_t t = pair; t < a.total_tiles && ok; t += npairs) {
        const Tile tl = tile_of<TAIL>(a, t);
        const int64_t xt = 2 * tl.mt + rank;   // this CTA's token tile
        int u = tl.u0 + tl.rot;
        for (int k = tl.u0; k < tl.u1 && ok; ++k, u = (u + 1 == tl.u1 ? tl.u0 : u + 1)) {
          for (int kb4 = 0; kb4 < 4; kb4 += 2, ++gs) {
            if (rnd > 0 && !wait_or_abort(s, &s.consumed[sq], (rnd - 1) & 1u, a.wait, 64)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&s.ready[sq], slot_b_bytes);
            if (gs == 0) pdl_wait();
            bulk_g2s(s.b + static_cast<size_t>(sq) * slot_b_bytes,
                     reinterpret_cast<const uint8_t *>(a.x16) +
                         ((xt * units + u) * 4 + kb4) * static_cast<int64_t>(stage_b_bytes),
                     slot_b_bytes, &s.ready[sq], keep);
            if (++sq == SQ) {
              sq = 0;
              ++rnd;
            }
          }
        }
      }
      if (!ok)
        for (int64_t g = (gs > SQ ? gs - SQ : 0); g < gs; ++g)
          mbar_wait_for(&s.ready[g % SQ], static_cast<uint32_t>((g / SQ) & 1), kDrainLimitNs);
    }
  } else if (warp == kWarpMma && rank == 1) {
    // ------------------------------- odd CTA: forward activation arrivals
    if (lane == 0) {
      const uint32_t ready_even = mapa_shared(smem_u32(s.ready), 0);
      int sq = 0;
      uint32_t par = 0;
      bool ok = true;
      for (int64_t t = pair; t < a.total_tiles && ok; t += npairs) {
        const Tile tl = tile_of<TAIL>(a, t);
        for (int g = 0; g < 2 * (tl.u1 - tl.u0); ++g) {
          if (!wait_or_abort(s, &s.ready[sq], par, a.wait)) {
            ok = false;
            break;
          }
          mbar_arrive_remote(ready_even + static_cast<uint32_t>(sq) * 8u);
          if (++sq == SQ) {
            sq = 0;
            par ^= 1u;
          }
        }
      }
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------- even CTA: MMA issuer
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_f16(kTileN, static_cast<uint32_t>(a.tn), 0);
      const uint32_t b_base = smem_u32(s.b);
      int64_t i = 0;
      int sq = 0;
      uint32_t pq = 0;   // phase parity of the current round of the slot ring
      bool ok = true;
      for (int64_t t = pair; t < a.total_tiles && ok; t += npairs, ++i) {
        const Tile tl = tile_of<TAIL>(a, t);
        if (i >= 1 && !wait_or_abort(s, s.accempty, static_cast<uint32_t>((i - 1) & 1), a.wait)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        // One wait and one commit per 8 MMAs: the MMA issue queue is shallow,
        // so what this thread does between issues must stay short.
        for (int q = 0; q < 2 * (tl.u1 - tl.u0); ++q) {
          if (!wait_or_abort(s, &s.ready[sq], pq, a.wait)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t b_addr = b_base + static_cast<uint32_t>(sq) * slot_b_bytes;
          const uint32_t a_tmem = tmem_base + a_col0 + static_cast<uint32_t>(sq * kAColsSlot);
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int k = 0; k < kBK / 16; ++k)
              umma_f16_ts_pair(tmem_base, a_tmem + static_cast<uint32_t>(h * kAColsStage + 8 * k),
                               umma_desc_sw128(b_addr + static_cast<uint32_t>(h) * stage_b_bytes + 32 * k), idesc,
                               (q > 0 || h > 0 || k > 0) ? 1u : 0u);
          umma_commit_pair_mc(&s.consumed[sq], 0x3);
          if (++sq == SQ) {
            sq = 0;
            pq ^= 1u;
          }
        }
        if (ok) umma_commit_pair_mc(s.accfull, 0x3);
      }
      if (!ok) {
        umma_commit_pair(s.drain);
        mbar_wait_for(s.drain, 0, kDrainLimitNs);
      }
    }
  } else if (warp == kWarpW) {
    // ------------------------------------------- raw weight units (TMA)
    if (lane == 0) {
      int64_t gu = 0;
      int rs = 0;
      uint32_t rnd = 0;
      bool ok = true;
      for (int64_t t = pair; t < a.total_tiles && ok; t += npairs) {
        const Tile tl = tile_of<TAIL>(a, t);
        const int32_t row0 = static_cast<int32_t>(tl.n0 + kRows * rank);
        int u = tl.u0 + tl.rot;
        for (int k = tl.u0; k < tl.u1; ++k, ++gu, u = (u + 1 == tl.u1 ? tl.u0 : u + 1)) {
          if (rnd > 0 && !wait_or_abort(s, &s.rempty[rs], (rnd - 1) & 1u, a.wait, 64)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&s.rfull[rs], RAW_BYTES);
          if (gu == 0) pdl_wait();
          tma_load_2d(s.raw + static_cast<size_t>(rs) * RAW_BYTES, &maps.m[tl.g], u * (UB / 4), row0,
                      &s.rfull[rs]);
          if (++rs == SR) {
            rs = 0;
            ++rnd;
          }
        }
      }
      if (!ok)
        for (int64_t g = (gu > SR ? gu - SR : 0); g < gu; ++g)
          mbar_wait_for(&s.rfull[g % SR], static_cast<uint32_t>((g / SR) & 1), kDrainLimitNs);
    }
  } else if (warp < kWarpEpi0) {
    // ------------------------------------------ converters (dequantize)
    const int q = warp & 3;   // TMEM lane quadrant this warp may access
    const uint32_t slot0 = tmem_base + (static_cast<uint32_t>(32 * q) << 16) + a_col0;
    const uint32_t ready_even = mapa_shared(smem_u32(s.ready), 0);
    if (warp < kWarpConv0 + 4) convert_role<TYPE, 0, TAIL>(s, a, slot0, 32 * q + lane, ready_even);
    else convert_role<TYPE, 1, TAIL>(s, a, slot0, 32 * q + lane, ready_even);
  } else {
    // ------------------------------- epilogue: TMEM -> y * 2^-s_m
    const int q = warp & 3;
    const int64_t r = kRows * rank + 32 * q + lane;   // weight row within the pair tile
    const uint32_t accempty_even = mapa_shared(smem_u32(s.accempty), 0);
    const int nchunks = a.tn / 32;
    int64_t i = 0;
    for (int64_t t = pair; t < a.total_tiles; t += npairs, ++i) {
      const Tile tl = tile_of<TAIL>(a, t);
      const int64_t n = tl.n0 + r;
      const int64_t Ng = a.N[tl.g];
      const bool n_ok = n < Ng;
      const int64_t m0 = tl.mt * a.tn;
      // before the accumulator wait: lane j holds 2^-s of token m0 + 32c + j for every
      // chunk c (0 for padding tokens), so the drain below has no loads
      if (i == 0) pdl_wait();
      float my_scale[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const int64_t m = m0 + 32 * c + lane;
        const int sft = (c < nchunks && m < a.M) ? __ldg(a.shift + m) : 0;
        my_scale[c] = __int_as_float((127 - sft) << 23);   // s in [-113, 126]: a normal 2^-s
      }
      const bool got = wait_or_abort(s, s.accfull, static_cast<uint32_t>(i & 1), a.wait, 256);
      if (__any_sync(0xffffffffu, !got)) break;
      tc_fence_after_sync();
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        if (c >= nchunks) break;
        uint32_t v[32];
        tmem_ld_32cols(tmem_base + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(32 * c), v);
        tmem_ld_wait();
        if (c == nchunks - 1) {
          // every accumulator column is in registers: let the next tile start
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive_remote(accempty_even);
        }
        // scale branch-free (the shuffles pipeline), then store
#pragma unroll
        for (int j = 0; j < 32; ++j)
          v[j] = __float_as_uint(__fmul_rn(__uint_as_float(v[j]), __shfl_sync(0xffffffffu, my_scale[c], j)));
        const int64_t mc = m0 + 32 * c;
        float *yp = a.y[tl.g] + static_cast<int64_t>(tl.split) * a.split_stride[tl.g] + mc * Ng + n;
        int64_t ys = Ng;
        if (TAIL && tl.piece >= 0) {
          // a last-wave piece writes its partial token-major into its own block
          yp = a.tail_part + (static_cast<int64_t>(tl.piece) * a.tn + 32 * c) * kTileN + r;
          ys = kTileN;
        }
        if (n_ok && mc + 32 <= a.M) {
#pragma unroll
          for (int j = 0; j < 32; ++j) yp[static_cast<int64_t>(j) * ys] = __uint_as_float(v[j]);
        } else if (n_ok) {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (mc + j < a.M) yp[static_cast<int64_t>(j) * ys] = __uint_as_float(v[j]);
        }
      }
    }
  }
  __syncwarp();
  tc_fence_before_sync();
  cluster_sync();   // no CTA leaves while its pair may still touch its memory
  if (warp == kWarpMma) {
    tc_fence_after_sync();
    tmem_dealloc_pair(tmem_base, static_cast<uint32_t>(kTmemCols));
  }
}

// --------------------------------------------------- activation rounding --
// One CTA per activation row: row max -> shift s (max |x| * 2^s in
// [2^14, 2^15), 0 for a zero row, clamped to [-113, 126] so that 2^s and
// 2^-s are both normal fp32: every finite row with max |x| >= 2^-112 lands in
// the binade, up to FLT_MAX) -> binary16 RNE of x * 2^s (an exact scaling
// unless the product is an fp32 subnormal, far below binary16's range).
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
    s = min(126, max(-113, 15 - e));
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

// The n <= kMaxKSplits partials p[0], p[stride], ... summed in index order.
// Loads go out four at a time before their adds, so up to four latencies
// overlap instead of adding up, in few enough registers to keep the kernel
// at full occupancy.
constexpr int kMaxKSplits = 16;
__device__ __forceinline__ void add4(float4 &acc, const float4 &v) {
  acc.x += v.x;
  acc.y += v.y;
  acc.z += v.z;
  acc.w += v.w;
}
__device__ __forceinline__ float4 sum_splits(const float4 *p, int64_t stride, int n) {
  float4 v[4];
#pragma unroll
  for (int j = 0; j < 4; ++j)
    if (j < n) v[j] = __ldg(p + j * stride);
  float4 acc = v[0];
#pragma unroll
  for (int j = 1; j < 4; ++j)
    if (j < n) add4(acc, v[j]);
  for (int s0 = 4; s0 < n; s0 += 4) {
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (s0 + j < n) v[j] = __ldg(p + (s0 + j) * stride);
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (s0 + j < n) add4(acc, v[j]);
  }
  return acc;
}

// Split-K partials -> output, summed in split order (deterministic).  Split
// s's partial of the M x N outputs starts at part + s * sstride, sstride =
// total rounded up to a multiple of 4, so every split is float4-aligned.
__global__ void __launch_bounds__(256) splitk_reduce_kernel(const float *__restrict__ part, int64_t total,
                                                            int64_t sstride, int splits, float *__restrict__ y) {
  pdl_trigger();
  pdl_wait();
  const int64_t n4 = total / 4, s4 = sstride / 4;
  const float4 *p4 = reinterpret_cast<const float4 *>(part);
  float4 *y4 = reinterpret_cast<float4 *>(y);
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4; i += stride)
    y4[i] = sum_splits(p4 + i, s4, splits);
  for (int64_t i = 4 * n4 + static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride) {
    float acc = part[i];
    for (int s = 1; s < splits; ++s) acc += part[static_cast<int64_t>(s) * sstride + i];
    y[i] = acc;
  }
}

// Last-wave pieces -> outputs: for each split tile of the last wave (tile
// head + j of the unsplit order), token m and weight row n, the pieces'
// partials are summed in split order (deterministic) and written to y.  One
// thread per 4 consecutive rows of one token of one tile.
__global__ void __launch_bounds__(256) tail_reduce_kernel(const __grid_constant__ PrefillArgs a) {
  pdl_trigger();
  pdl_wait();
  const uint32_t per_tile = static_cast<uint32_t>(a.tn) * (kTileN / 4);   // float4s per piece
  const uint32_t total = static_cast<uint32_t>(a.tail_tiles) * per_tile;
  const int64_t split_stride4 = static_cast<int64_t>(a.tail_tiles) * per_tile;
  const float4 *p4 = reinterpret_cast<const float4 *>(a.tail_part);
  const uint32_t tm = static_cast<uint32_t>(a.tiles_m);
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i += gridDim.x * blockDim.x) {
    const uint32_t j = i / per_tile, rem = i - j * per_tile;
    const uint32_t ml = rem / (kTileN / 4), r4 = rem - ml * (kTileN / 4);
    const uint32_t ut = static_cast<uint32_t>(a.head_tiles) + j;
    const uint32_t nt = ut / tm, mt = ut - nt * tm;
    const int64_t m = static_cast<int64_t>(mt) * a.tn + ml;
    if (m >= a.M) continue;
    int g = 0;
    while (g + 1 < a.G && nt >= static_cast<uint32_t>(a.tile_n0[g + 1])) ++g;
    const int64_t Ng = a.N[g];
    const int64_t n = static_cast<int64_t>(nt - static_cast<uint32_t>(a.tile_n0[g])) * kTileN + 4 * r4;
    if (n >= Ng) continue;
    const float4 acc = sum_splits(p4 + i, split_stride4, a.tail_splits);
    float *yr = a.y[g] + m * Ng + n;
    if ((Ng & 3) == 0) {
      *reinterpret_cast<float4 *>(yr) = acc;   // y is 16-byte aligned and n is a multiple of 4
    } else {
      yr[0] = acc.x;
      if (n + 1 < Ng) yr[1] = acc.y;
      if (n + 2 < Ng) yr[2] = acc.z;
      if (n + 3 < Ng) yr[3] = acc.w;
    }
  }
}

// Test hook: the whole dequantized weight matrix in binary16, produced by the
// same device functions as the GEMM's converter warps (one thread per
// 256-element unit of a row, both stage pairs).
template <int TYPE, int J>
__device__ __forceinline__ void pair_to_f16(const uint4 *unit, uint16_t *dst, uint32_t *status) {
  PairRegs<TYPE> r;
  load_pair<TYPE, J>(r, unit);
  if (!pair_in_range<TYPE, J>(r)) record_range(status);
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    uint32_t v[32];
    if (i == 0) dequant_pair_piece<TYPE, J, 0>(r, v);
    else dequant_pair_piece<TYPE, J, 1>(r, v);
    uint4 *d4 = reinterpret_cast<uint4 *>(dst + (2 * J + i) * 64);
#pragma unroll
    for (int c = 0; c < 8; ++c) d4[c] = make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
  }
}

template <int TYPE>
__global__ void __launch_bounds__(128) w_to_f16_kernel(const uint8_t *__restrict__ w, int64_t N, int64_t K,
                                                       int64_t row_bytes, uint16_t *__restrict__ w16,
                                                       uint32_t *status) {
  const int64_t units = K / 256;
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= N * units) return;
  const int64_t n = idx / units, u = idx % units;
  const uint4 *unit = reinterpret_cast<const uint4 *>(w + n * row_bytes + u * unit_bytes<TYPE>());
  uint16_t *dst = w16 + n * K + u * 256;
  pair_to_f16<TYPE, 0>(unit, dst, status);
  pair_to_f16<TYPE, 1>(unit, dst, status);
}

// ------------------------------------------------------ small-M bridge --
// For a single token the tensor-core pipeline is all fill and drain: the
// weights stream once, but three launches (activation rounding, GEMM, split
// reduction) and the pair pipeline's start-up dominate.  Those token counts
// (small_max_m below, chosen from the measured sweep) take this CUDA-core
// kernel instead, with the same operands: every
// activation row rounded to binary16 after the same exact 2^s_m scaling,
// every weight element dequantized by the converter's own functions, each
// product exact in fp32, fp32 sums, the result scaled back by 2^-s_m.
//  * One launch.  Each CTA copies the M fp32 activation rows into shared
//    memory, finds the row shifts and rounds the rows in place, while its
//    first weight boxes are in flight.
//  * lane = weight row: a warp takes 32 rows of one weight, one 256-element
//    unit at a time (a 2-D TMA box of 32 rows x 272 / 144 B); warp w takes the
//    units u = w, w+8, ...; all lanes read the same activation values
//    (broadcast), two K elements per paired fp32 FMA.
//  * The 8 warps' partial sums meet in shared memory in a fixed order.
constexpr int kSmallMaxM = 3;
constexpr int kSmallWarps = 8;
constexpr int kSmallRows = 32;
constexpr size_t kSmallMaxActSmem = 128 * 1024;
constexpr size_t kSmallPipeSmem = 227 * 1024;   // dynamic shared memory the kernel may take

struct SmallArgs {
  int64_t K, M;
  int G;
  int64_t N[kMaxGroup];
  float *y[kMaxGroup];
  int64_t group0[kMaxGroup + 1];   // first 32-row group of each weight
  int64_t total_groups;
  const float *x;                  // [M][K] fp32
  const __half *x16;               // mma form: [8][K] rounded activations (rows >= M zero)
  const int32_t *shift;            // mma form: [M] row shifts
  int nunits, stages;
  uint32_t box_bytes, ring_off, bar_off, red_off, sc_off;
  WaitCtl wait;
};

// Item position of a warp: row group g, unit u (warp, warp + 8, ...).
struct SmallCursor {
  int64_t g;
  int u;
  __device__ __forceinline__ void first(const SmallArgs &a, int warp) {
    g = blockIdx.x;
    u = warp;
    if (u >= a.nunits) g = a.total_groups;
  }
  __device__ __forceinline__ void next(const SmallArgs &a, int warp, int nw = kSmallWarps) {
    u += nw;
    if (u >= a.nunits) {
      u = warp;
      g += gridDim.x;
    }
  }
  __device__ __forceinline__ bool valid(const SmallArgs &a) const { return g < a.total_groups; }
};

__device__ __forceinline__ int small_weight_of(const SmallArgs &a, int64_t g) {
  int w = 0;
  while (w + 1 < a.G && g >= a.group0[w + 1]) ++w;
  return w;
}

template <int UB>
__device__ __forceinline__ void small_issue(const WeightMaps &maps, const SmallArgs &a, const SmallCursor &c,
                                            uint8_t *dst, uint64_t *bar) {
  const int w = small_weight_of(a, c.g);
  const int32_t row0 = static_cast<int32_t>((c.g - a.group0[w]) * kSmallRows);
  mbar_arrive_expect_tx(bar, a.box_bytes);
  tma_load_2d(dst, &maps.m[w], c.u * (UB / 4), row0, bar);
}

// acc2[m] (two fp32 lanes: even and odd K) += w16[k .. k+63] * x[m][k .. k+63]
// for one 64-element piece whose binary16 weights are the 32 words `piece`.
template <int M>
__device__ __forceinline__ void small_piece_fma(const uint32_t (&piece)[32], const float *xk, int64_t K,
                                                uint64_t (&acc2)[M]) {
#pragma unroll
  for (int c = 0; c < 16; ++c) {   // 4 elements per step
    const float2 w01 = __half22float2(bits_h2(piece[2 * c]));
    const float2 w23 = __half22float2(bits_h2(piece[2 * c + 1]));
    const uint64_t wa = pack2(w01.x, w01.y), wb = pack2(w23.x, w23.y);
#pragma unroll
    for (int m = 0; m < M; ++m) {
      const float4 xv = *reinterpret_cast<const float4 *>(xk + m * K + 4 * c);
      acc2[m] = fma2_rn(wa, pack2(xv.x, xv.y), acc2[m]);
      acc2[m] = fma2_rn(wb, pack2(xv.z, xv.w), acc2[m]);
    }
  }
}

// The binary16 range guard of pair_in_range for a whole 256-element unit
// held as NV uint4 granules.
template <int TYPE, int NV>
__device__ __forceinline__ bool unit_in_range(const uint4 (&v)[NV]) {
  if constexpr (TYPE == DSQ_Q8_0) {
    uint32_t worst = 0;
#pragma unroll
    for (int b = 0; b < 8; ++b) {
      const int wd = (b & 1) ? (17 * b - 1) / 2 : 17 * b / 2;   // word holding block b's scale
      const uint32_t w = word4(v[wd >> 2], wd & 3);
      worst = max(worst, ((b & 1) ? (w >> 16) : w) & 0x7fffu);
    }
    return worst < 0x6008u;
  } else {
    PairRegs<DSQ_Q4_K> r;
    r.hdr = v[0];
    return pair_in_range<DSQ_Q4_K, 0>(r) && pair_in_range<DSQ_Q4_K, 1>(r);
  }
}

template <int TYPE, int M>
__device__ __forceinline__ void small_unit(const uint8_t *p, const float *xf, int64_t K, int u, uint64_t (&acc2)[M],
                                           uint32_t *status) {
  constexpr int NV = TYPE == DSQ_Q8_0 ? 17 : 9;
  uint4 v[NV];
  const uint4 *p4 = reinterpret_cast<const uint4 *>(p);
#pragma unroll
  for (int i = 0; i < NV; ++i) v[i] = p4[i];
  if (!unit_in_range<TYPE, NV>(v)) record_range(status);
  const float *xu = xf + static_cast<int64_t>(u) * 256;
#pragma unroll
  for (int P = 0; P < 4; ++P) {
    uint32_t piece[32];
    if constexpr (TYPE == DSQ_Q8_0) {
      piece_q8_0([&](int i) { return word4(v[(17 * P + i) >> 2], (17 * P + i) & 3); }, piece);
    } else {
      if (P == 0) piece_q4_k<0>(v[0], [&](int i) { return word4(v[1 + (i >> 2)], i & 3); }, piece);
      if (P == 1) piece_q4_k<1>(v[0], [&](int i) { return word4(v[3 + (i >> 2)], i & 3); }, piece);
      if (P == 2) piece_q4_k<2>(v[0], [&](int i) { return word4(v[5 + (i >> 2)], i & 3); }, piece);
      if (P == 3) piece_q4_k<3>(v[0], [&](int i) { return word4(v[7 + (i >> 2)], i & 3); }, piece);
    }
    small_piece_fma<M>(piece, xu + 64 * P, K, acc2);
  }
}

template <int TYPE, int M>
__global__ void __launch_bounds__(kSmallWarps * 32, 1)
    prefill_small_kernel(const __grid_constant__ WeightMaps maps, const __grid_constant__ SmallArgs a) {
  constexpr int UB = unit_bytes<TYPE>();
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = a.stages;
  const int64_t K = a.K;
  float *xf = reinterpret_cast<float *>(base);   // [M][K]
  uint8_t *ring = base + a.ring_off + static_cast<size_t>(warp) * S * a.box_bytes;
  uint64_t *act_bar = reinterpret_cast<uint64_t *>(base + a.bar_off);
  uint64_t *bars = act_bar + 1 + warp * 2;
  volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(act_bar + 1 + 2 * kSmallWarps);
  __shared__ float row_scale[kSmallMaxM], scale_back[kSmallMaxM];   // 2^s_m and 2^-s_m
  float *red = reinterpret_cast<float *>(base + a.red_off);   // [2][8 warps][M][32]

  if (threadIdx.x == 0) {
    mbar_init(act_bar, 1);
    *abort_flag = 0u;
    for (int w = 0; w < a.G; ++w) prefetch_tensormap(&maps.m[w]);
  }
  if (lane == 0)
    for (int s = 0; s < S; ++s) mbar_init(&bars[s], 1);
  fence_barrier_init();
  SmallCursor issue;
  issue.first(a, warp);
  if (lane == 0) {
    // weights are read-only: this warp's first boxes toward L2 while the
    // kernel before us finishes
    SmallCursor c = issue;
    for (int s = 0; s < S && c.valid(a); ++s, c.next(a, warp)) {
      const int w = small_weight_of(a, c.g);
      prefetch_l2_tile_2d(&maps.m[w], c.u * (UB / 4), static_cast<int32_t>((c.g - a.group0[w]) * kSmallRows));
    }
  }
  __syncthreads();
  pdl_trigger();
  pdl_wait();

  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(act_bar, static_cast<uint32_t>(M * K * 4));
    bulk_g2s(xf, a.x, static_cast<uint32_t>(M * K * 4), act_bar, l2_policy_evict_last());
  }
  int64_t n_issued = 0, n_waited = 0;
  if (lane == 0)
    for (int s = 0; s < S && issue.valid(a); ++s, issue.next(a, warp), ++n_issued)
      small_issue<UB>(maps, a, issue, ring + static_cast<size_t>(s) * a.box_bytes, &bars[s]);
  bool ok = __all_sync(0xffffffffu, mbar_wait_for(act_bar, 0, a.wait.limit_ns));
  if (!ok && lane == 0 && *abort_flag == 0u) {
    *abort_flag = 1u;
    record_timeout(a.wait);
  }
  // row shifts (warp m takes row m), then every element rounded in place:
  // float(binary16_rne(x * 2^s_m)), exactly as the tensor-core path rounds it
  if (warp < M) {
    float amax = 0.0f;
    if (ok)
      for (int64_t k = lane; k < K; k += 32) amax = fmaxf(amax, fabsf(xf[warp * K + k]));
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    int sft = 0;
    if (amax > 0.0f && !isinf(amax)) {
      int e;
      frexpf(amax, &e);
      sft = min(126, max(-113, 15 - e));
    }
    if (lane == 0) {
      row_scale[warp] = __int_as_float((127 + sft) << 23);
      scale_back[warp] = __int_as_float((127 - sft) << 23);
    }
  }
  __syncthreads();
  if (ok) {
    for (int m = 0; m < M; ++m) {
      const float sc = row_scale[m];
      for (int64_t k = threadIdx.x; k < K; k += blockDim.x)
        xf[m * K + k] = __half2float(__float2half_rn(__fmul_rn(xf[m * K + k], sc)));
    }
  }
  __syncthreads();

  int slot = 0;
  uint32_t parity = 0;
  int buf = 0;
  for (int64_t g = blockIdx.x; g < a.total_groups; g += gridDim.x, buf ^= 1) {
    uint64_t acc2[M];
#pragma unroll
    for (int m = 0; m < M; ++m) acc2[m] = 0ull;
    for (int u = warp; u < a.nunits; u += kSmallWarps) {
      ok = ok && *abort_flag == 0u;
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait_for(&bars[slot], parity, a.wait.limit_ns));
      if (!ok) {
        if (lane == 0 && *abort_flag == 0u) {
          *abort_flag = 1u;
          record_timeout(a.wait);
        }
      } else {
        ++n_waited;
        small_unit<TYPE, M>(ring + static_cast<size_t>(slot) * a.box_bytes + static_cast<size_t>(lane) * UB, xf, K,
                            u, acc2, a.wait.status);
        __syncwarp();
        if (lane == 0 && issue.valid(a)) {
          fence_proxy_async_smem();
          small_issue<UB>(maps, a, issue, ring + static_cast<size_t>(slot) * a.box_bytes, &bars[slot]);
          issue.next(a, warp);
          ++n_issued;
        }
      }
      if (++slot == S) {
        slot = 0;
        parity ^= 1u;
      }
    }
    float *rb = red + static_cast<size_t>(buf) * kSmallWarps * M * 32;
#pragma unroll
    for (int m = 0; m < M; ++m) rb[(warp * M + m) * 32 + lane] = __fadd_rn(lo_of(acc2[m]), hi_of(acc2[m]));
    __syncthreads();
    for (int m = warp; m < M; m += kSmallWarps) {
      float v = 0.0f;
#pragma unroll
      for (int w = 0; w < kSmallWarps; ++w) v += rb[(w * M + m) * 32 + lane];
      const int wi = small_weight_of(a, g);
      const int64_t row = (g - a.group0[wi]) * kSmallRows + lane;
      if (row < a.N[wi] && *abort_flag == 0u) a.y[wi][m * a.N[wi] + row] = __fmul_rn(v, scale_back[m]);
    }
  }
  if (lane == 0)
    for (int64_t k = n_waited; k < n_issued; ++k)
      mbar_wait_for(&bars[k % S], static_cast<uint32_t>((k / S) & 1), kDrainLimitNs);
  if (threadIdx.x == 0 && !ok) mbar_wait_for(act_bar, 0, kDrainLimitNs);
}

// ------------------------------------------- 4 to 8 tokens on mma.sync ---
// Between the CUDA-core bridge and the CTA-pair pipeline.  One launch after
// the activation rounding multiplies the tensor-core path's binary16 operands
// -- the converters' formulas, element for element -- on the warp-level
// tensor-core instruction mma.sync.m16n8k16 (fp16 operands, fp32
// accumulation).  A warp takes a 32-row box of one K unit: two 16-row
// m-tiles, 16 k-steps of 16.  Lane 4 grp + t dequantizes exactly the weights
// its A fragments hold (rows grp and grp + 8 of each m-tile, eight elements
// of each 32-element block, see mma_box), so every weight is converted once.
// The activations sit in shared memory as 32-bit words of two binary16 K
// elements, [k-step][pair][8 tokens] (tokens M..7 zero), so the B fragments
// load without bank conflicts.  The 8 warps' partials meet in shared memory in a
// fixed order, then each output is scaled back by 2^-s as in the epilogue of
// the CTA-pair kernel.
constexpr int kSmallMmaMaxM = 8;
// 16 warps per CTA with one ring slot each (more latency hidden than 8 warps
// with two; a 4096-row weight is one box per warp).  Q8_0's larger boxes
// leave room for only one reduction buffer, so its CTAs take a second
// barrier per row group before the buffer is reused.
__host__ __device__ constexpr int small_mma_warps(int) { return 16; }
__host__ __device__ constexpr int small_mma_stages(int) { return 1; }
__host__ __device__ constexpr int small_mma_red_bufs(int type) { return type == DSQ_Q4_K ? 2 : 1; }
constexpr int kScrStride = 18;   // words per row of the Q4_K scale scratch (8 pairs + pad)

__device__ __forceinline__ void mma_f16_m16n8k16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                                 uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Lane = row of the box: the binary16 range guard of the unit and, for Q4_K,
// the eight (d*sc_j, -dmin*m_j) of the row into the warp's scratch.
template <int TYPE>
__device__ __forceinline__ void mma_row_prep(const uint8_t *row, float *scr, int lane, uint32_t *status) {
  if constexpr (TYPE == DSQ_Q8_0) {
    uint32_t worst = 0;
#pragma unroll
    for (int b = 0; b < 8; ++b)
      worst = max(worst, static_cast<uint32_t>(*reinterpret_cast<const uint16_t *>(row + 34 * b)) & 0x7fffu);
    if (worst >= 0x6008u) record_range(status);
  } else {
    PairRegs<DSQ_Q4_K> r;
    r.hdr = *reinterpret_cast<const uint4 *>(row);
    if (!(pair_in_range<DSQ_Q4_K, 0>(r) && pair_in_range<DSQ_Q4_K, 1>(r))) record_range(status);
    const float d = __half2float(__ushort_as_half(static_cast<unsigned short>(r.hdr.x & 0xffffu)));
    const float dmin = __half2float(__ushort_as_half(static_cast<unsigned short>(r.hdr.x >> 16)));
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      uint32_t scw, mw;
      if (j < 4) {
        scw = r.hdr.y & 0x3f3f3f3fu;
        mw = r.hdr.z & 0x3f3f3f3fu;
      } else {
        scw = (r.hdr.w & 0x0f0f0f0fu) | ((r.hdr.y >> 2) & 0x30303030u);
        mw = ((r.hdr.w >> 4) & 0x0f0f0f0fu) | ((r.hdr.z >> 2) & 0x30303030u);
      }
      const int sh = 8 * (j & 3);
      *reinterpret_cast<float2 *>(scr + lane * kScrStride + 2 * j) =
          make_float2(__fmul_rn(d, static_cast<float>((scw >> sh) & 0xffu)),
                      -__fmul_rn(dmin, static_cast<float>((mw >> sh) & 0xffu)));
    }
  }
}

// The K order inside a 32-element block is free as long as both operands
// follow it.  Lane 4 grp + t takes the block's elements 8t .. 8t+7 (one
// contiguous run of codes, converted four or eight at a time as the
// converters do): pairs p0 = (8t, 8t+1) and p1 = (8t+2, 8t+3) feed the first
// k-step of the block as its (2t, 2t+1) and (2t+8, 2t+9) elements, p2 and p3
// the second step; the activation layout is permuted to match when it is
// filled.
template <int TYPE>
__device__ __forceinline__ void mma_row_pairs(const uint8_t *box, const float *scr, int r, int blk, int t,
                                              uint32_t (&p)[4]) {
  if constexpr (TYPE == DSQ_Q8_0) {
    const uint8_t *rb = box + r * 272 + 34 * blk;
    const __half2 d2 = __half2half2(*reinterpret_cast<const __half *>(rb));
    uint32_t c0, c1;
    if (blk & 1) {   // codes start word-aligned
      c0 = *reinterpret_cast<const uint32_t *>(rb + 2 + 8 * t);
      c1 = *reinterpret_cast<const uint32_t *>(rb + 6 + 8 * t);
    } else {         // codes start 2 bytes past a word boundary
      const uint32_t w0 = *reinterpret_cast<const uint32_t *>(rb + 8 * t);
      const uint32_t w1 = *reinterpret_cast<const uint32_t *>(rb + 4 + 8 * t);
      const uint32_t w2 = *reinterpret_cast<const uint32_t *>(rb + 8 + 8 * t);
      c0 = __funnelshift_r(w0, w1, 16);
      c1 = __funnelshift_r(w1, w2, 16);
    }
    q8x4_to_h(c0, d2, p[0], p[1]);
    q8x4_to_h(c1, d2, p[2], p[3]);
  } else {
    const uint2 w = *reinterpret_cast<const uint2 *>(box + r * 144 + 16 + 32 * (blk >> 1) + 8 * t);
    const bool high = blk & 1;
    const uint32_t q0 = high ? (w.x >> 4) & 0x0f0f0f0fu : w.x & 0x0f0f0f0fu;
    const uint32_t q1 = high ? (w.y >> 4) & 0x0f0f0f0fu : w.y & 0x0f0f0f0fu;
    const float2 an = *reinterpret_cast<const float2 *>(scr + r * kScrStride + 2 * blk);
    const uint64_t a2 = pack2(an.x, an.x), nb2 = pack2(an.y, an.y);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t q = i < 2 ? q0 : q1;
      const int e = 2 * (i & 1);
      const uint64_t f2 = pack2(__uint_as_float(__byte_perm(q, 0x4B000000u, 0x7540 + e)),
                                __uint_as_float(__byte_perm(q, 0x4B000000u, 0x7540 + e + 1)));
      const uint64_t v2 = fma2_rn(sub2_rn(f2, kMagic2), a2, nb2);
      p[i] = h2_bits(__floats2half2_rn(lo_of(v2), hi_of(v2)));
    }
  }
}

// One box (32 rows x unit u) into the accumulators: acc[mt] holds rows
// grp + 16 mt (+8) x tokens 2t, 2t + 1.
template <int TYPE>
__device__ __forceinline__ void mma_box(const uint8_t *box, const float *scr, const uint32_t *xa, int u, int grp,
                                        int t, float (&acc)[2][4]) {
#pragma unroll 2
  for (int blk = 0; blk < 8; ++blk) {
    uint32_t P[2][2][4];   // [m-tile][row half][pair]
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int h = 0; h < 2; ++h) mma_row_pairs<TYPE>(box, scr, grp + 8 * h + 16 * mt, blk, t, P[mt][h]);
#pragma unroll
    for (int st = 0; st < 2; ++st) {
      const uint32_t *xk = xa + ((u * 16 + 2 * blk + st) * 8 + t) * 8 + grp;
      const uint32_t b0 = xk[0], b1 = xk[32];
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        const uint32_t A[4] = {P[mt][0][2 * st], P[mt][1][2 * st], P[mt][0][2 * st + 1], P[mt][1][2 * st + 1]};
        mma_f16_m16n8k16(acc[mt], A, b0, b1);
      }
    }
  }
}

template <int TYPE, int M>
__global__ void __launch_bounds__(small_mma_warps(TYPE) * 32, 1)
    prefill_small_mma_kernel(const __grid_constant__ WeightMaps maps, const __grid_constant__ SmallArgs a) {
  constexpr int UB = unit_bytes<TYPE>();
  constexpr int NW = small_mma_warps(TYPE);
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, grp = lane >> 2, t = lane & 3;
  const int S = a.stages;
  uint32_t *xa = reinterpret_cast<uint32_t *>(base);   // [K/2][8]
  uint8_t *ring = base + a.ring_off + static_cast<size_t>(warp) * S * a.box_bytes;
  uint64_t *bars = reinterpret_cast<uint64_t *>(base + a.bar_off) + warp * 2;
  volatile uint32_t *abort_flag =
      reinterpret_cast<volatile uint32_t *>(reinterpret_cast<uint64_t *>(base + a.bar_off) + 2 * NW);
  float *red = reinterpret_cast<float *>(base + a.red_off);   // [2][NW warps][M][32]
  float *scr = reinterpret_cast<float *>(base + a.sc_off) + warp * kSmallRows * kScrStride;
  __shared__ float scale_back[kSmallMmaMaxM];   // 2^-s_m

  if (threadIdx.x == 0) {
    *abort_flag = 0u;
    for (int w = 0; w < a.G; ++w) prefetch_tensormap(&maps.m[w]);
  }
  if (lane == 0)
    for (int s = 0; s < S; ++s) mbar_init(&bars[s], 1);
  fence_barrier_init();
  SmallCursor issue;
  issue.first(a, warp);
  if (lane == 0) {
    // weights are read-only: this warp's first boxes toward L2 while the
    // activation rounding before us finishes
    SmallCursor c = issue;
    for (int s = 0; s < S && c.valid(a); ++s, c.next(a, warp, NW)) {
      const int w = small_weight_of(a, c.g);
      prefetch_l2_tile_2d(&maps.m[w], c.u * (UB / 4), static_cast<int32_t>((c.g - a.group0[w]) * kSmallRows));
    }
  }
  __syncthreads();
  pdl_trigger();
  pdl_wait();

  int64_t n_issued = 0, n_waited = 0;
  if (lane == 0)
    for (int s = 0; s < S && issue.valid(a); ++s, issue.next(a, warp, NW), ++n_issued)
      small_issue<UB>(maps, a, issue, ring + static_cast<size_t>(s) * a.box_bytes, &bars[s]);
  {
    // the rounded activations into [k-step][pair][8 tokens] words in the
    // permuted K order of mma_box: K pair q = 4t + c of a 32-element block
    // (elements 2q, 2q+1) is pair t + 4 (c & 1) of the block's k-step c >> 1.
    // A thread takes one pair of every token (coalesced across the warp) and
    // stores two 16-byte words.
    const uint32_t kp_n = static_cast<uint32_t>(a.K / 2);
    const uint32_t *x32 = reinterpret_cast<const uint32_t *>(a.x16);
#pragma unroll 4
    for (uint32_t kp = threadIdx.x; kp < kp_n; kp += blockDim.x) {
      uint32_t v[8];
#pragma unroll
      for (int tok = 0; tok < 8; ++tok) v[tok] = tok < M ? __ldg(x32 + tok * kp_n + kp) : 0u;
      const uint32_t blk32 = kp >> 4, q = kp & 15u, tq = q >> 2, c = q & 3u;   // block of 32 (unit*8 + block)
      const uint32_t slot = ((2u * blk32 + (c >> 1)) * 8u + tq + 4u * (c & 1u)) * 8u;
      uint4 *dst = reinterpret_cast<uint4 *>(xa + slot);
      dst[0] = make_uint4(v[0], v[1], v[2], v[3]);
      dst[1] = make_uint4(v[4], v[5], v[6], v[7]);
    }
    if (threadIdx.x < M) scale_back[threadIdx.x] = __int_as_float((127 - __ldg(a.shift + threadIdx.x)) << 23);
  }
  __syncthreads();

  bool ok = true;
  int slot = 0;
  uint32_t parity = 0;
  int buf = 0;
  for (int64_t g = blockIdx.x; g < a.total_groups; g += gridDim.x, buf ^= 1) {
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    for (int u = warp; u < a.nunits; u += NW) {
      ok = ok && *abort_flag == 0u;
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait_for(&bars[slot], parity, a.wait.limit_ns));
      if (!ok) {
        if (lane == 0 && *abort_flag == 0u) {
          *abort_flag = 1u;
          record_timeout(a.wait);
        }
      } else {
        ++n_waited;
        const uint8_t *box = ring + static_cast<size_t>(slot) * a.box_bytes;
        mma_row_prep<TYPE>(box + static_cast<size_t>(lane) * UB, scr, lane, a.wait.status);
        __syncwarp();
        mma_box<TYPE>(box, scr, xa, u, grp, t, acc);
        __syncwarp();
        if (lane == 0 && issue.valid(a)) {
          fence_proxy_async_smem();
          small_issue<UB>(maps, a, issue, ring + static_cast<size_t>(slot) * a.box_bytes, &bars[slot]);
          issue.next(a, warp, NW);
          ++n_issued;
        }
      }
      if (++slot == S) {
        slot = 0;
        parity ^= 1u;
      }
    }
    float *rb = red + static_cast<size_t>(small_mma_red_bufs(TYPE) == 2 ? buf : 0) * NW * M * 32;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int tok = 2 * t + (c & 1), row = grp + 8 * (c >> 1) + 16 * mt;
        if (tok < M) rb[(warp * M + tok) * 32 + row] = acc[mt][c];
      }
    __syncthreads();
    for (int m = warp; m < M; m += NW) {
      float v = 0.0f;
#pragma unroll
      for (int w = 0; w < NW; ++w) v += rb[(w * M + m) * 32 + lane];
      const int wi = small_weight_of(a, g);
      const int64_t row = (g - a.group0[wi]) * kSmallRows + lane;
      if (row < a.N[wi] && *abort_flag == 0u) a.y[wi][m * a.N[wi] + row] = __fmul_rn(v, scale_back[m]);
    }
    if (small_mma_red_bufs(TYPE) == 1) __syncthreads();   // the single buffer is rewritten by the next group
  }
  if (lane == 0)
    for (int64_t k = n_waited; k < n_issued; ++k)
      mbar_wait_for(&bars[k % S], static_cast<uint32_t>((k / S) & 1), kDrainLimitNs);
}

// ------------------------------------------------------------------- host --
struct Plan {
  int tn, slots, slots_raw, splits, units_per_split;
  int64_t tiles_m, tiles_n, total_tiles, m_pad;
  int64_t head_tiles;                    // tiles before the last-wave pieces
  int tail_tiles, tail_splits, tail_ups;   // last-wave split (tail_splits = 1: none)
  size_t tail_off;                       // byte offset of the last-wave partials
  unsigned grid;   // CTAs (2 per pair)
  size_t smem, x16_bytes, shift_off, part_off, total;
  int64_t split_stride[kMaxGroup];   // floats per split of each weight's partials
  size_t part_g_off[kMaxGroup];      // byte offset of each weight's partials
};

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

constexpr size_t kSmemLimit = 227 * 1024;

template <int TYPE, bool TAIL>
cudaError_t launch_pair(const WeightMaps &maps, const PrefillArgs &args, unsigned grid, size_t smem,
                        cudaStream_t stream) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, prefill_kernel<TYPE, TAIL>, maps, args);
}

// How many CTA pairs of the GEMM kernel can be resident at once (clusters
// of 2 need two SMs of one GPC).  The shared-memory size is a function of
// (type, tn), so the answer is cached per device, type and tn (tn = 32 ..
// 256 in steps of 32): after the first call of each shape no call asks the
// runtime again.
int resident_pairs(int type, int tn, size_t smem, int sms) {
  static std::mutex mu;
  static int cache[kMaxDevices][2][8] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return sms / 2;
  const int ti = type == DSQ_Q8_0 ? 0 : 1;
  const int ni = tn / 32 - 1;   // 0..7
  std::lock_guard<std::mutex> lk(mu);
  if (cache[dev][ti][ni] > 0) return cache[dev][ti][ni];
  // both instantiations of a type take the same resources
  const void *kern = type == DSQ_Q8_0 ? reinterpret_cast<const void *>(prefill_kernel<DSQ_Q8_0, false>)
                                      : reinterpret_cast<const void *>(prefill_kernel<DSQ_Q4_K, false>);
  if (set_smem_once(kern, static_cast<int>(smem), "prefill") != DSQ_OK) return sms / 2;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(sms / 2 * 2));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) {
    (void)cudaGetLastError();
    n = sms / 2;
  }
  if (n > sms / 2) n = sms / 2;
  cache[dev][ti][ni] = n;
  return n;
}

// pairs < 0: ask the device (needs a current device), else use that count
// G weights of N[0..G-1] rows share the M x K activation.
Plan make_plan(int type, int G, const int64_t *N, int64_t K, int64_t M, int sms, int pairs) {
  Plan p{};
  // tokens per pair tile: the smallest multiple of 32 that covers M, at most
  // 256 (the MMA's N; each CTA holds tn/2 of them)
  p.tn = M <= 256 ? static_cast<int>((M + 31) / 32 * 32) : 256;
  p.tiles_m = (M + p.tn - 1) / p.tn;
  p.tiles_n = 0;
  for (int g = 0; g < G; ++g) p.tiles_n += (N[g] + kTileN - 1) / kTileN;
  const int units = static_cast<int>(K / 256);
  // TMEM: tn accumulator columns, then up to 8 (an even number of) 32-column
  // weight stages
  // pipeline slots (a stage pair each): as many as TMEM holds next to the
  // accumulators (at most 6, even, so the two converter groups alternate)
  p.slots = (kTmemCols - p.tn) / kAColsSlot;
  if (p.slots > kMaxSlots) p.slots = kMaxSlots;
  p.slots &= ~1;
  // shared memory: the slots' activation pairs (32 KB each for 128 tokens:
  // the copy engine's cost is mostly per copy), the rest to raw weight
  // units (at least 2, at most 4)
  const size_t slot_b = 2 * static_cast<size_t>(p.tn / 2) * 128;
  const size_t raw_bytes = static_cast<size_t>(kRows) * (type == DSQ_Q8_0 ? 272 : 144);
  const size_t fixed = 1024 + barrier_bytes(kMaxSlots, 4);
  while (p.slots > 2 && fixed + p.slots * slot_b + 2 * raw_bytes > kSmemLimit) p.slots -= 2;
  p.slots_raw = static_cast<int>((kSmemLimit - fixed - p.slots * slot_b) / raw_bytes);
  if (p.slots_raw > 4) p.slots_raw = 4;
  p.smem = 1024 + p.slots * slot_b + p.slots_raw * raw_bytes + barrier_bytes(p.slots, p.slots_raw);
  if (pairs < 0) pairs = resident_pairs(type, p.tn, p.smem, sms);
  const int64_t tiles = p.tiles_m * p.tiles_n;
  // split K only when the tiles leave more than half the pairs idle
  p.splits = 1;
  while (tiles * p.splits * 2 <= pairs && p.splits * 2 <= kMaxKSplits && p.splits * 2 <= units) p.splits *= 2;
  p.units_per_split = (units + p.splits - 1) / p.splits;
  p.splits = (units + p.units_per_split - 1) / p.units_per_split;
  p.total_tiles = tiles * p.splits;
  p.head_tiles = p.total_tiles;
  p.tail_tiles = 0;
  p.tail_splits = 1;
  p.tail_ups = units;
  // Last-wave split: tiles that fill whole waves of pairs and a last wave at
  // most a quarter full leave most pairs idle for a whole tile.  Splitting
  // the last wave's tiles s ways in K (s * tail <= pairs, so the pieces are
  // one wave) cuts that wave to ceil(units / s) units, at the price of the
  // pieces' partials and one more launch to sum them.  Estimates: a unit of
  // K takes ~1.6 us at 256 tokens per tile (measured, scaled with the
  // tokens, at least a quarter of it); the sum re-reads the partials at
  // ~6 TB/s after ~2 us of launch.  A fuller last wave does not pay: with
  // 34 of 74 pairs busy (Q8_0, 8192 rows, 2048 tokens) its tiles already
  // finish early, and the split measured 13 % slower; with 12 of 74 (two
  // Q4_K weights of 4096 + 1024 rows, 2048 tokens) it measured 11 % faster.
  if (p.splits == 1 && tiles > pairs) {
    const int64_t tail = tiles % pairs;
    if (tail > 0 && 4 * tail <= pairs) {
      int s = static_cast<int>(pairs / tail);
      if (s > kMaxKSplits) s = kMaxKSplits;
      if (s > units) s = units;
      const int ups = (units + s - 1) / s;
      s = (units + ups - 1) / ups;
      const double unit_us = 1.6 * (p.tn >= 64 ? p.tn / 256.0 : 0.25);
      const double part_bytes = static_cast<double>(tail) * s * p.tn * kTileN * 4;
      if (s > 1 && (units - ups) * unit_us > 2.0 + part_bytes / 6.0e6) {
        p.head_tiles = tiles - tail;
        p.tail_tiles = static_cast<int>(tail);
        p.tail_splits = s;
        p.tail_ups = ups;
        p.total_tiles = p.head_tiles + tail * s;
      }
    }
  }
  p.grid = static_cast<unsigned>(2 * (p.total_tiles < pairs ? p.total_tiles : pairs));
  // the fp16 activation buffer is padded with zero rows to whole token tiles
  p.m_pad = p.tiles_m * p.tn;
  p.x16_bytes = align_up(static_cast<size_t>(p.m_pad) * K * 2, 1024);
  p.shift_off = p.x16_bytes;
  p.part_off = align_up(p.shift_off + static_cast<size_t>(p.m_pad) * 4, 1024);
  // split-K partials: per weight, splits x (M x N_g rounded up to 4 floats)
  size_t off = p.part_off;
  for (int g = 0; g < G; ++g) {
    p.split_stride[g] = static_cast<int64_t>(align_up(static_cast<size_t>(M) * N[g], 4));
    p.part_g_off[g] = off;
    if (p.splits > 1) off += static_cast<size_t>(p.splits) * p.split_stride[g] * 4;
  }
  // last-wave partials: one tn x 256 block per piece
  p.tail_off = align_up(off, 1024);
  if (p.tail_splits > 1)
    off = p.tail_off + static_cast<size_t>(p.tail_tiles) * p.tail_splits * p.tn * kTileN * 4;
  p.total = off;
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

template <int TYPE, bool TAIL>
int launch_gemm(const WeightMaps &maps, const PrefillArgs &args, const Plan &p, cudaStream_t stream) {
  const void *kern = reinterpret_cast<const void *>(prefill_kernel<TYPE, TAIL>);
  const int rc = set_smem_once(kern, static_cast<int>(p.smem), "prefill");
  if (rc != DSQ_OK) return rc;
  const cudaError_t e = launch_pair<TYPE, TAIL>(maps, args, p.grid, p.smem, stream);
  if (e != cudaSuccess) return fail(DSQ_ERR_LAUNCH, "dsq_gemm_prefill: gemm: %s", cudaGetErrorString(e));
  return after_launch("dsq_gemm_prefill: gemm");
}

}  // namespace
}  // namespace dsq

namespace dsq {
namespace {

// ---- small-M bridge: plan and launch ----
// The workspace the small-M kernel asks for (it keeps its activations in
// shared memory and needs none; a token amount keeps the API uniform).
constexpr size_t kSmallWorkspace = 256;

size_t small_act_bytes(int64_t K, int64_t M) { return static_cast<size_t>(M) * K * 4; }

// Where the CUDA-core kernel beats the mma.sync bridge above it (interleaved
// A/B on one B200, K = 4096): one token only.  At 2 tokens the bridge takes
// Q4_K 4096 rows in 10.1 against 10.6 us (16384 rows: 26.5 against 30.7)
// and Q8_0 8192 rows in 15.1 against 17.3 us (1024 rows: 9.0 against 9.4).
int small_max_m(int) { return 1; }   // at most kSmallMaxM

bool small_fits(int type, int64_t K, int64_t M) {
  return M >= 1 && M <= small_max_m(type) && small_act_bytes(K, M) <= kSmallMaxActSmem;
}

template <int TYPE, int M>
cudaError_t small_launch(const WeightMaps &maps, const SmallArgs &a, unsigned grid, size_t smem, cudaStream_t st) {
  return launch_pdl(prefill_small_kernel<TYPE, M>, dim3(grid), dim3(kSmallWarps * 32), smem, st, maps, a);
}

// small_max_m is 1: the kernel is instantiated for a single token (the
// template takes up to kSmallMaxM).
template <int TYPE>
const void *small_kernel_ptr(int) {
  return reinterpret_cast<const void *>(prefill_small_kernel<TYPE, 1>);
}

template <int TYPE>
cudaError_t small_dispatch(int, const WeightMaps &maps, const SmallArgs &a, unsigned grid, size_t smem,
                           cudaStream_t st) {
  return small_launch<TYPE, 1>(maps, a, grid, smem, st);
}

int run_prefill_small(const char *name, int type, int G, const void *const *w, const int64_t *N, int64_t K,
                      const float *x, int64_t M, float *const *y, void *workspace, size_t workspace_bytes,
                      const WaitCtl &ctl, int sms, cudaStream_t st) {
  DSQ_REQUIRE(workspace != nullptr && workspace_bytes >= kSmallWorkspace, DSQ_ERR_WORKSPACE,
              "%s: workspace of %zu bytes needed, %zu given", name, kSmallWorkspace, workspace_bytes);
  DSQ_REQUIRE(aligned(workspace, 256), DSQ_ERR_ALIGNMENT, "%s: workspace must be 256-byte aligned", name);
  SmallArgs a{};
  a.K = K;
  a.M = M;
  a.G = G;
  int64_t g0 = 0;
  for (int g = 0; g < kMaxGroup; ++g) {
    const bool used = g < G;
    a.N[g] = used ? N[g] : 1;
    a.y[g] = used ? y[g] : nullptr;
    a.group0[g] = g0;
    if (used) g0 += (N[g] + kSmallRows - 1) / kSmallRows;
  }
  a.group0[kMaxGroup] = g0;
  a.total_groups = g0;
  a.x = x;
  a.nunits = static_cast<int>(K / 256);
  a.box_bytes = static_cast<uint32_t>(kSmallRows * (type == DSQ_Q8_0 ? 272 : 144));
  a.wait = ctl;
  // shared memory: activations [M][K] fp32 | ring (8 warps x stages x box) |
  // barriers | reduction [2][8][M][32]
  const size_t act = align_up(small_act_bytes(K, M), 1024);
  const size_t bars = align_up((1 + 2 * kSmallWarps + 1) * sizeof(uint64_t), 128);
  const size_t red = 2 * static_cast<size_t>(kSmallWarps) * M * 32 * sizeof(float);
  const size_t fixed = 1024 + act + bars + red + 2 * kSmallMaxM * sizeof(float);
  const size_t per_stage = static_cast<size_t>(kSmallWarps) * a.box_bytes;
  int stages = fixed < kSmallPipeSmem ? static_cast<int>((kSmallPipeSmem - fixed) / per_stage) : 0;
  if (stages > 2) stages = 2;
  DSQ_REQUIRE(stages >= 1, DSQ_ERR_SHAPE, "%s: no pipeline fits next to %lld tokens of K=%lld", name, (long long)M,
              (long long)K);
  a.stages = stages;
  a.ring_off = static_cast<uint32_t>(act);
  a.bar_off = static_cast<uint32_t>(act + per_stage * stages);
  a.red_off = static_cast<uint32_t>(a.bar_off + bars);
  const size_t smem = 1024 + a.red_off + red;

  auto enc = encode_fn();
  DSQ_REQUIRE(enc != nullptr, DSQ_ERR_CUDA, "%s: cuTensorMapEncodeTiled unavailable", name);
  WeightMaps maps;
  const int64_t rb = static_cast<int64_t>(dsq_row_bytes(type, K));
  for (int g = 0; g < G; ++g) {
    const cuuint64_t gdim[2] = {static_cast<cuuint64_t>(rb / 4), static_cast<cuuint64_t>(N[g])};
    const cuuint64_t gstride[1] = {static_cast<cuuint64_t>(rb)};
    const cuuint32_t box[2] = {type == DSQ_Q8_0 ? 68u : 36u, static_cast<cuuint32_t>(kSmallRows)};
    const cuuint32_t estride[2] = {1u, 1u};
    const CUresult cr = enc(&maps.m[g], CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void *>(w[g]), gdim, gstride,
                            box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    DSQ_REQUIRE(cr == CUDA_SUCCESS, DSQ_ERR_CUDA, "%s: weight tensor map %d (%d)", name, g, (int)cr);
  }
  for (int g = G; g < kMaxGroup; ++g) maps.m[g] = maps.m[0];
  const int mi = static_cast<int>(M);
  const int rc = set_smem_once(type == DSQ_Q8_0 ? small_kernel_ptr<DSQ_Q8_0>(mi) : small_kernel_ptr<DSQ_Q4_K>(mi),
                               static_cast<int>(smem), name);
  if (rc != DSQ_OK) return rc;
  const unsigned grid = static_cast<unsigned>(a.total_groups < sms ? a.total_groups : sms);
  const cudaError_t e = type == DSQ_Q8_0 ? small_dispatch<DSQ_Q8_0>(mi, maps, a, grid, smem, st)
                                         : small_dispatch<DSQ_Q4_K>(mi, maps, a, grid, smem, st);
  if (e != cudaSuccess) return fail(DSQ_ERR_LAUNCH, "%s: %s", name, cudaGetErrorString(e));
  return after_launch(name);
}

// ---- 4 to 8 tokens on mma.sync: plan and launch ----
// Workspace: the rounded activations [8][K] binary16 (rows >= M zero), then
// the row shifts.
size_t small_mma_workspace(int64_t K) { return align_up(static_cast<size_t>(8) * K * 2, 256) + 256; }

// Shared memory of the mma.sync form for `stages` ring slots per warp:
// activations [K/2][8] words | ring | barriers | reduction [2][8][M][32] |
// Q4_K scale scratch.
size_t small_mma_smem(int type, int64_t K, int64_t M, int stages, SmallArgs *a) {
  const size_t nw = static_cast<size_t>(small_mma_warps(type));
  const size_t act = align_up(static_cast<size_t>(K) * 16, 1024);
  const size_t box = static_cast<size_t>(kSmallRows) * (type == DSQ_Q8_0 ? 272 : 144);
  const size_t bars = align_up((2 * nw + 1) * sizeof(uint64_t), 128);
  const size_t red = static_cast<size_t>(small_mma_red_bufs(type)) * nw * M * 32 * sizeof(float);
  const size_t scr = type == DSQ_Q4_K ? nw * kSmallRows * kScrStride * 4 : 0;
  if (a) {
    a->box_bytes = static_cast<uint32_t>(box);
    a->ring_off = static_cast<uint32_t>(act);
    a->bar_off = static_cast<uint32_t>(act + nw * box * stages);
    a->red_off = static_cast<uint32_t>(a->bar_off + bars);
    a->sc_off = static_cast<uint32_t>(a->red_off + red);
  }
  return 1024 + act + nw * box * stages + bars + red + scr;
}

// Where the mma.sync form takes the call: above the CUDA-core bridge, up to 8
// tokens, with its ring slots next to its activations.
bool small_mma_fits(int type, int64_t K, int64_t M) {
  return M > small_max_m(type) && M <= kSmallMmaMaxM &&
         small_mma_smem(type, K, M, small_mma_stages(type), nullptr) <= kSmallPipeSmem;
}

template <int TYPE>
const void *small_mma_kernel_ptr(int M) {
  switch (M) {
    case 1: return reinterpret_cast<const void *>(prefill_small_mma_kernel<TYPE, 1>);
    case 2: return reinterpret_cast<const void *>(prefill_small_mma_kernel<TYPE, 2>);
    case 3: return reinterpret_cast<const void *>(prefill_small_mma_kernel<TYPE, 3>);
    case 4: return reinterpret_cast<const void *>(prefill_small_mma_kernel<TYPE, 4>);
    case 5: return reinterpret_cast<const void *>(prefill_small_mma_kernel<TYPE, 5>);
    case 6: return reinterpret_cast<const void *>(prefill_small_mma_kernel<TYPE, 6>);
    case 7: return reinterpret_cast<const void *>(prefill_small_mma_kernel<TYPE, 7>);
    default: return reinterpret_cast<const void *>(prefill_small_mma_kernel<TYPE, 8>);
  }
}

template <int TYPE, int M>
cudaError_t small_mma_launch(const WeightMaps &maps, const SmallArgs &a, unsigned grid, size_t smem, cudaStream_t st) {
  return launch_pdl(prefill_small_mma_kernel<TYPE, M>, dim3(grid), dim3(small_mma_warps(TYPE) * 32), smem, st, maps,
                    a);
}

template <int TYPE>
cudaError_t small_mma_dispatch(int M, const WeightMaps &maps, const SmallArgs &a, unsigned grid, size_t smem,
                               cudaStream_t st) {
  switch (M) {
    case 1: return small_mma_launch<TYPE, 1>(maps, a, grid, smem, st);
    case 2: return small_mma_launch<TYPE, 2>(maps, a, grid, smem, st);
    case 3: return small_mma_launch<TYPE, 3>(maps, a, grid, smem, st);
    case 4: return small_mma_launch<TYPE, 4>(maps, a, grid, smem, st);
    case 5: return small_mma_launch<TYPE, 5>(maps, a, grid, smem, st);
    case 6: return small_mma_launch<TYPE, 6>(maps, a, grid, smem, st);
    case 7: return small_mma_launch<TYPE, 7>(maps, a, grid, smem, st);
    default: return small_mma_launch<TYPE, 8>(maps, a, grid, smem, st);
  }
}

int run_prefill_small_mma(const char *name, int type, int G, const void *const *w, const int64_t *N, int64_t K,
                          const float *x, int64_t M, float *const *y, void *workspace, size_t workspace_bytes,
                          const WaitCtl &ctl, int sms, cudaStream_t st) {
  const size_t need = small_mma_workspace(K);
  DSQ_REQUIRE(workspace != nullptr && workspace_bytes >= need, DSQ_ERR_WORKSPACE,
              "%s: workspace of %zu bytes needed, %zu given", name, need, workspace_bytes);
  DSQ_REQUIRE(aligned(workspace, 256), DSQ_ERR_ALIGNMENT, "%s: workspace must be 256-byte aligned", name);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  __half *x16 = reinterpret_cast<__half *>(ws);
  int32_t *shift = reinterpret_cast<int32_t *>(ws + need - 256);
  SmallArgs a{};
  a.K = K;
  a.M = M;
  a.G = G;
  int64_t g0 = 0;
  for (int g = 0; g < kMaxGroup; ++g) {
    const bool used = g < G;
    a.N[g] = used ? N[g] : 1;
    a.y[g] = used ? y[g] : nullptr;
    a.group0[g] = g0;
    if (used) g0 += (N[g] + kSmallRows - 1) / kSmallRows;
  }
  a.group0[kMaxGroup] = g0;
  a.total_groups = g0;
  a.x16 = x16;
  a.shift = shift;
  a.nunits = static_cast<int>(K / 256);
  a.wait = ctl;
  a.stages = small_mma_stages(type);
  const size_t smem = small_mma_smem(type, K, M, a.stages, &a);
  DSQ_REQUIRE(smem <= kSmallPipeSmem, DSQ_ERR_SHAPE, "%s: no pipeline fits next to the activations of K=%lld", name,
              (long long)K);

  auto enc = encode_fn();
  DSQ_REQUIRE(enc != nullptr, DSQ_ERR_CUDA, "%s: cuTensorMapEncodeTiled unavailable", name);
  WeightMaps maps;
  const int64_t rb = static_cast<int64_t>(dsq_row_bytes(type, K));
  for (int g = 0; g < G; ++g) {
    const cuuint64_t gdim[2] = {static_cast<cuuint64_t>(rb / 4), static_cast<cuuint64_t>(N[g])};
    const cuuint64_t gstride[1] = {static_cast<cuuint64_t>(rb)};
    const cuuint32_t box[2] = {type == DSQ_Q8_0 ? 68u : 36u, static_cast<cuuint32_t>(kSmallRows)};
    const cuuint32_t estride[2] = {1u, 1u};
    const CUresult cr = enc(&maps.m[g], CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void *>(w[g]), gdim, gstride,
                            box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    DSQ_REQUIRE(cr == CUDA_SUCCESS, DSQ_ERR_CUDA, "%s: weight tensor map %d (%d)", name, g, (int)cr);
  }
  for (int g = G; g < kMaxGroup; ++g) maps.m[g] = maps.m[0];

  // the activation rounding of the tensor-core path, row-major, 8 rows
  cudaError_t e = launch_pdl(x_to_f16_kernel<false>, dim3(8u), dim3(256), 0, st, x, M, K, int64_t(8), x16, shift);
  if (e != cudaSuccess) return fail(DSQ_ERR_LAUNCH, "%s: x_to_f16: %s", name, cudaGetErrorString(e));
  int rc = after_launch(name);
  if (rc != DSQ_OK) return rc;
  const int mi = static_cast<int>(M);
  rc = set_smem_once(type == DSQ_Q8_0 ? small_mma_kernel_ptr<DSQ_Q8_0>(mi) : small_mma_kernel_ptr<DSQ_Q4_K>(mi),
                     static_cast<int>(smem), name);
  if (rc != DSQ_OK) return rc;
  const unsigned grid = static_cast<unsigned>(a.total_groups < sms ? a.total_groups : sms);
  e = type == DSQ_Q8_0 ? small_mma_dispatch<DSQ_Q8_0>(mi, maps, a, grid, smem, st)
                       : small_mma_dispatch<DSQ_Q4_K>(mi, maps, a, grid, smem, st);
  if (e != cudaSuccess) return fail(DSQ_ERR_LAUNCH, "%s: %s", name, cudaGetErrorString(e));
  return after_launch(name);
}

// Argument checks shared by the prefill entry points (nothing launched on
// failure).
int validate_group(const char *name, int type, int64_t G, const void *const *w, const int64_t *N, int64_t K,
                   const float *x, int64_t M, float *const *y) {
  DSQ_REQUIRE(G >= 1 && G <= kMaxGroup, DSQ_ERR_INVALID_ARG, "%s: G=%lld weights (1..%d supported)", name,
              (long long)G, kMaxGroup);
  DSQ_REQUIRE(w && N && y, DSQ_ERR_INVALID_ARG, "%s: null weight, size or output array", name);
  int64_t total = 0;
  for (int64_t g = 0; g < G; ++g) {
    const int rc = validate(name, type, w[g], N[g], K, x, M);
    if (rc != DSQ_OK) return rc;
    DSQ_REQUIRE(y[g] != nullptr, DSQ_ERR_INVALID_ARG, "%s: null output %lld", name, (long long)g);
    DSQ_REQUIRE(aligned(y[g], 16), DSQ_ERR_ALIGNMENT, "%s: y must be 16-byte aligned", name);
    total += N[g];
  }
  DSQ_REQUIRE(total <= (int64_t(1) << 24), DSQ_ERR_SHAPE, "%s: the weights hold more than 2^24 rows", name);
  return DSQ_OK;
}

size_t group_workspace_bytes(int type, int64_t G, const int64_t *N, int64_t K, int64_t M) {
  if ((type != DSQ_Q8_0 && type != DSQ_Q4_K) || G < 1 || G > kMaxGroup || N == nullptr || M < 1 || K < 256 ||
      K % 256 != 0)
    return 0;
  for (int64_t g = 0; g < G; ++g)
    if (N[g] < 1) return 0;
  if (small_fits(type, K, M)) return kSmallWorkspace;
  if (small_mma_fits(type, K, M)) return small_mma_workspace(K);
  int sms = 148;
  if (device_ready(nullptr, &sms) != DSQ_OK) sms = 148;
  return make_plan(type, static_cast<int>(G), N, K, M, sms, -1).total;
}

// One activation conversion, one GEMM launch over the tiles of all G weights,
// and (when K is split) one in-order reduction per weight.
int run_prefill(const char *name, int type, int64_t G, const void *const *w, const int64_t *N, int64_t K,
                const float *x, int64_t M, float *const *y, void *workspace, size_t workspace_bytes,
                cudaStream_t st) {
  int rc = validate_group(name, type, G, w, N, K, x, M, y);
  if (rc != DSQ_OK) return rc;
  WaitCtl ctl;
  int sms = 0;
  rc = wait_ctl(&ctl, &sms);
  if (rc != DSQ_OK) return rc;
  const int Gi = static_cast<int>(G);
  if (small_fits(type, K, M))
    return run_prefill_small(name, type, Gi, w, N, K, x, M, y, workspace, workspace_bytes, ctl, sms, st);
  if (small_mma_fits(type, K, M))
    return run_prefill_small_mma(name, type, Gi, w, N, K, x, M, y, workspace, workspace_bytes, ctl, sms, st);
  const Plan p = make_plan(type, Gi, N, K, M, sms, -1);
  DSQ_REQUIRE(p.total_tiles < (int64_t(1) << 31), DSQ_ERR_SHAPE, "%s: %lld tiles exceed one launch", name,
              static_cast<long long>(p.total_tiles));
  DSQ_REQUIRE(workspace != nullptr && workspace_bytes >= p.total, DSQ_ERR_WORKSPACE,
              "%s: workspace of %zu bytes needed, %zu given", name, p.total, workspace_bytes);
  DSQ_REQUIRE(aligned(workspace, 256), DSQ_ERR_ALIGNMENT, "%s: workspace must be 256-byte aligned", name);
  DSQ_REQUIRE(p.smem <= kSmemLimit && p.slots >= 2 && p.slots_raw >= 2, DSQ_ERR_SHAPE, "%s: no pipeline fits",
              name);

  uint8_t *ws = static_cast<uint8_t *>(workspace);
  __half *x16 = reinterpret_cast<__half *>(ws);
  int32_t *shift = reinterpret_cast<int32_t *>(ws + p.shift_off);

  // raw weight units: the packed rows viewed as uint32 [N][row_bytes/4], one
  // 256-element unit (68 or 36 words) x 128 rows per box; rows past N read as
  // zero (a zero block dequantizes to zero).  The kernel reads the weights
  // only through these maps.
  auto enc = encode_fn();
  DSQ_REQUIRE(enc != nullptr, DSQ_ERR_CUDA, "%s: cuTensorMapEncodeTiled unavailable", name);
  WeightMaps maps;
  const int64_t rb = static_cast<int64_t>(dsq_row_bytes(type, K));
  for (int g = 0; g < Gi; ++g) {
    const cuuint32_t unit_words = type == DSQ_Q8_0 ? 68u : 36u;
    const cuuint64_t gdim[2] = {static_cast<cuuint64_t>(rb / 4), static_cast<cuuint64_t>(N[g])};
    const cuuint64_t gstride[1] = {static_cast<cuuint64_t>(rb)};
    const cuuint32_t box[2] = {unit_words, static_cast<cuuint32_t>(kRows)};
    const cuuint32_t estride[2] = {1u, 1u};
    const CUresult cr = enc(&maps.m[g], CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void *>(w[g]), gdim, gstride,
                            box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    DSQ_REQUIRE(cr == CUDA_SUCCESS, DSQ_ERR_CUDA, "%s: weight tensor map %d (%d)", name, g, (int)cr);
  }
  for (int g = Gi; g < kMaxGroup; ++g) maps.m[g] = maps.m[0];

  cudaError_t e = launch_pdl(x_to_f16_kernel<true>, dim3(static_cast<unsigned>(p.m_pad)), dim3(256), 0, st, x, M, K,
                             static_cast<int64_t>(p.tn / 2), x16, shift);
  if (e != cudaSuccess) return fail(DSQ_ERR_LAUNCH, "%s: x_to_f16: %s", name, cudaGetErrorString(e));
  rc = after_launch(name);
  if (rc != DSQ_OK) return rc;

  PrefillArgs args{};
  args.K = K;
  args.M = M;
  args.G = Gi;
  int64_t t0 = 0;
  for (int g = 0; g < kMaxGroup; ++g) {
    const bool used = g < Gi;
    args.N[g] = used ? N[g] : 1;
    args.y[g] = used ? (p.splits > 1 ? reinterpret_cast<float *>(ws + p.part_g_off[g]) : y[g]) : nullptr;
    args.split_stride[g] = used ? p.split_stride[g] : 0;
    args.tile_n0[g] = t0;
    if (used) t0 += (N[g] + kTileN - 1) / kTileN;
  }
  args.tile_n0[kMaxGroup] = t0;
  args.x16 = x16;
  args.shift = shift;
  args.units_per_split = p.units_per_split;
  args.splits = p.splits;
  args.tn = p.tn;
  args.slots = p.slots;
  args.slots_raw = p.slots_raw;
  args.tiles_m = p.tiles_m;
  args.tiles_n = p.tiles_n;
  args.total_tiles = p.total_tiles;
  args.head_tiles = p.head_tiles;
  args.tail_tiles = p.tail_tiles;
  args.tail_splits = p.tail_splits;
  args.tail_ups = p.tail_ups;
  args.tail_part = p.tail_splits > 1 ? reinterpret_cast<float *>(ws + p.tail_off) : nullptr;
  args.wait = ctl;
  if (p.tail_splits > 1)
    rc = type == DSQ_Q8_0 ? launch_gemm<DSQ_Q8_0, true>(maps, args, p, st)
                          : launch_gemm<DSQ_Q4_K, true>(maps, args, p, st);
  else
    rc = type == DSQ_Q8_0 ? launch_gemm<DSQ_Q8_0, false>(maps, args, p, st)
                          : launch_gemm<DSQ_Q4_K, false>(maps, args, p, st);
  if (rc != DSQ_OK) return rc;
  if (p.splits > 1) {
    for (int g = 0; g < Gi; ++g) {
      const int64_t total = M * N[g];
      const int64_t blocks = (total / 4 + 255) / 256 + 1;
      const unsigned grid = static_cast<unsigned>(blocks < 8 * sms ? blocks : 8 * sms);
      e = launch_pdl(splitk_reduce_kernel, dim3(grid), dim3(256), 0, st,
                     static_cast<const float *>(reinterpret_cast<float *>(ws + p.part_g_off[g])), total,
                     p.split_stride[g], p.splits, y[g]);
      if (e != cudaSuccess) return fail(DSQ_ERR_LAUNCH, "%s: reduce: %s", name, cudaGetErrorString(e));
      rc = after_launch(name);
      if (rc != DSQ_OK) return rc;
    }
  }
  if (p.tail_splits > 1) {
    const int64_t total4 = static_cast<int64_t>(p.tail_tiles) * p.tn * (kTileN / 4);
    const int64_t blocks = (total4 + 255) / 256;
    const unsigned grid = static_cast<unsigned>(blocks < 8 * sms ? blocks : 8 * sms);
    e = launch_pdl(tail_reduce_kernel, dim3(grid), dim3(256), 0, st, args);
    if (e != cudaSuccess) return fail(DSQ_ERR_LAUNCH, "%s: last-wave reduce: %s", name, cudaGetErrorString(e));
    rc = after_launch(name);
    if (rc != DSQ_OK) return rc;
  }
  return DSQ_OK;
}

}  // namespace
}  // namespace dsq

extern "C" size_t dsq_prefill_workspace_bytes(int type, int64_t N, int64_t K, int64_t M) {
  return dsq::group_workspace_bytes(type, 1, &N, K, M);
}

extern "C" size_t dsq_prefill_grouped_workspace_bytes(int type, int64_t G, const int64_t *N, int64_t K, int64_t M) {
  return dsq::group_workspace_bytes(type, G, N, K, M);
}

extern "C" int dsq_gemm_prefill(int type, const void *w, int64_t N, int64_t K, const float *x, int64_t M, float *y,
                                void *workspace, size_t workspace_bytes, void *stream) {
  using namespace dsq;
  DSQ_REQUIRE(y != nullptr, DSQ_ERR_INVALID_ARG, "dsq_gemm_prefill: null output");
  const void *ws_[1] = {w};
  float *ys_[1] = {y};
  return run_prefill("dsq_gemm_prefill", type, 1, ws_, &N, K, x, M, ys_, workspace, workspace_bytes,
                     as_stream(stream));
}

extern "C" int dsq_gemm_prefill_grouped(int type, int64_t G, const void *const *w, const int64_t *N, int64_t K,
                                        const float *x, int64_t M, float *const *y, void *workspace,
                                        size_t workspace_bytes, void *stream) {
  using namespace dsq;
  return run_prefill("dsq_gemm_prefill_grouped", type, G, w, N, K, x, M, y, workspace, workspace_bytes,
                     as_stream(stream));
}

extern "C" int dsq_test_prefill_operands(int type, const void *w, int64_t N, int64_t K, const float *x, int64_t M,
                                         uint16_t *x16, int32_t *shift, uint16_t *w16, void *stream) {
  using namespace dsq;
  int rc = validate("dsq_test_prefill_operands", type, w, N, K, x, M);
  if (rc != DSQ_OK) return rc;
  DSQ_REQUIRE(x16 && shift && w16, DSQ_ERR_INVALID_ARG, "dsq_test_prefill_operands: null output");
  DSQ_REQUIRE(aligned(x16, 16) && aligned(w16, 16) && aligned(shift, 4), DSQ_ERR_ALIGNMENT,
              "dsq_test_prefill_operands: output alignment");
  uint32_t *status = nullptr;
  rc = device_ready(&status, nullptr);
  if (rc != DSQ_OK) return rc;
  cudaStream_t st = as_stream(stream);
  x_to_f16_kernel<false><<<static_cast<unsigned>(M), 256, 0, st>>>(x, M, K, M, reinterpret_cast<__half *>(x16), shift);
  rc = after_launch("dsq_test_prefill_operands: x");
  if (rc != DSQ_OK) return rc;
  const int64_t work = N * (K / 256);
  const unsigned grid = static_cast<unsigned>((work + 127) / 128);
  const int64_t rb = static_cast<int64_t>(dsq_row_bytes(type, K));
  if (type == DSQ_Q8_0)
    w_to_f16_kernel<DSQ_Q8_0><<<grid, 128, 0, st>>>(static_cast<const uint8_t *>(w), N, K, rb, w16, status);
  else
    w_to_f16_kernel<DSQ_Q4_K><<<grid, 128, 0, st>>>(static_cast<const uint8_t *>(w), N, K, rb, w16, status);
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
// Device address of g_prefill_scratch, per device, with the id of the CUDA
// context it was looked up in: a new context (cudaDeviceReset, or a driver
// context the caller made current) maps the array elsewhere, so the address
// is looked up again once in it.
struct ScratchAddr {
  uint64_t ctx = 0;
  void *addr = nullptr;
};
ScratchAddr g_scratch_addr[kMaxDevices];
}  // namespace
}  // namespace dsq

extern "C" int dsq_gemm_prefill_noalloc(int type, const void *w, int64_t N, int64_t K, const float *x, int64_t M,
                                        float *y, void *stream) {
  using namespace dsq;
  // the argument checks of dsq_gemm_prefill come first, so a bad argument is
  // named as such even when the problem would also be too large
  int rc = validate("dsq_gemm_prefill_noalloc", type, w, N, K, x, M);
  if (rc != DSQ_OK) return rc;
  DSQ_REQUIRE(y != nullptr, DSQ_ERR_INVALID_ARG, "dsq_gemm_prefill_noalloc: null output");
  DSQ_REQUIRE(aligned(y, 16), DSQ_ERR_ALIGNMENT, "dsq_gemm_prefill_noalloc: y must be 16-byte aligned");
  const size_t need = dsq_prefill_workspace_bytes(type, N, K, M);
  DSQ_REQUIRE(need <= DSQ_PREFILL_NOALLOC_SCRATCH_BYTES, DSQ_ERR_WORKSPACE,
              "dsq_gemm_prefill_noalloc: this problem needs %zu bytes of scratch but the built-in scratch holds "
              "%llu bytes (M x K x 2 bytes of fp16 activations plus split-K partials must fit); use "
              "dsq_gemm_prefill with a caller-provided workspace",
              need, (unsigned long long)DSQ_PREFILL_NOALLOC_SCRATCH_BYTES);
  int dev = -1;
  uint64_t ctx = 0;
  rc = current_context(&dev, &ctx);
  if (rc != DSQ_OK) return rc;
  void *scratch = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    ScratchAddr &sa = g_scratch_addr[dev];
    if (sa.ctx != ctx) {
      // One-time set-up in this context (its device is current): the host
      // name of the array is only a stand-in, so fetch its device address.
      void *p = nullptr;
      const cudaError_t e = cudaGetSymbolAddress(&p, g_prefill_scratch);
      DSQ_REQUIRE(e == cudaSuccess && p != nullptr, DSQ_ERR_CUDA,
                  "dsq_gemm_prefill_noalloc: cudaGetSymbolAddress of the scratch failed: %s", cudaGetErrorString(e));
      sa.addr = p;
      sa.ctx = ctx;
    }
    scratch = sa.addr;
  }
  return dsq_gemm_prefill(type, w, N, K, x, M, y, scratch, static_cast<size_t>(DSQ_PREFILL_NOALLOC_SCRATCH_BYTES),
                          stream);
}
