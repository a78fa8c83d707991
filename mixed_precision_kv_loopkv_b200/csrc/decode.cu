// Fused LoopKV decode attention (sm_100a).
//
// LoopKV: Loop-Aware KV Cache Compression for Serving Looped Transformers,
// Abstract: each (loop, layer) cell is read at its planned precision (4-bit,
// 2-bit, or the final loop's cell reused); every token's high 2-bit value
// plane is read, and the low plane only where the cell's own attention
// weights need 4-bit precision; one fused kernel executes the plan.  The
// threshold reading used here: token t takes its low plane when its fp32
// softmax weight p_t >= tau.  Split-K over the context follows the
// streaming-softmax idea (O(1)-memory attention in the same pages' listing).
//
// Grid (splits, query heads, batch); the splits of one (sequence, head) form
// one thread-block cluster (with grouped queries and a low-plane selection,
// the splits of all query heads sharing a KV head, which OR their selections
// into one union).  Each CTA owns a chunk of 32-token groups:
//   - every warp streams its own groups (interleaved with the other warps)
//     through a private ring of shared-memory stages: lane 0 issues 1-D bulk
//     copies (TMA, no multicast) of each block record's pass-1 prefix (keys,
//     key meta, value high plane, value meta: 2048 B of the 2560-B 4-bit
//     record at D = 128), completion on an mbarrier per stage;
//   - the warp dequantises the keys at the cell's precision, forms the
//     logits, keeps an online softmax and accumulates the high-plane values
//     (a reuse cell's optional current token joins as one exact token);
//   - the splits exchange (max, sum) through distributed shared memory, so
//     every CTA knows the exact normaliser Z before any low-plane read;
//   - pass 2 re-reads the CTA's logits from shared memory, ballots the tokens
//     with p >= tau and gathers only their 32-byte low-plane rows, adding
//     p * scale * (lo - 1.5) per channel (turning the bucket midpoint into
//     the full 4-bit value);
//   - a cluster-wide reduction over distributed shared memory writes bf16 out
//     (kinds that cannot select push their sums with their (max, sum) table
//     entries and meet once: the owners rescale after that one barrier).
//
// Arithmetic of the inner loop.  Keys (one FP32x2 FMA per two codes): a
// code's bits are isolated in place with one AND and read as an fp32
// subnormal, code * 2^pos * 2^-149; the per-channel factor 2^(149 - pos - E)
// is folded into the query coefficient.  Subnormal FMA inputs are exact on
// this hardware (no FTZ), so every product equals q * scale * code up to the
// global power of two 2^-E, and the logits keep fp32 precision for the
// selection.  Values (dp2a, two tokens per instruction): the value plane is
// column-major within a block, so one word holds one 4-channel column of four
// tokens; each token's softmax weight becomes 16-bit fixed-point weights
// (one per 32-channel group, scaled to the group's own largest weight and the
// largest value scale seen), each lane sums its column over the group's 32
// tokens exactly in integers, and the sums are added in fp32.
#include <float.h>
#include <limits.h>

#include <algorithm>
#include <map>
#include <mutex>
#include <tuple>

#include "append_ops.cuh"
#include "device_common.cuh"
#include "kernels.h"

namespace loopkv {
namespace {

constexpr int kNW = 4;                 // warps per CTA, each streams its own groups
constexpr int kThreads = 32 * kNW;
constexpr int kExpOff = 64;            // E: key products live at 2^-64 of their size
constexpr size_t kMaxDynamicSmem = 227u * 1024u;  // opt-in dynamic shared memory of one CTA

__device__ __forceinline__ float pow2i(int e) { return __int_as_float((127 + e) << 23); }

// Field position (bits) of channel i of a 16-channel chunk.
// 2-bit plane word: channel i at bits 2i; i >= 11 is read from (w >> 22).
__host__ __device__ constexpr int pos2(int i) { return 2 * (i < 11 ? i : i - 11); }
// 4-bit nibble words (even/odd channels): channel i in nibble i/2;
// nibbles >= 5 are read from (w >> 20).
__host__ __device__ constexpr int pos4(int i) { return 4 * ((i >> 1) < 5 ? (i >> 1) : (i >> 1) - 5); }

// Subnormal view of field i of a 2-bit plane word.
__device__ __forceinline__ float fld2(uint32_t w, uint32_t w22, int i) {
  return i < 11 ? __uint_as_float(w & (3u << (2 * i))) : __uint_as_float(w22 & (3u << (2 * (i - 11))));
}
// Subnormal view of nibble m of a nibble word.
__device__ __forceinline__ float nib(uint32_t w, uint32_t w20, int m) {
  return m < 5 ? __uint_as_float(w & (15u << (4 * m))) : __uint_as_float(w20 & (15u << (4 * (m - 5))));
}
// Full 4-bit codes of 16 channels from their high and low plane words:
// even = channels 0,2,..,14 in nibbles 0..7; odd = channels 1,3,..,15.
// (a & c) | (b & ~c) in one LOP3
__device__ __forceinline__ uint32_t bit_select(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xE4;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ void combine_planes(uint32_t hi, uint32_t lo, uint32_t& even, uint32_t& odd) {
  even = bit_select(hi << 2, lo, 0xCCCCCCCCu);
  odd = bit_select(hi, lo >> 2, 0xCCCCCCCCu);
}

// Dot product of the subnormal code views of one 16-channel word with 8
// coefficient pairs (channels 2p, 2p+1), accumulated into acc (one chain;
// a lane interleaves the chains of its four tokens).
template <bool FOUR>
__device__ __forceinline__ float2 dot16(const float2* c, uint32_t a, uint32_t b, float2 acc) {
  if constexpr (FOUR) {  // a, b = high / low plane words
    uint32_t e, o;
    combine_planes(a, b, e, o);
    const uint32_t e20 = e >> 20, o20 = o >> 20;
#pragma unroll
    for (int m = 0; m < 8; ++m) acc = __ffma2_rn(c[m], make_float2(nib(e, e20, m), nib(o, o20, m)), acc);
  } else {  // a = 2-bit plane word
    const uint32_t a22 = a >> 22;
#pragma unroll
    for (int p = 0; p < 8; ++p) acc = __ffma2_rn(c[p], make_float2(fld2(a, a22, 2 * p), fld2(a, a22, 2 * p + 1)), acc);
  }
  return acc;
}

// Two-way integer dot products (unsigned): d = c + a.lo16 * b.byte0 + a.hi16 * b.byte1
// (lo) or ... * b.byte2, b.byte3 (hi).  a packs the fixed-point weights of two
// tokens, b the 2-bit codes (pre-shifted fields) of four tokens of one channel.
__device__ __forceinline__ uint32_t dp2a_lo(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("dp2a.lo.u32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ uint32_t dp2a_hi(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("dp2a.hi.u32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
// acc[f] += the four tokens' codes of channel 4 col + f, weighted by the two
// weight pairs a01 (tokens 0, 1 of the word) and a23 (tokens 2, 3).  Byte t
// of w holds token t's channels 4 col .. 4 col + 3 at bits 0-1, 2-3, 4-5,
// 6-7; field f is isolated in place by one AND and carries the factor 4^f
// (a byte of at most 192), undone when the group's sums are added up.
__device__ __forceinline__ void column_dot(uint32_t* acc, uint32_t w, uint32_t a01, uint32_t a23) {
  const uint32_t x0 = w & 0x03030303u, x1 = w & 0x0C0C0C0Cu;
  const uint32_t x2 = w & 0x30303030u, x3 = w & 0xC0C0C0C0u;
  acc[0] = dp2a_hi(a23, x0, dp2a_lo(a01, x0, acc[0]));
  acc[1] = dp2a_hi(a23, x1, dp2a_lo(a01, x1, acc[1]));
  acc[2] = dp2a_hi(a23, x2, dp2a_lo(a01, x2, acc[2]));
  acc[3] = dp2a_hi(a23, x3, dp2a_lo(a01, x3, acc[3]));
}
// Largest value over the warp (one instruction; NaN inputs are ignored).
__device__ __forceinline__ float warp_max_f32(float x) {
  float m;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(m) : "f"(x));
  return m;
}

// Index of the sequence with rank r when the batch is ordered by decreasing
// length, ties by increasing index (a bijection of [0, B)).  Batches of
// equal lengths, or of more than kMaxRankedBatch sequences, keep the
// identity.  Every lane of the warp must call it; lengths are compared as
// given (a bad length only moves that sequence in the order).
constexpr int kMaxRankedBatch = 64;
__device__ __forceinline__ int sequence_of_rank(const int32_t* seq_lens, int B, int r, int lane) {
  if (B > kMaxRankedBatch) return r;
  const int n0 = lane < B ? seq_lens[lane] : 0;
  const int n1 = lane + 32 < B ? seq_lens[lane + 32] : 0;
  const int mn = __reduce_min_sync(0xffffffffu, lane < B ? (lane + 32 < B ? min(n0, n1) : n0) : INT_MAX);
  const int mx = __reduce_max_sync(0xffffffffu, lane < B ? (lane + 32 < B ? max(n0, n1) : n0) : INT_MIN);
  if (mn == mx) return r;
  int found = -1;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int bb = lane + 32 * half;
    const int nb = half ? n1 : n0;
    int rank = 0;
    for (int i = 0; i < min(B, 32); ++i) {
      const int n2 = __shfl_sync(0xffffffffu, n0, i);
      rank += (n2 > nb) || (n2 == nb && i < bb);
    }
    for (int i = 32; i < B; ++i) {
      const int n2 = __shfl_sync(0xffffffffu, n1, i - 32);
      rank += (n2 > nb) || (n2 == nb && i < bb);
    }
    if (bb < B && rank == r) found = bb;
  }
  return __reduce_max_sync(0xffffffffu, found);
}

// The decode step's append of one token at position pos into (b, KV head h), run by
// every thread of the CTA that holds the token's group: the value row (both
// planes and meta) from v_new; the key either joins the exact residual or,
// as its group's 32nd token, completes the group, which is then quantised
// per channel from the residual.
template <int KIND, int D>
__device__ __forceinline__ void append_token(const DecodeParams& p, int b, int h, int pos, int warp, int lane) {
  using R = Rec<KIND, D>;
  const CellRows cell{p.wr_arena, p.block_table + static_cast<size_t>(b) * p.max_blocks, p.err, p.Hkv, h,
                      p.max_blocks, p.num_blocks};
  const __nv_bfloat16* kb = p.k_new + (static_cast<size_t>(b) * p.Hkv + h) * D;
  const __nv_bfloat16* vb = p.v_new + (static_cast<size_t>(b) * p.Hkv + h) * D;
  uint8_t* rec = record_at<KIND, D>(cell, pos);
  const int row = pos % kBlock;
  if constexpr (KIND == LOOPKV_CELL_BF16) {
    constexpr int kVec = D * 2 / 16;
    if (rec && static_cast<int>(threadIdx.x) < 2 * kVec) {
      const int c = threadIdx.x % kVec;
      const bool value = static_cast<int>(threadIdx.x) >= kVec;
      reinterpret_cast<uint4*>(rec + (value ? R::kBfV : R::kBfK) + row * D * 2)[c] =
          reinterpret_cast<const uint4*>(value ? vb : kb)[c];
    }
  } else {
    if (warp < D / kGroup) store_value_group<KIND, D>(rec, row, warp, __bfloat162float(vb[warp * kGroup + lane]), lane);
    __nv_bfloat16* res = p.wr_residual + (static_cast<size_t>(b) * p.Hkv + h) * kGroup * D;
    if (pos % kGroup == kGroup - 1) {
      store_key_group<KIND, D>(cell, pos / kGroup, lane == kGroup - 1 ? kb : res + lane * D, warp, lane, kNW);
    } else if (static_cast<int>(threadIdx.x) < D * 2 / 16) {
      reinterpret_cast<uint4*>(res + (pos % kGroup) * D)[threadIdx.x] = reinterpret_cast<const uint4*>(kb)[threadIdx.x];
    }
  }
}

template <int KIND, int D, bool FULLV>
struct Cfg {
  using R = Rec<KIND, D>;
  static constexpr bool kQuant = KIND != LOOPKV_CELL_BF16;
  static constexpr bool kQ4 = KIND == LOOPKV_CELL_Q4;
  // bytes of one block record streamed in pass 1
  static constexpr int kLoad = kQ4 ? (FULLV ? R::kBytes : R::kQ4VLo) : R::kBytes;
  // one 32-token group: two block prefixes, the second shifted by 64 B so the
  // same offsets of the two halves fall in different shared-memory banks
  static constexpr int kHalf = kLoad + 64;
  static constexpr int kStage = kHalf + kLoad;
  static constexpr int kNSW = 2;                           // ring stages per warp
  // keys: lane (r, k) takes channels kCW*k .. kCW*k + kCW - 1 of tokens r + 8j
  static constexpr int kCH = 4;                            // lanes per token
  static constexpr int kCW = D / kCH;                      // channels per lane
  static constexpr int kNWRD = kCW / 16;                   // plane words per lane and token
  static constexpr int kTS = 32 / kCH;                     // token sub-groups per warp
  static constexpr int kTPL = 32 / kTS;                    // tokens per lane per group
  static constexpr int kE = kQuant ? kExpOff : 0;
  // values: the plane is column-major within a block; lane (hb, col) takes
  // the 4 channels of column col (of the block hb for D = 64, of both blocks
  // for D = 128) for every token
  static constexpr int kCols = D / 4;                      // 4-channel columns
  static constexpr int kLPC = 32 / kCols;                  // lanes per column (1 or 2)
  static constexpr int kVG = D / kGroup;                   // value groups per token
  static constexpr bool kLogits = kQ4 && !FULLV;           // pass 2 needs the logits
  static constexpr bool kFourV = kQ4 && FULLV;             // full 4-bit values in pass 1
  // the streamed value codes count 4 x hi for a 4-bit cell: fixed-point
  // weights are scaled for 4 x scale
  static constexpr float kMult = kQ4 ? 4.f : 1.f;
};

// Shared-memory carve-up (bytes), identical on host and device.
// After pass 1 a warp's ring is idle and holds the warp's results: its
// per-channel sums (wres, at the ring's start) and its low-plane corrections
// (after them).  The exchange area (xchg) is never aliased: peers of the
// cluster store into it while this CTA may still be in pass 1.
//   xchg: table float4[8 * kNW] (every warp's max, sum, error bits),
//         red float[D] (the owner's slice sums of every split),
//         cnts int32[8] (every split's selection count)
struct Smem {
  size_t rings, ring_bytes, bars, qconst, q2buf, logits, ids, masks, gmax, xchg, scal, total;
};
// Per-warp buffer of 512 B, used twice per group: the key coefficients (128
// floats) while the keys are read, then the group's value weights
// (fixed-point u16 [2][D/32][32]: high and, for full 4-bit values, low plane;
// fp32 [32] for bf16 cells) once every lane has its logit.
constexpr int kWarpBufBytes = 512;
__host__ __device__ inline Smem smem_plan(int stage_bytes, int nsw, int cg, int d, bool logits) {
  Smem s;
  s.rings = 0;
  s.ring_bytes = static_cast<size_t>(stage_bytes) * nsw;
  s.bars = s.rings + s.ring_bytes * kNW;
  s.qconst = s.bars + 8 * nsw * kNW;                       // qf[D], qs[D]
  s.q2buf = s.qconst + static_cast<size_t>(8) * d;         // per warp: kWarpBufBytes
  s.logits = s.q2buf + static_cast<size_t>(kWarpBufBytes) * kNW;
  s.ids = s.logits + (logits ? 128 * static_cast<size_t>(cg) : 0);  // two block ids per group
  s.masks = s.ids + (logits ? 8 * static_cast<size_t>(cg) : 0);     // selection word per group
  s.gmax = s.masks + (logits ? 4 * static_cast<size_t>(cg) : 0);    // largest logit per group
  s.xchg = s.gmax + (logits ? 4 * static_cast<size_t>(cg) : 0);
  s.xchg = (s.xchg + 15) & ~static_cast<size_t>(15);
  s.scal = s.xchg + 16 * 8 * kNW + 4 * static_cast<size_t>(d) + 32;  // CTA scalars, warp counts
  s.total = s.scal + 32;
  return s;
}

// Per-CTA scalar slots.
enum { kSlotBad = 0, kSlotCnt0 = 4 };

// Largest exponent F of the fixed-point value weights (their scale before
// the first group sets it), and the largest gap (log2 units) between the
// running maximum and a group's own maximum that the group's weights are
// scaled up by.
constexpr int kMaxFixedExp = 100;
constexpr float kMaxGroupGap = 60.f;

// Per-lane running state of one warp's online softmax.  m is warp-uniform
// (log2 units); l and beta cover the token this lane owns in every group;
// facc holds the lane's value column (4 channels over every token of the
// warp's groups) in fp32.  Quantised cells carry each group's value weights
// in 16-bit fixed point, round(w * 2^d * scale * sF) with sF = kMult * 2^F
// warp-uniform and d the group's own gap below the running maximum, and add
// the group's exact integer column sums into facc.
template <int D>
struct WarpState {
  float m, l;
  float beta[D / kGroup];
  float facc[4];
  float sF, slim;  // scale of w * scale, and the largest value scale it admits (w <= 1)
  int F;
};

// Slot (in floats) of the 16-byte piece v (channels CW*k + 4v .. +3) in a
// warp's q2 buffer: per-chunk reads (fixed v, k = 0..3) hit distinct bank
// groups; the cooperative writes conflict at most two ways.
template <int CW>
__device__ __forceinline__ int q2_slot(int k, int v) { return v * 16 + ((k + v) & 3) * 4; }

// One 32-token group.  Lane (r, k), r = lane / 4, k = lane % 4: channels
// CW*k .. CW*k + CW - 1 of tokens r + 8j (j < 4).  TAIL: the sequence's
// unfinished key group: keys from the exact residual, tokens past the end
// masked.
template <int KIND, int D, bool FULLV, bool TAIL>
__device__ __forceinline__ void group_step(const uint8_t* st, const float* qconst, float* q2buf, uint8_t* vbuf,
                                           const float* qfr, const __nv_bfloat16* res, int tok0, int nn,
                                           int lane, int r, int k, float* logits_g, float* gmax_g,
                                           WarpState<D>& ws) {
  using C = Cfg<KIND, D, FULLV>;
  using R = typename C::R;
  constexpr int CH = C::kCH, CW = C::kCW, NWRD = C::kNWRD, TS = C::kTS, TPL = C::kTPL, HALF = C::kHalf;
  constexpr int VG = C::kVG, COLS = C::kCols, LPC = C::kLPC;
  const float esc = pow2i(C::kE);

  // this lane's plane words of token j: rowbase + a compile-time offset
  const uint8_t* rowbase = st + r * R::kRow + 4 * NWRD * k;
  auto tok_off = [](int j) { return ((TS * j) >> 4) * HALF + ((TS * j) & 15) * R::kRow; };
  auto plane_words = [&](int j, int section, uint32_t* w) {
    const uint8_t* a = rowbase + tok_off(j) + section;
    if constexpr (NWRD == 2) {
      const uint2 x = *reinterpret_cast<const uint2*>(a);
      w[0] = x.x;
      w[1] = x.y;
    } else {
      w[0] = *reinterpret_cast<const uint32_t*>(a);
    }
  };

  // ---- keys -> logits (scaled by 2^-E)
  float part[TPL];
  if constexpr (C::kQuant && !TAIL) {
    // cooperative key coefficients of this group: lane (r, k) prepares
    // channels CW*k + 4r .. +3 of its own quarter (contiguous meta), q2 =
    // qs * scale, and its share of alpha_k = sum over the quarter of qf_c *
    // min_c; the quarter's 32 coefficients are then read back by its lanes
    float alpha;
    {
      float a4 = 0.f;
      if (4 * r < CW) {
        const int c0 = CW * k + 4 * r;
        const uint4 mw = *reinterpret_cast<const uint4*>(st + ((c0 < D / 2) ? 0 : HALF) + R::kKMetaOff +
                                                         (c0 % (D / 2)) * 4);
        const float4 qfv = *reinterpret_cast<const float4*>(qconst + c0);
        const float4 qsv = *reinterpret_cast<const float4*>(qconst + D + c0);
        const float2 q01 = __fmul2_rn(make_float2(qsv.x, qsv.y), make_float2(bf16_lo(mw.x), bf16_lo(mw.y)));
        const float2 q23 = __fmul2_rn(make_float2(qsv.z, qsv.w), make_float2(bf16_lo(mw.z), bf16_lo(mw.w)));
        float2 a2 = __fmul2_rn(make_float2(qfv.x, qfv.y), make_float2(bf16_hi(mw.x), bf16_hi(mw.y)));
        a2 = __ffma2_rn(make_float2(qfv.z, qfv.w), make_float2(bf16_hi(mw.z), bf16_hi(mw.w)), a2);
        a4 = a2.x + a2.y;
        *reinterpret_cast<float4*>(q2buf + q2_slot<CW>(k, r)) = make_float4(q01.x, q01.y, q23.x, q23.y);
      }
      // the quarter's lanes share lane % 4: sum over r
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) a4 += __shfl_xor_sync(0xffffffffu, a4, o);
      alpha = a4;
    }
    __syncwarp();
    // every lane of a token row starts its partial logits from its quarter's
    // alpha_k, so the transposed all-reduce over the row adds alpha once
    alpha *= pow2i(-C::kE);
    float2 d[TPL];
#pragma unroll
    for (int j = 0; j < TPL; ++j) d[j] = make_float2(alpha, 0.f);
    // one 16-channel word at a time: only its 8 coefficient pairs are live
#pragma unroll
    for (int u = 0; u < NWRD; ++u) {
      float2 q2[8];
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const float4 x = *reinterpret_cast<const float4*>(q2buf + q2_slot<CW>(k, 4 * u + v));
        q2[2 * v] = make_float2(x.x, x.y);
        q2[2 * v + 1] = make_float2(x.z, x.w);
      }
#pragma unroll
      for (int j = 0; j < TPL; ++j) {
        uint32_t hi[NWRD], lo[NWRD] = {};
        plane_words(j, R::kKHi, hi);
        if constexpr (C::kQ4) plane_words(j, R::kQ4KLo, lo);
        d[j] = dot16<C::kQ4>(q2, hi[u], lo[u], d[j]);
      }
    }
#pragma unroll
    for (int j = 0; j < TPL; ++j) part[j] = d[j].x + d[j].y;
  } else if constexpr (C::kQuant) {
    // unfinished key group: exact bf16 keys from the residual
    const float* qf = qconst + CW * k;
#pragma unroll
    for (int j = 0; j < TPL; ++j) {
      const int t = r + TS * j;
      float d = 0.f;
      if (tok0 + t < nn) {
        const uint4* kp = reinterpret_cast<const uint4*>(res + t * D + CW * k);
        float2 s2 = make_float2(0.f, 0.f);
#pragma unroll
        for (int v = 0; v < CW / 8; ++v) {
          const uint4 a = kp[v];
          const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
          for (int i = 0; i < 4; ++i)
            s2 = __ffma2_rn(make_float2(qf[8 * v + 2 * i], qf[8 * v + 2 * i + 1]),
                            make_float2(bf16_lo(w[i]), bf16_hi(w[i])), s2);
        }
        d = (s2.x + s2.y) * pow2i(-C::kE);
      }
      part[j] = d;
    }
  } else {
#pragma unroll
    for (int j = 0; j < TPL; ++j) {
      const uint4* kp = reinterpret_cast<const uint4*>(st + ((TS * j) >> 4) * HALF + R::kBfK +
                                                       (r + ((TS * j) & 15)) * D * 2 + 2 * CW * k);
      float2 s2 = make_float2(0.f, 0.f);
#pragma unroll
      for (int v = 0; v < CW / 8; ++v) {
        const uint4 a = kp[v];
        const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
          s2 = __ffma2_rn(make_float2(qfr[8 * v + 2 * i], qfr[8 * v + 2 * i + 1]),
                          make_float2(bf16_lo(w[i]), bf16_hi(w[i])), s2);
      }
      part[j] = s2.x + s2.y;
    }
  }
  // ---- the logit of this lane's token tk = r + 8k: a transposed all-reduce
  //      over the 4 lanes of token row r, after which each lane keeps one
  //      token (k selects j = k among the row's tokens r + 8j)
  static_assert(CH == 4 && TPL == 4, "the transposed reduction assumes 4 lanes and 4 tokens per lane");
  float L;
  {
    const bool up = k & 2;
    const float s0 = up ? part[0] : part[2], s1 = up ? part[1] : part[3];
    const float k0 = up ? part[2] : part[0], k1 = up ? part[3] : part[1];
    const float q0 = k0 + __shfl_xor_sync(0xffffffffu, s0, 2);
    const float q1 = k1 + __shfl_xor_sync(0xffffffffu, s1, 2);
    const bool odd = k & 1;
    L = (odd ? q1 : q0) + __shfl_xor_sync(0xffffffffu, odd ? q0 : q1, 1);
  }
  const int tk = r + TS * k;
  const bool valid = !TAIL || tok0 + tk < nn;
  L = valid ? L * esc : -INFINITY;
  // every lane's coefficient reads are done before the buffer takes weights
  // (the shuffles above do not order shared-memory accesses)
  __syncwarp();

  // ---- online softmax over the group (log2 units)
  const float gm = warp_max_f32(L);
  if constexpr (C::kLogits) {
    if (lane == 0) gmax_g[0] = gm;  // lets the selection pass skip groups far below tau
  }
  if (gm > ws.m) {
    const float c = fast_exp2(ws.m - gm);  // 0 before the first group
    ws.l *= c;
#pragma unroll
    for (int g = 0; g < VG; ++g) ws.beta[g] *= c;
#pragma unroll
    for (int f = 0; f < 4; ++f) ws.facc[f] *= c;
    ws.m = gm;
  }
  // the group's own gap d below the running maximum (an integer, warp-
  // uniform): its weights are scaled by 2^d so that its largest is in (1/2, 1]
  const float dref = C::kQuant ? floorf(fminf(ws.m - gm, kMaxGroupGap)) : 0.f;
  const float pw = fast_exp2(-dref);  // an exact power of two: dref is an integer
  const float wg = valid ? fast_exp2(L - ws.m + dref) : 0.f;
  const float w = wg * pw;
  ws.l += w;
  if constexpr (C::kLogits) logits_g[tk] = L;

  // ---- values: the owner of token tk turns its weight into per-group value
  //      weights; then every lane runs its column over all 32 tokens
  const int ob = tk >> 4, orow = tk & 15;
  const int col = lane % COLS, hb = lane / COLS;
  if constexpr (C::kQuant) {
    const uint8_t* mp = st + ob * HALF + R::kVMetaOff + orow * (VG * 4);
    uint32_t mv[VG];
    if constexpr (VG == 4) {
      const uint4 x = *reinterpret_cast<const uint4*>(mp);
      mv[0] = x.x;
      mv[1] = x.y;
      mv[2] = x.z;
      mv[3] = x.w;
    } else {
      const uint2 x = *reinterpret_cast<const uint2*>(mp);
      mv[0] = x.x;
      mv[1] = x.y;
    }
    float sv[VG];
    float smax = 0.f;
#pragma unroll
    for (int g = 0; g < VG; g += 2) {
      const float2 sc = make_float2(bf16_lo(mv[g]), bf16_lo(mv[g + 1]));
      const float2 mn = make_float2(bf16_hi(mv[g]), bf16_hi(mv[g + 1]));
      sv[g] = valid ? sc.x : 0.f;
      sv[g + 1] = valid ? sc.y : 0.f;
      smax = fmaxf(smax, fmaxf(sv[g], sv[g + 1]));
      // the minimum (plus the bucket midpoint of the high plane) of every
      // channel of the group, weighted once per token
      const float2 base = C::kLogits ? __ffma2_rn(make_float2(1.5f, 1.5f), sc, mn) : mn;
      if (valid) {
        const float2 b = __ffma2_rn(make_float2(w, w), base, make_float2(ws.beta[g], ws.beta[g + 1]));
        ws.beta[g] = b.x;
        ws.beta[g + 1] = b.y;
      }
    }
    // fixed-point scale: every 2^d w * scale * sF stays below 2^15 (2^d w
    // <= 1); a larger scale than any seen so far lowers F for the whole warp
    if (__any_sync(0xffffffffu, smax >= ws.slim)) {
      const float x = warp_max_f32(smax);
      const int e = min(static_cast<int>((__float_as_uint(x * C::kMult) >> 23) & 0xFFu) - 127, kMaxFixedExp + 14);
      ws.F = min(14 - e, kMaxFixedExp);
      ws.sF = C::kMult * pow2i(ws.F);
      ws.slim = pow2i(15 - ws.F) / C::kMult;
    }
    const float wF = wg * ws.sF;
    uint16_t* av = reinterpret_cast<uint16_t*>(vbuf);
    const float2 magic = make_float2(12582912.f, 12582912.f);  // 1.5 * 2^23: round to an integer
#pragma unroll
    for (int g = 0; g < VG; g += 2) {
      const float2 a = __ffma2_rn(make_float2(wF, wF), make_float2(sv[g], sv[g + 1]), magic);
      av[g * 32 + tk] = static_cast<uint16_t>(__float_as_uint(a.x));
      av[(g + 1) * 32 + tk] = static_cast<uint16_t>(__float_as_uint(a.y));
      if constexpr (C::kFourV) {
        const float2 b = __ffma2_rn(make_float2(0.25f * wF, 0.25f * wF), make_float2(sv[g], sv[g + 1]), magic);
        av[(VG + g) * 32 + tk] = static_cast<uint16_t>(__float_as_uint(b.x));
        av[(VG + g + 1) * 32 + tk] = static_cast<uint16_t>(__float_as_uint(b.y));
      }
    }
    __syncwarp();
    // this lane's column: the weight pairs of its value group, token order;
    // exact integer sums of the group (below 2^28), then added in fp32
    const uint32_t* ap = reinterpret_cast<const uint32_t*>(vbuf) + ((4 * col) / kGroup) * 16;
    uint32_t acc[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int bi = 0; bi < 2 / LPC; ++bi) {
      const int blk = LPC == 1 ? bi : hb;
      const uint4 cw = *reinterpret_cast<const uint4*>(st + blk * HALF + R::kVHi + col * 16);
      const uint4 a0 = *reinterpret_cast<const uint4*>(ap + 8 * blk);
      const uint4 a1 = *reinterpret_cast<const uint4*>(ap + 8 * blk + 4);
      column_dot(acc, cw.x, a0.x, a0.y);
      column_dot(acc, cw.y, a0.z, a0.w);
      column_dot(acc, cw.z, a1.x, a1.y);
      column_dot(acc, cw.w, a1.z, a1.w);
      if constexpr (C::kFourV) {
        // the low plane is row-major: gather byte col of every token row
        const uint8_t* lp = st + blk * HALF + R::kQ4VLo + col;
        const uint32_t* apl = ap + VG * 16;
        uint32_t lw[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
          lw[i] = static_cast<uint32_t>(lp[(4 * i) * R::kRow]) | (static_cast<uint32_t>(lp[(4 * i + 1) * R::kRow]) << 8) |
                  (static_cast<uint32_t>(lp[(4 * i + 2) * R::kRow]) << 16) |
                  (static_cast<uint32_t>(lp[(4 * i + 3) * R::kRow]) << 24);
        const uint4 l0 = *reinterpret_cast<const uint4*>(apl + 8 * blk);
        const uint4 l1 = *reinterpret_cast<const uint4*>(apl + 8 * blk + 4);
        column_dot(acc, lw[0], l0.x, l0.y);
        column_dot(acc, lw[1], l0.z, l0.w);
        column_dot(acc, lw[2], l1.x, l1.y);
        column_dot(acc, lw[3], l1.z, l1.w);
      }
    }
    // back to value units: 2^-(F + d), and 4^-f for field f
    const float u0 = pow2i(-ws.F) * pw;
#pragma unroll
    for (int f = 0; f < 4; ++f) ws.facc[f] = fmaf(__uint2float_rn(acc[f]), u0 * pow2i(-2 * f), ws.facc[f]);
  } else {
    float* wv = reinterpret_cast<float*>(vbuf);
    wv[tk] = w;
    __syncwarp();
#pragma unroll
    for (int bi = 0; bi < 2 / LPC; ++bi) {
      const int blk = LPC == 1 ? bi : hb;
#pragma unroll 4
      for (int t = 0; t < kBlock; ++t) {
        // past the end of the tail group the stage holds stale bytes, which
        // may read as Inf / NaN: skip them rather than multiply by zero
        if (TAIL && tok0 + kBlock * blk + t >= nn) break;
        const uint2 x = *reinterpret_cast<const uint2*>(st + blk * HALF + R::kBfV + t * D * 2 + col * 8);
        const float wt = wv[kBlock * blk + t];
        const float2 ww = make_float2(wt, wt);
        float2 a01 = __ffma2_rn(ww, make_float2(bf16_lo(x.x), bf16_hi(x.x)), make_float2(ws.facc[0], ws.facc[1]));
        float2 a23 = __ffma2_rn(ww, make_float2(bf16_lo(x.y), bf16_hi(x.y)), make_float2(ws.facc[2], ws.facc[3]));
        ws.facc[0] = a01.x;
        ws.facc[1] = a01.y;
        ws.facc[2] = a23.x;
        ws.facc[3] = a23.y;
      }
    }
  }
}

// MINB: CTAs per SM the register budget is cut for (4: 128 registers per
// thread; 5: 102, for grids of many waves where occupancy pays).
// GQ: grouped queries (2^g_log2 > 1 query heads per KV head); the build for
// one query per KV head carries none of their index arithmetic.
template <int KIND, int D, bool FULLV, bool CLUSTER, int MINB, bool GQ>
__global__ void __launch_bounds__(kThreads, MINB) decode_kernel(const DecodeParams p) {
  using C = Cfg<KIND, D, FULLV>;
  using R = typename C::R;
  constexpr int CH = C::kCH, NSW = C::kNSW;
  constexpr int LOAD = C::kLoad, STAGE = C::kStage;
  constexpr int COLS = C::kCols, LPC = C::kLPC, VG = C::kVG;

  extern __shared__ __align__(128) uint8_t smem[];
  const Smem sp = smem_plan(STAGE, NSW, p.chunk_groups, D, C::kLogits);
  float* logits = reinterpret_cast<float*>(smem + sp.logits);
  auto wres_of = [&](int w) { return reinterpret_cast<float*>(smem + sp.rings + sp.ring_bytes * w); };
  constexpr int kCorrOff = D * 4;  // after the warp's D channel sums
  auto corr_of = [&](int w) { return reinterpret_cast<float*>(smem + sp.rings + sp.ring_bytes * w + kCorrOff); };
  // the CTA's per-channel sums in its own scale, after warp 0's corrections
  float* cacc = reinterpret_cast<float*>(smem + sp.rings + kCorrOff + D * 4);
  int32_t* ids_smem = reinterpret_cast<int32_t*>(smem + sp.ids);
  uint32_t* masks_smem = reinterpret_cast<uint32_t*>(smem + sp.masks);
  float* gmax_smem = reinterpret_cast<float*>(smem + sp.gmax);
  float4* table = reinterpret_cast<float4*>(smem + sp.xchg);
  float* red = reinterpret_cast<float*>(smem + sp.xchg + 16 * 8 * kNW);
  int* cnts = reinterpret_cast<int*>(smem + sp.xchg + 16 * 8 * kNW + 4 * D);
  int* cta_i = reinterpret_cast<int*>(smem + sp.scal);
  static_assert(kCorrOff + 2 * D * 4 <= NSW * STAGE, "warp results must fit in an idle ring");

  const int split = blockIdx.x;
  const int S = gridDim.x;
  // KV head of this CTA's query head blockIdx.y (G = 2^g_log2 query heads
  // per KV head); with grouped queries the query head itself is read again
  // after pass 1, so that only one of the two stays live through it
  const int hk = GQ ? static_cast<int>(blockIdx.y) >> p.g_log2 : static_cast<int>(blockIdx.y);
  const int Hkv = GQ ? p.Hkv : p.H;
  // Grouped queries with a low-plane selection: the CTAs of the G query
  // heads of one KV head (and all their splits) form one cluster of S x G
  // (up to 16 CTAs),
  // rank split + S * (h % G), so that the heads can merge their selections.
  constexpr bool head_cl = GQ && CLUSTER && C::kLogits;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Long grids let the next kernel launch at once; a grid of one wave lets
  // it launch only after its pass 1, so that the next kernel's first CTAs
  // do not stream into the spare slots while this one is still streaming.
  if (p.pdl_early) pdl_allow_dependents();
  // Speculative block ids: the first 16 iterations' table entries of batch
  // slot z, for the chunk this split would get from a sequence of the host
  // bound max_seq_len.  They are used below when the actual sequence and
  // chunk match (every uniform-length batch), so the first bulk copies do
  // not wait for the lengths before reading the block table.
  const int zslot = blockIdx.z;
  const int ng_spec = (p.max_seq_len + kGroup - 1) / kGroup;
  const int g0_spec = min(split * ((ng_spec + S - 1) / S), ng_spec);
  int raw_spec = -1;
  {
    const int lb = 2 * (g0_spec + warp + kNW * (lane >> 1)) + (lane & 1);
    if (lb < p.max_blocks) raw_spec = p.block_table[static_cast<size_t>(zslot) * p.max_blocks + lb];
  }
  // Clusters are dispatched roughly in launch order; the z-th batch slot
  // takes the sequence of rank z by decreasing length (ties by index), so
  // ragged batches start their longest sequences first.
  const int b = sequence_of_rank(p.seq_lens, static_cast<int>(gridDim.z), static_cast<int>(blockIdx.z), lane);

  // ---- this split's chunk of 32-token groups (seq_lens and the block table
  //      are not written by the previous kernel: read before its completion)
  const bool fused_append = p.k_new != nullptr;
  const int n = fused_append ? (p.seq_lens[b] >= 0 ? p.seq_lens[b] + 1 : 0) : p.seq_lens[b];
  int bad = 0;
  if (n < 0 || n > p.max_seq_len || n > p.max_blocks * kBlock) bad = LOOPKV_DEVERR_SEQ_LEN;
  const int nn = bad ? 0 : n;
  const int ng = (nn + kGroup - 1) / kGroup;
  const int per = (ng + S - 1) / S;
  const int g0 = min(split * per, ng);
  const int cg = min(per, ng - g0);
  if (cg > p.chunk_groups) bad = LOOPKV_DEVERR_SEQ_LEN;
  const int n_blocks = (nn + kBlock - 1) / kBlock;

  // this warp's ring and barriers
  uint8_t* ring = smem + sp.rings + static_cast<size_t>(warp) * NSW * STAGE;
  const uint32_t bar0 = smem_addr(smem + sp.bars) + 8 * NSW * warp;
  if (lane == 0) {
    for (int i = 0; i < NSW; ++i) mbar_init(bar0 + 8 * i, 1);
    fence_mbar_init();
  }
  if (threadIdx.x == 0) cta_i[kSlotBad] = bad;
  // the heads of a group OR their selections into every member's words
  // after the exchange barrier below, which orders these zeros before them
  if (head_cl)
    for (int i = threadIdx.x; i < p.chunk_groups; i += kThreads) masks_smem[i] = 0u;
  __syncthreads();
  if constexpr (CLUSTER) cluster_arrive_relaxed();

  const int k = lane % CH, r = lane / CH;
  WarpState<D> ws;
  ws.m = -INFINITY;
  ws.l = 0.f;
#pragma unroll
  for (int g = 0; g < VG; ++g) ws.beta[g] = 0.f;
#pragma unroll
  for (int f = 0; f < 4; ++f) ws.facc[f] = 0.f;
  ws.F = kMaxFixedExp;
  ws.sF = C::kMult * pow2i(kMaxFixedExp);
  ws.slim = pow2i(15 - kMaxFixedExp) / C::kMult;

  // groups of this warp: gi = warp + kNW * it
  const int nit = (!bad && cg > warp) ? (cg - warp + kNW - 1) / kNW : 0;
  const int g_unsafe = (nn - 1) / kGroup;  // may be written by the previous kernel
  const uint64_t pol = l2_evict_first_policy();
  // record (block id, this KV head) lies at arena_h + id * rec_stride
  const uint8_t* arena_h = p.arena + static_cast<size_t>(hk) * R::kBytes;
  const size_t rec_stride = static_cast<size_t>(Hkv) * R::kBytes;
  const uint32_t ring_addr = smem_addr(ring);
  const int32_t* btab = p.block_table + static_cast<size_t>(b) * p.max_blocks;
  // block ids of 16 iterations, two per iteration, spread over the lanes
  auto load_ids = [&](int it0, bool speculated) {
    const int it = it0 + (lane >> 1);
    int id = -1;
    if (it < nit) {
      const int lb = 2 * (g0 + warp + kNW * it) + (lane & 1);
      if (lb < n_blocks) {
        id = speculated ? raw_spec : btab[lb];
        if (id < 0 || id >= p.num_blocks) {
          atomicOr(&cta_i[kSlotBad], LOOPKV_DEVERR_BLOCK_ID);
          id = -1;
        }
      }
    }
    return id;
  };
  // current and next batch of 16 iterations' ids: the next batch is loaded a
  // whole batch ahead, so its latency never stalls the ring
  int ids = load_ids(0, b == zslot && g0 == g0_spec), ids_next = load_ids(16, false), ids_base = 0;
  // issue the bulk copies of iteration `it` into its stage (all lanes call)
  auto issue = [&](int it) {
    if (it >= nit) return;
    if (it - ids_base >= 16) {
      ids_base += 16;
      ids = ids_next;
      ids_next = load_ids(ids_base + 16, false);
    }
    const int id0 = __shfl_sync(0xffffffffu, ids, 2 * (it - ids_base));
    const int id1 = __shfl_sync(0xffffffffu, ids, 2 * (it - ids_base) + 1);
    if (lane == 0) {
      if constexpr (C::kLogits) {  // kept for the low-plane gather of pass 2
        ids_smem[2 * (warp + kNW * it)] = id0;
        ids_smem[2 * (warp + kNW * it) + 1] = id1;
      }
      const int stage = it % NSW;
      const uint32_t bar = bar0 + 8 * stage;
      const uint32_t dst = ring_addr + stage * STAGE;
      const uint32_t bytes = (id0 >= 0 ? LOAD : 0) + (id1 >= 0 ? LOAD : 0);
      mbar_arrive_expect_tx(bar, bytes);
      if (id0 >= 0) bulk_load(dst, arena_h + static_cast<size_t>(id0) * rec_stride, LOAD, bar, pol);
      if (id1 >= 0) bulk_load(dst + C::kHalf, arena_h + static_cast<size_t>(id1) * rec_stride, LOAD, bar, pol);
    }
  };

  // ---- pass 1
  int issued = 0;
  if (nit > 0)
    while (issued < NSW && issued < nit && g0 + warp + kNW * issued < g_unsafe) issue(issued++);
  pdl_wait_prior_grid();  // q, the residual and the newest group may come from the previous kernel
  if (fused_append) {
    // the split holding the new token stores it first; its copies of the
    // newest group are issued after the writes are visible to the bulk copies
    if (!bad && nn > 0 && (nn - 1) / kGroup >= g0 && (nn - 1) / kGroup < g0 + cg) {
      append_token<KIND, D>(p, b, hk, nn - 1, warp, lane);
      fence_proxy_async_global();
    }
    __syncthreads();
  }
  if (nit > 0) {
    while (issued < NSW) issue(issued++);

    // query constants (log2 units): qf_c, and qs_c = qf_c * 2^(149 - pos - E)
    // for the subnormal code views; both in shared memory for all warps
    float* qconst = reinterpret_cast<float*>(smem + sp.qconst);
    float* q2buf = reinterpret_cast<float*>(smem + sp.q2buf) + warp * 128;
    uint8_t* vbuf = reinterpret_cast<uint8_t*>(q2buf);  // the same 512 B, reused after the keys
    for (int c = lane; c < D; c += 32) {
      const float qv = __bfloat162float(p.q[(static_cast<size_t>(b) * p.H + blockIdx.y) * D + c]) * p.sm_scale_log2;
      const int i = c & 15;
      // every warp writes the same values: no cross-warp ordering is needed
      qconst[c] = qv;
      qconst[D + c] = qv * pow2i(149 - (C::kQ4 ? pos4(i) : pos2(i)) - C::kE);
    }
    __syncwarp();
    // bf16 cells keep this lane's query channels in registers
    float qfr[C::kQuant ? 1 : C::kCW];
    if constexpr (!C::kQuant) {
#pragma unroll
      for (int i = 0; i < C::kCW; ++i) qfr[i] = qconst[C::kCW * k + i];
    }
    const __nv_bfloat16* res = C::kQuant ? p.residual + (static_cast<size_t>(b) * Hkv + hk) * kGroup * D : nullptr;

    for (int it = 0; it < nit; ++it) {
      const int stage = it % NSW;
      if (!mbar_wait(bar0 + 8 * stage, (it / NSW) & 1)) {
        atomicOr(&cta_i[kSlotBad], LOOPKV_DEVERR_TIMEOUT);
        // give the copies still in flight one more bounded wait before this
        // CTA moves on (and eventually releases its shared memory)
        for (int pend = it; pend < min(nit, it + NSW); ++pend) mbar_wait(bar0 + 8 * (pend % NSW), (pend / NSW) & 1);
        break;
      }
      const int gi = warp + kNW * it;
      const int tok0 = (g0 + gi) * kGroup;
      const uint8_t* st = ring + stage * STAGE;
      float* lg = logits + gi * kGroup;
      if (tok0 + kGroup <= nn)
        group_step<KIND, D, FULLV, false>(st, qconst, q2buf, vbuf, qfr, res, tok0, nn, lane, r, k, lg,
                                            gmax_smem + gi, ws);
      else
        group_step<KIND, D, FULLV, true>(st, qconst, q2buf, vbuf, qfr, res, tok0, nn, lane, r, k, lg,
                                           gmax_smem + gi, ws);
      // every shared-memory read of this stage has been consumed above, so
      // the stage can be refilled
      __syncwarp();
      issue(it + NSW);
    }
  }
  pdl_wait_prior_grid();  // nothing below may run ahead of the previous kernel
  if (!p.pdl_early) pdl_allow_dependents();

  const int h = GQ ? cta_id_y() : hk;  // query head

  // ---- this warp's result in its own scale 2^-m_w: true per-channel sums
  //      (lane (hb, col) holds channels 4 col .. 4 col + 3)
  float lw;
  {
    lw = ws.l;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) lw += __shfl_xor_sync(0xffffffffu, lw, off);
    const int col = lane % COLS, hb = lane / COLS;
    float o[4];
    if constexpr (C::kQuant) {
      // the value minima of the lane's group gv, summed over every lane's
      // owned tokens: a transposed all-reduce that halves the groups a lane
      // keeps at each of the first log2(VG) steps (lane bit 4, then 3 picks
      // the half, matching gv = lane / (32 / VG) for D = 128 and 64)
      float bmine;
      if constexpr (VG == 4) {
        const bool up = lane & 16;
        const float s0 = up ? ws.beta[0] : ws.beta[2], s1 = up ? ws.beta[1] : ws.beta[3];
        const float q0 = (up ? ws.beta[2] : ws.beta[0]) + __shfl_xor_sync(0xffffffffu, s0, 16);
        const float q1 = (up ? ws.beta[3] : ws.beta[1]) + __shfl_xor_sync(0xffffffffu, s1, 16);
        const bool odd = lane & 8;
        bmine = (odd ? q1 : q0) + __shfl_xor_sync(0xffffffffu, odd ? q0 : q1, 8);
#pragma unroll
        for (int off = 4; off > 0; off >>= 1) bmine += __shfl_xor_sync(0xffffffffu, bmine, off);
      } else {
        static_assert(VG == 2, "value groups per token: 4 (D = 128) or 2 (D = 64)");
        // D = 64: gv = col / 8 with col = lane % 16, i.e. lane bit 3
        const bool odd = lane & 8;
        bmine = (odd ? ws.beta[1] : ws.beta[0]) + __shfl_xor_sync(0xffffffffu, odd ? ws.beta[0] : ws.beta[1], 8);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
          if (off != 8) bmine += __shfl_xor_sync(0xffffffffu, bmine, off);
      }
#pragma unroll
      for (int f = 0; f < 4; ++f) o[f] = ws.facc[f];
      if constexpr (LPC == 2) {
#pragma unroll
        for (int f = 0; f < 4; ++f) o[f] += __shfl_xor_sync(0xffffffffu, o[f], 16);
      }
#pragma unroll
      for (int f = 0; f < 4; ++f) o[f] += bmine;
    } else {
#pragma unroll
      for (int f = 0; f < 4; ++f) o[f] = ws.facc[f];
      if constexpr (LPC == 2) {
#pragma unroll
        for (int f = 0; f < 4; ++f) o[f] += __shfl_xor_sync(0xffffffffu, o[f], 16);
      }
    }
    // the current token of the cell's own loop (exact K and V, one more
    // softmax entry after the stored tokens): warp 0 of the last split
    if (p.k_cur != nullptr && split == S - 1 && warp == 0 && !cta_i[kSlotBad]) {
      const size_t kv_row = (static_cast<size_t>(b) * Hkv + hk) * D;
      const __nv_bfloat16* qh = p.q + (static_cast<size_t>(b) * p.H + h) * D;
      float sd = 0.f;
      for (int c = lane; c < D; c += 32)
        sd = fmaf(__bfloat162float(qh[c]) * p.sm_scale_log2, __bfloat162float(p.k_cur[kv_row + c]), sd);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) sd += __shfl_xor_sync(0xffffffffu, sd, off);
      const float mnew = fmaxf(ws.m, sd);
      const float a = fast_exp2(ws.m - mnew), bw = fast_exp2(sd - mnew);
      lw = fmaf(lw, a, bw);
#pragma unroll
      for (int f = 0; f < 4; ++f) o[f] = fmaf(o[f], a, bw * __bfloat162float(p.v_cur[kv_row + 4 * col + f]));
      ws.m = mnew;
    }
    if (hb == 0) *reinterpret_cast<float4*>(wres_of(warp) + 4 * col) = make_float4(o[0], o[1], o[2], o[3]);
  }

  const int HC = head_cl ? 1 << p.g_log2 : 1;
  const int rbase = S * (h & (HC - 1));  // cluster rank of this head's split 0
  // Kinds that cannot select (2-bit, bf16) need no normaliser before the
  // combine: their splits meet once, each pushing its table entries and its
  // channel sums in its own scale, and the owners rescale after that barrier.
  constexpr bool kOneMeet = CLUSTER && !C::kQ4;
  const int per_rank = D / S;

  // ---- publish (max, sum, error bits) of this warp into every split's table
  if constexpr (CLUSTER) cluster_wait();  // every CTA of the cluster has started
  {
    const float4 ent = make_float4(ws.m, lw, __int_as_float(cta_i[kSlotBad]), 0.f);
    const int e = split * kNW + warp;
    if constexpr (CLUSTER) {
      if (lane < S) st_peer_v4(peer_addr(smem_addr(table + e), rbase + lane), ent);
    } else if (lane == 0) {
      table[e] = ent;
    }
  }
  if constexpr (CLUSTER && !kOneMeet) cluster_arrive_release();

  // ---- while the splits meet: this CTA's share of every channel in its own
  //      scale 2^-m_c (the warps' sub-group sums, rescaled and added)
  __syncthreads();  // every warp's partial sums and table entry are in place
  float m_c = -INFINITY;
#pragma unroll
  for (int w = 0; w < kNW; ++w) m_c = fmaxf(m_c, table[split * kNW + w].x);
  for (int c = threadIdx.x; c < D; c += kThreads) {
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kNW; ++w) {
      const float mw = table[split * kNW + w].x;
      if (mw != -INFINITY) v = fmaf(fast_exp2(mw - m_c), wres_of(w)[c], v);
    }
    cacc[c] = v;
    if constexpr (kOneMeet) {
      // the owner of channel c gets it in this CTA's scale (m_c, from the table)
      st_peer_f32(peer_addr(smem_addr(red + split * per_rank + c % per_rank), rbase + c / per_rank), v);
    }
  }
  if constexpr (kOneMeet) cluster_arrive_release();  // tables and sums are in place after the wait
  if constexpr (CLUSTER) cluster_wait_acquire(); else __syncthreads();

  // ---- global (max, normaliser, errors) from the local table
  float m_g, z;
  int any_bad;
  {
    float me = -INFINITY, le = 0.f;
    int be = 0;
    if (lane < S * kNW) {
      const float4 t = table[lane];
      me = t.x;
      le = t.y;
      be = __float_as_int(t.z);
    }
    m_g = me;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m_g = fmaxf(m_g, __shfl_xor_sync(0xffffffffu, m_g, off));
    z = (me == -INFINITY) ? 0.f : le * fast_exp2(me - m_g);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
    any_bad = static_cast<int>(__reduce_or_sync(0xffffffffu, static_cast<unsigned>(be)));
  }
  const bool live = !any_bad && z > 0.f;
  const float inv_z = live ? 1.f / z : 0.f;

  // ---- pass 2a: low-plane selection of every group of this warp
  // only a 4-bit cell can select (its count); other kinds write their
  // empty selection words only when asked for them
  const bool want_mask = p.sel_mask != nullptr || (C::kQ4 && p.sel_count != nullptr);
  const bool gather = C::kLogits && p.tau < INFINITY;
  int cnt = 0;
  if (live && (gather || want_mask)) {
    // the selection word of group gi (all lanes call; warp-uniform gi)
    auto select_group = [&](int gi) {
      const bool valid = (g0 + gi) * kGroup + lane < nn;
      bool sel;
      if constexpr (C::kLogits) {
        sel = valid && (fast_exp2(logits[gi * kGroup + lane] - m_g) * inv_z >= p.tau);
      } else {
        sel = C::kQ4 && valid;  // tau = 0: every token took its low plane in pass 1
      }
      uint32_t mask = __ballot_sync(0xffffffffu, sel);
      if (C::kLogits && p.sel_unit > 1) {
        // coarser units: a 16-token block or the whole group takes its low
        // plane when any of its tokens reaches tau (groups and blocks align)
        const uint32_t valid_mask = __ballot_sync(0xffffffffu, valid);
        if (p.sel_unit == 16)
          mask = ((mask & 0x0000FFFFu) ? 0x0000FFFFu : 0u) | ((mask & 0xFFFF0000u) ? 0xFFFF0000u : 0u);
        else
          mask = mask ? 0xFFFFFFFFu : 0u;
        mask &= valid_mask;
      }
      if (HC > 1) {
        // into the same split of every head of the group (itself included)
        if (lane < HC && mask) or_peer_u32(peer_addr(smem_addr(masks_smem + gi), split + S * lane), mask);
        return;
      }
      if (lane == 0) {
        if (p.sel_mask) p.sel_mask[(static_cast<size_t>(b) * p.H + h) * p.mask_words + g0 + gi] = mask;
        if constexpr (C::kLogits) masks_smem[gi] = mask;
      }
      cnt += __popc(mask);
    };
    if constexpr (C::kLogits) {
      // a group whose largest weight is below tau selects nothing (the same
      // fp32 test as the tokens', on its largest logit): 32 groups tested at
      // once, one per lane, and only the groups that pass are walked
      const int ngw = cg > warp ? (cg - warp + kNW - 1) / kNW : 0;
      for (int base = 0; base < ngw; base += 32) {
        const int gl = warp + kNW * (base + lane);
        const bool pass = base + lane < ngw && fast_exp2(gmax_smem[gl] - m_g) * inv_z >= p.tau;
        if (base + lane < ngw && !pass && HC == 1) {
          if (p.sel_mask) p.sel_mask[(static_cast<size_t>(b) * p.H + h) * p.mask_words + g0 + gl] = 0u;
          masks_smem[gl] = 0u;
        }
        uint32_t todo = __ballot_sync(0xffffffffu, pass);
        while (todo) {
          const int j = __ffs(todo) - 1;
          todo &= todo - 1u;
          select_group(warp + kNW * (base + j));
        }
      }
    } else {
      for (int gi = warp; gi < cg; gi += kNW) select_group(gi);
    }
  }
  if (C::kLogits && HC > 1) {
    // every head of the group has merged its selection: the union, which
    // every head gathers and reports
    cluster_arrive_release();
    cluster_wait_acquire();
    if (live && (gather || want_mask)) {
      for (int gi = warp; gi < cg; gi += kNW) {
        const uint32_t mask = masks_smem[gi];
        if (lane == 0 && p.sel_mask) p.sel_mask[(static_cast<size_t>(b) * p.H + h) * p.mask_words + g0 + gi] = mask;
        cnt += __popc(mask);
      }
    }
  }
  __syncwarp();  // lane 0's selection words are read by the whole warp below

  // ---- pass 2b: gather the selected tokens' low-plane rows, kNB tokens per
  //      round trip; lane l owns channels 4l .. 4l + 3 (one byte of the row)
  //      and adds p * scale * (lo - 1.5) in the final units
  if constexpr (C::kLogits) {
    if (live && gather) {
      constexpr int kNB = 4;
      float corr[4] = {0.f, 0.f, 0.f, 0.f};
      // coarser selection units: walk the selected 16-token blocks, loading
      // every selected row of a block in one round trip
      for (int gi = warp; p.sel_unit > 1 && cnt > 0 && gi < cg; gi += kNW) {
        const uint32_t m = masks_smem[gi];
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
          const uint32_t bm = (m >> (16 * half)) & 0xFFFFu;
          const int phys = bm ? ids_smem[2 * gi + half] : -1;
          if (phys < 0) continue;
          const uint8_t* rec = p.arena + (static_cast<size_t>(phys) * Hkv + hk) * R::kBytes;
          uint32_t lo16[kBlock], mv16[kBlock];
#pragma unroll
          for (int t = 0; t < kBlock; ++t) {
            lo16[t] = mv16[t] = 0u;
            if (lane < D / 4 && ((bm >> t) & 1u)) {
              lo16[t] = rec[R::kQ4VLo + t * R::kRow + lane];
              mv16[t] = *reinterpret_cast<const uint32_t*>(rec + R::kQ4VMeta +
                                                           (t * (D / kGroup) + (4 * lane) / kGroup) * 4);
            }
          }
#pragma unroll
          for (int t = 0; t < kBlock; ++t) {
            if ((bm >> t) & 1u) {
              const float wsel =
                  fast_exp2(logits[gi * kGroup + kBlock * half + t] - m_g) * inv_z * bf16_lo(mv16[t]);
#pragma unroll
              for (int i = 0; i < 4; ++i)
                corr[i] = fmaf(wsel, static_cast<float>((lo16[t] >> (2 * i)) & 3u) - 1.5f, corr[i]);
            }
          }
        }
      }
      int gcur = warp;
      uint32_t mcur = (p.sel_unit == 1 && cnt > 0 && gcur < cg) ? masks_smem[gcur] : 0u;
      int left = p.sel_unit == 1 ? cnt : 0;
      while (left > 0) {
        int tg[kNB], tt[kNB];
#pragma unroll
        for (int j = 0; j < kNB; ++j) {
          while (mcur == 0u && left > 0 && gcur + kNW < cg) {
            gcur += kNW;
            mcur = masks_smem[gcur];
          }
          tg[j] = -1;
          tt[j] = 0;
          if (mcur != 0u && left > 0) {
            tg[j] = gcur;
            tt[j] = __ffs(mcur) - 1;
            mcur &= mcur - 1u;
            --left;
          }
        }
        uint32_t mv[kNB], lo[kNB];
        float lgv[kNB];
#pragma unroll
        for (int j = 0; j < kNB; ++j) {
          mv[j] = 0u;
          lo[j] = 0u;
          lgv[j] = -INFINITY;
          if (tg[j] >= 0) {
            const int phys = ids_smem[2 * tg[j] + (tt[j] >> 4)];
            lgv[j] = logits[tg[j] * kGroup + tt[j]];
            if (phys >= 0 && lane < D / 4) {
              const uint8_t* rec = p.arena + (static_cast<size_t>(phys) * Hkv + hk) * R::kBytes;
              mv[j] = *reinterpret_cast<const uint32_t*>(rec + R::kQ4VMeta +
                                                         ((tt[j] & 15) * (D / kGroup) + (4 * lane) / kGroup) * 4);
              lo[j] = rec[R::kQ4VLo + (tt[j] & 15) * R::kRow + lane];
            }
          }
        }
#pragma unroll
        for (int j = 0; j < kNB; ++j) {
          const float wsel = fast_exp2(lgv[j] - m_g) * inv_z * bf16_lo(mv[j]);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            corr[i] = fmaf(wsel, static_cast<float>((lo[j] >> (2 * i)) & 3u) - 1.5f, corr[i]);
        }
      }
      if (lane < D / 4)
        *reinterpret_cast<float4*>(corr_of(warp) + 4 * lane) = make_float4(corr[0], corr[1], corr[2], corr[3]);
    }
  }
  if (lane == 0) cta_i[kSlotCnt0 + warp] = cnt;
  __syncthreads();  // every warp's sums, corrections and counts are in shared memory

  if constexpr (kOneMeet) {
    // ---- the owner's channels: every split's sum in the final units, added
    //      in split order (the same arithmetic as the two-barrier combine)
    if (threadIdx.x < per_rank) {
      float v = 0.f;
      for (int s = 0; s < S; ++s) {
        float m_s = -INFINITY;
#pragma unroll
        for (int w = 0; w < kNW; ++w) m_s = fmaxf(m_s, table[s * kNW + w].x);
        float vs = 0.f;
        if (live && m_s != -INFINITY) vs = red[s * per_rank + threadIdx.x] * fast_exp2(m_s - m_g) * inv_z;
        v += vs;
      }
      p.out[(static_cast<size_t>(b) * p.H + h) * D + split * per_rank + threadIdx.x] = __float2bfloat16_rn(v);
    }
    if (split == 0 && threadIdx.x == 0) {
      if (p.sel_count) p.sel_count[static_cast<size_t>(b) * p.H + h] = 0;
      if (any_bad) flag_error(p.err, any_bad);
    }
    return;
  }

  // ---- push this CTA's share of every channel, in the final units, to the
  //      split that owns the channel: rank s owns [s*D/S, (s+1)*D/S)
  if (threadIdx.x < D) {
    const int c = threadIdx.x;
    float v = 0.f;
    if (live) {
      if (m_c != -INFINITY) v = cacc[c] * fast_exp2(m_c - m_g) * inv_z;
      if (C::kLogits && gather) {
#pragma unroll
        for (int w = 0; w < kNW; ++w) v += corr_of(w)[c];
      }
    }
    const int slot = split * per_rank + c % per_rank;
    if constexpr (CLUSTER) st_peer_f32(peer_addr(smem_addr(red + slot), rbase + c / per_rank), v);
    else red[slot] = v;
  }
  if (threadIdx.x == 0) {
    int total = 0;
#pragma unroll
    for (int w = 0; w < kNW; ++w) total += cta_i[kSlotCnt0 + w];
    if constexpr (CLUSTER) st_peer_s32(peer_addr(smem_addr(cnts + split), rbase), total);
    else cnts[split] = total;
  }
  // after this barrier no CTA touches another's shared memory
  if constexpr (CLUSTER) cluster_sync_all(); else __syncthreads();

  if (threadIdx.x < per_rank) {
    float v = 0.f;
    for (int s = 0; s < S; ++s) v += red[s * per_rank + threadIdx.x];
    p.out[(static_cast<size_t>(b) * p.H + h) * D + split * per_rank + threadIdx.x] = __float2bfloat16_rn(v);
  }
  if (split == 0 && threadIdx.x == 0) {
    if (p.sel_count) {
      int total = 0;
      if (live && C::kQ4)
        for (int s = 0; s < S; ++s) total += cnts[s];
      p.sel_count[static_cast<size_t>(b) * p.H + h] = total;
    }
    if (any_bad) flag_error(p.err, any_bad);
  }
}

template <int KIND, int D, bool FULLV>
size_t smem_bytes_t(int cg) {
  using C = Cfg<KIND, D, FULLV>;
  return smem_plan(C::kStage, C::kNSW, cg, D, C::kLogits).total;
}

// Host-side launch state, set up once per (kernel build, device) and shared
// by every thread: the dynamic shared-memory limit of each build is raised
// once to the largest size a CTA may request (so no call ever lowers it
// under another thread's launch), non-portable cluster sizes are allowed
// once, and the device's SM count and every occupancy answer are cached.
constexpr int kMaxDevices = 64;

int device_sms(int* dev_out) {
  static std::mutex mu;
  static int sms_of[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) dev = -1;
  if (dev_out) *dev_out = dev;
  if (dev < 0) return 148;
  std::lock_guard<std::mutex> lock(mu);
  if (sms_of[dev] == 0) {
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) return 148;
    sms_of[dev] = sms;
  }
  return sms_of[dev];
}

template <int KIND, int D, bool FULLV, bool CLUSTER, int MINB, bool GQ>
cudaError_t prepare_kernel(int dev) {
  static std::mutex mu;
  static bool done[kMaxDevices] = {};
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (done[dev]) return cudaSuccess;
  auto kern = decode_kernel<KIND, D, FULLV, CLUSTER, MINB, GQ>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kMaxDynamicSmem));
  if (e == cudaSuccess && CLUSTER) e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e == cudaSuccess) done[dev] = true;
  return e;
}

// CTAs of this instantiation that can be resident at once on the device
// (for clusters of splits x hc: co-resident clusters times the cluster size);
// 0 when the build cannot run the configuration.  Answers are cached.
template <int KIND, int D, bool FULLV, bool CLUSTER, int MINB, bool GQ = false>
long resident_ctas_t(int cg, int splits, int hc) {
  const size_t smem = smem_bytes_t<KIND, D, FULLV>(cg);
  if (smem > kMaxDynamicSmem) return 0;
  int dev = -1;
  const int sms = device_sms(&dev);
  if (dev < 0 || prepare_kernel<KIND, D, FULLV, CLUSTER, MINB, GQ>(dev) != cudaSuccess) return 0;
  static std::mutex mu;
  static std::map<std::tuple<int, size_t, int, int>, long> cache;
  const auto key = std::make_tuple(dev, smem, splits, hc);
  {
    std::lock_guard<std::mutex> lock(mu);
    const auto it = cache.find(key);
    if (it != cache.end()) return it->second;
  }
  auto kern = decode_kernel<KIND, D, FULLV, CLUSTER, MINB, GQ>;
  long slots = 0;
  if (!CLUSTER) {
    int blocks = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks, kern, kThreads, smem) != cudaSuccess) return 0;
    slots = static_cast<long>(blocks) * sms;
  } else {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(splits, hc, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = splits;
    attr.val.clusterDim.y = hc;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg) != cudaSuccess) return 0;
    slots = static_cast<long>(clusters) * splits * hc;
  }
  std::lock_guard<std::mutex> lock(mu);
  cache[key] = slots;
  return slots;
}

// balance: ask the hardware to place a cluster's CTAs on the least loaded
// SMs (cluster scheduling policy "load balancing") instead of the default.
template <int KIND, int D, bool FULLV, bool CLUSTER, int MINB, bool GQ>
cudaError_t launch_t(const DecodeParams& p, int batch, int splits, int hc, cudaStream_t stream, bool pdl,
                     bool balance) {
  const size_t smem = smem_bytes_t<KIND, D, FULLV>(p.chunk_groups);
  if (smem > kMaxDynamicSmem) return cudaErrorInvalidValue;
  auto kern = decode_kernel<KIND, D, FULLV, CLUSTER, MINB, GQ>;
  int dev = -1;
  device_sms(&dev);
  cudaError_t e = prepare_kernel<KIND, D, FULLV, CLUSTER, MINB, GQ>(dev);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(splits, p.H, batch);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[3];
  int na = 0;
  if (CLUSTER) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = splits;
    attr[na].val.clusterDim.y = hc;
    attr[na].val.clusterDim.z = 1;
    ++na;
    if (balance) {
      attr[na].id = cudaLaunchAttributeClusterSchedulingPolicyPreference;
      attr[na].val.clusterSchedulingPolicyPreference = cudaClusterSchedulingPolicyLoadBalancing;
      ++na;
    }
  }
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

template <int KIND, int D, bool FULLV, int MINB>
long resident_m(int cg, int splits, int hc) {
  return splits * hc > 1 ? resident_ctas_t<KIND, D, FULLV, true, MINB>(cg, splits, hc)
                         : resident_ctas_t<KIND, D, FULLV, false, MINB>(cg, splits, 1);
}

// A grid of at least this many waves of 4-per-SM residency runs the
// 5-per-SM build: its extra warps hide latency once every SM stays busy for
// long; short grids keep the full register budget.
constexpr long kHighOccupancyWaves = 3;
// Grids of at most this many waves let the hardware load-balance each
// cluster's CTAs over the SMs: a short grid cannot spread evenly (512 CTAs
// on 148 SMs leave some SMs one CTA more), and the busiest SMs set the
// launch time; longer grids keep the default placement, which measured
// faster there.
constexpr long kBalancedWaves = 2;

template <int KIND, int D, bool FULLV>
cudaError_t launch_c(const DecodeParams& p, int batch, int splits, cudaStream_t stream, bool pdl) {
  const int hc = head_cluster(KIND, 1 << p.g_log2, FULLV);
  if (splits > kMaxClusterSplits || splits * hc > kMaxClusterCtas) return cudaErrorInvalidValue;
  const bool cl = splits * hc > 1;
  const long ctas = static_cast<long>(batch) * p.H * splits;
  const long slots4 = resident_m<KIND, D, FULLV, 4>(p.chunk_groups, splits, hc);
  const bool balance = cl && slots4 > 0 && ctas <= kBalancedWaves * slots4;
  DecodeParams q = p;
  q.pdl_early = slots4 <= 0 || ctas > slots4;
  // grouped queries: one build, at four CTAs per SM
  if (p.g_log2 > 0)
    return cl ? launch_t<KIND, D, FULLV, true, 4, true>(q, batch, splits, hc, stream, pdl, balance)
              : launch_t<KIND, D, FULLV, false, 4, true>(q, batch, splits, 1, stream, pdl, false);
  if constexpr (KIND != LOOPKV_CELL_BF16 && !FULLV) {
    if (slots4 > 0 && ctas >= kHighOccupancyWaves * slots4 &&
        resident_m<KIND, D, FULLV, 5>(p.chunk_groups, splits, 1) > slots4)
      return cl ? launch_t<KIND, D, FULLV, true, 5, false>(q, batch, splits, 1, stream, pdl, balance)
                : launch_t<KIND, D, FULLV, false, 5, false>(q, batch, splits, 1, stream, pdl, false);
  }
  return cl ? launch_t<KIND, D, FULLV, true, 4, false>(q, batch, splits, 1, stream, pdl, balance)
            : launch_t<KIND, D, FULLV, false, 4, false>(q, batch, splits, 1, stream, pdl, false);
}

// Co-resident CTAs of one decode build (0 without a device); minb 5 only
// exists for the 4-bit and 2-bit kinds.
long resident_ctas(int kind, int d, int cg, int splits, int hc, int minb) {
  if (minb == 5) {
    switch (kind * 1000 + d) {
      case LOOPKV_CELL_Q4 * 1000 + 128: return resident_m<LOOPKV_CELL_Q4, 128, false, 5>(cg, splits, hc);
      case LOOPKV_CELL_Q4 * 1000 + 64: return resident_m<LOOPKV_CELL_Q4, 64, false, 5>(cg, splits, hc);
      case LOOPKV_CELL_Q2 * 1000 + 128: return resident_m<LOOPKV_CELL_Q2, 128, false, 5>(cg, splits, 1);
      case LOOPKV_CELL_Q2 * 1000 + 64: return resident_m<LOOPKV_CELL_Q2, 64, false, 5>(cg, splits, 1);
      default: return 0;
    }
  }
  switch (kind * 1000 + d) {
    case LOOPKV_CELL_Q4 * 1000 + 128: return resident_m<LOOPKV_CELL_Q4, 128, false, 4>(cg, splits, hc);
    case LOOPKV_CELL_Q4 * 1000 + 64: return resident_m<LOOPKV_CELL_Q4, 64, false, 4>(cg, splits, hc);
    case LOOPKV_CELL_Q2 * 1000 + 128: return resident_m<LOOPKV_CELL_Q2, 128, false, 4>(cg, splits, 1);
    case LOOPKV_CELL_Q2 * 1000 + 64: return resident_m<LOOPKV_CELL_Q2, 64, false, 4>(cg, splits, 1);
    case LOOPKV_CELL_BF16 * 1000 + 128: return resident_m<LOOPKV_CELL_BF16, 128, false, 4>(cg, splits, 1);
    case LOOPKV_CELL_BF16 * 1000 + 64: return resident_m<LOOPKV_CELL_BF16, 64, false, 4>(cg, splits, 1);
    default: return 0;
  }
}

}  // namespace

// Splits are chosen so that a split holds at most this many groups (its
// logits buffer stays small enough for four CTAs per SM, and the longest
// chunk of a ragged batch stays short) ...
constexpr int kTargetGroupsPerSplit = 160;

int decode_splits(int kind, int head_dim, int batch, int heads, int max_seq_len, int hc) {
  const int groups = (max_seq_len + kGroup - 1) / kGroup;
  const long pairs = static_cast<long>(batch) * heads;
  const int smax = max_splits(hc);
  int s = 1;
  while (s < smax && (groups + s - 1) / s > kTargetGroupsPerSplit) s <<= 1;
  if (pairs <= 0 || groups <= 1) return s;
  const int sms = device_sms(nullptr);
  // ... and, past that, doubled while the grid fills less than 80 % of the
  // resident slots once (short grids: more, shorter CTAs put every SM to
  // work), keeping at least two groups per warp
  while (s < smax && groups >= 2 * kNW * 2 * s) {
    long slots = resident_ctas(kind, head_dim, (groups + s - 1) / s, s, hc, 4);
    if (slots <= 0) slots = 4L * sms;  // no device: a fixed guess keeps the choice deterministic
    if (pairs * s * 5 >= slots * 4) break;
    s <<= 1;
  }
  return s;
}

size_t decode_smem_bytes(int kind, int head_dim, bool full_values, int chunk_groups) {
  switch (kind * 1000 + head_dim) {
    case LOOPKV_CELL_Q4 * 1000 + 128:
      return full_values ? smem_bytes_t<LOOPKV_CELL_Q4, 128, true>(chunk_groups)
                         : smem_bytes_t<LOOPKV_CELL_Q4, 128, false>(chunk_groups);
    case LOOPKV_CELL_Q4 * 1000 + 64:
      return full_values ? smem_bytes_t<LOOPKV_CELL_Q4, 64, true>(chunk_groups)
                         : smem_bytes_t<LOOPKV_CELL_Q4, 64, false>(chunk_groups);
    case LOOPKV_CELL_Q2 * 1000 + 128: return smem_bytes_t<LOOPKV_CELL_Q2, 128, false>(chunk_groups);
    case LOOPKV_CELL_Q2 * 1000 + 64: return smem_bytes_t<LOOPKV_CELL_Q2, 64, false>(chunk_groups);
    case LOOPKV_CELL_BF16 * 1000 + 128: return smem_bytes_t<LOOPKV_CELL_BF16, 128, false>(chunk_groups);
    case LOOPKV_CELL_BF16 * 1000 + 64: return smem_bytes_t<LOOPKV_CELL_BF16, 64, false>(chunk_groups);
    default: return 0;
  }
}

cudaError_t launch_decode(int kind, int head_dim, const DecodeParams& p, int batch, int splits,
                          bool full_values, cudaStream_t stream, bool pdl) {
  if (batch == 0) return cudaSuccess;
  const int key = kind * 1000 + head_dim;
  switch (key) {
    case LOOPKV_CELL_Q4 * 1000 + 128:
      return full_values ? launch_c<LOOPKV_CELL_Q4, 128, true>(p, batch, splits, stream, pdl)
                         : launch_c<LOOPKV_CELL_Q4, 128, false>(p, batch, splits, stream, pdl);
    case LOOPKV_CELL_Q4 * 1000 + 64:
      return full_values ? launch_c<LOOPKV_CELL_Q4, 64, true>(p, batch, splits, stream, pdl)
                         : launch_c<LOOPKV_CELL_Q4, 64, false>(p, batch, splits, stream, pdl);
    case LOOPKV_CELL_Q2 * 1000 + 128: return launch_c<LOOPKV_CELL_Q2, 128, false>(p, batch, splits, stream, pdl);
    case LOOPKV_CELL_Q2 * 1000 + 64: return launch_c<LOOPKV_CELL_Q2, 64, false>(p, batch, splits, stream, pdl);
    case LOOPKV_CELL_BF16 * 1000 + 128: return launch_c<LOOPKV_CELL_BF16, 128, false>(p, batch, splits, stream, pdl);
    case LOOPKV_CELL_BF16 * 1000 + 64: return launch_c<LOOPKV_CELL_BF16, 64, false>(p, batch, splits, stream, pdl);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace loopkv
