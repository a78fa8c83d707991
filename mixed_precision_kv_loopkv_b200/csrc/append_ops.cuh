// Quantise-append building blocks shared by the append kernel and the fused
// append + decode kernel (sm_100a).
//
// LoopKV: Loop-Aware KV Cache Compression for Serving Looped Transformers,
// Abstract: cells are stored 4-bit (as high and low 2-bit planes) or 2-bit.
// The quantiser is the library's reading of the open format: asymmetric, with
// bf16 scale and minimum; values per token over 32-channel groups, keys per
// channel over 32-token groups.  Every step of the quantiser is one correctly
// rounded fp32 operation (no contraction), so the integer codes are exactly
// reproducible on any IEEE machine.
#pragma once

#include "device_common.cuh"

namespace loopkv {

__device__ __forceinline__ float warp_min(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fminf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
// OR over the 16 lanes of each half-warp.
__device__ __forceinline__ uint32_t half_warp_or(uint32_t x) {
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) x |= __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// bf16 scale and minimum of a group with extremes mn, mx.
template <int BITS>
__device__ __forceinline__ void group_params(float mn, float mx, float& s_b, float& mn_b) {
  mn_b = __bfloat162float(__float2bfloat16_rn(mn));
  const float s = __fdiv_rn(__fsub_rn(mx, mn_b), static_cast<float>((1 << BITS) - 1));
  s_b = __bfloat162float(__float2bfloat16_rn(s));
}

template <int BITS>
__device__ __forceinline__ uint32_t group_code(float x, float s_b, float mn_b) {
  if (s_b == 0.f) return 0u;
  float t = rintf(__fdiv_rn(__fsub_rn(x, mn_b), s_b));
  t = fminf(fmaxf(t, 0.f), static_cast<float>((1 << BITS) - 1));
  return static_cast<uint32_t>(t);
}

__device__ __forceinline__ uint32_t meta_word(float s_b, float mn_b) {
  return static_cast<uint32_t>(bf16_bits_rn(s_b)) |
         (static_cast<uint32_t>(bf16_bits_rn(mn_b)) << 16);
}

// One head of one sequence of a stored cell, as the writers see it.
struct CellRows {
  uint8_t* arena;           // [num_blocks][H][record]
  const int32_t* btab;      // this sequence's row of the block table
  int32_t* err;             // optional error word
  int H, h, max_blocks, num_blocks;
};

// Record holding position pos, or null after flagging a bad length or block.
template <int KIND, int D>
__device__ __forceinline__ uint8_t* record_at(const CellRows& c, int pos) {
  const int lb = pos / kBlock;
  if (lb >= c.max_blocks) {
    flag_error(c.err, LOOPKV_DEVERR_SEQ_LEN);
    return nullptr;
  }
  const int phys = c.btab[lb];
  if (phys < 0 || phys >= c.num_blocks) {
    flag_error(c.err, LOOPKV_DEVERR_BLOCK_ID);
    return nullptr;
  }
  return c.arena + (static_cast<size_t>(phys) * c.H + c.h) * Rec<KIND, D>::kBytes;
}

// Value group g of one token (whole warp; x = this lane's channel 32g + lane):
// its (scale, min) word, its high plane (2-bit cells: its only plane) in the
// block's column-major layout (byte 16 j + row = the token's channels 4j ..
// 4j + 3), and for 4-bit cells its low plane in the row-major layout.  rec
// may be null (the warp still takes part in the shuffles).
template <int KIND, int D>
__device__ __forceinline__ void store_value_group(uint8_t* rec, int row, int g, float x, int lane) {
  using R = Rec<KIND, D>;
  constexpr int BITS = KIND == LOOPKV_CELL_Q4 ? 4 : 2;
  constexpr bool kSplit = KIND == LOOPKV_CELL_Q4;
  constexpr int kVGroups = D / kGroup;
  float s_b, mn_b;
  group_params<BITS>(warp_min(x), warp_max(x), s_b, mn_b);
  const uint32_t code = group_code<BITS>(x, s_b, mn_b);
  // the high plane: 4 channels (lanes) per byte
  uint32_t byte = (kSplit ? code >> 2 : code) << (2 * (lane & 3));
  byte |= __shfl_xor_sync(0xffffffffu, byte, 1);
  byte |= __shfl_xor_sync(0xffffffffu, byte, 2);
  const uint32_t w_lo = kSplit ? half_warp_or((code & 3u) << (2 * (lane & 15))) : 0u;
  if (!rec) return;
  if ((lane & 3) == 0) rec[R::kVHi + (g * (kGroup / 4) + lane / 4) * kBlock + row] = static_cast<uint8_t>(byte);
  if (kSplit && (lane & 15) == 0)
    *reinterpret_cast<uint32_t*>(rec + R::kQ4VLo + row * R::kRow + (2 * g + (lane >> 4)) * 4) = w_lo;
  if (lane == 0) *reinterpret_cast<uint32_t*>(rec + R::kVMetaOff + (row * kVGroups + g) * 4) = meta_word(s_b, mn_b);
}

// Key group G (positions 32G .. 32G + 31), quantised per channel: lane =
// token, src = that token's exact key row (bf16[D]).  Warps warp, warp +
// nwarps, ... take the 16-channel chunks; every chunk writes the tokens'
// plane words and its channels' (scale, min) words (channels [0, D/2) in the
// group's even block, the rest in the odd one).
template <int KIND, int D>
__device__ __forceinline__ void store_key_group(const CellRows& c, int G, const __nv_bfloat16* src, int warp,
                                                int lane, int nwarps) {
  using R = Rec<KIND, D>;
  constexpr int BITS = KIND == LOOPKV_CELL_Q4 ? 4 : 2;
  constexpr bool kSplit = KIND == LOOPKV_CELL_Q4;
  constexpr int kChunks = D / 16;
  const int pos = G * kGroup + lane;
  for (int ck = warp; ck < kChunks; ck += nwarps) {
    uint32_t w_hi = 0, w_lo = 0;
#pragma unroll 4
    for (int i = 0; i < 16; ++i) {
      const int ch = ck * 16 + i;
      const float x = __bfloat162float(src[ch]);
      float s_b, mn_b;
      group_params<BITS>(warp_min(x), warp_max(x), s_b, mn_b);
      const uint32_t code = group_code<BITS>(x, s_b, mn_b);
      w_hi |= (kSplit ? code >> 2 : code) << (2 * i);
      if constexpr (kSplit) w_lo |= (code & 3u) << (2 * i);
      if (lane == 0) {
        uint8_t* mrec = record_at<KIND, D>(c, G * kGroup + (ch < D / 2 ? 0 : kBlock));
        if (mrec)
          *reinterpret_cast<uint32_t*>(mrec + R::kKMetaOff + (ch % (D / 2)) * 4) = meta_word(s_b, mn_b);
      }
    }
    uint8_t* rec = record_at<KIND, D>(c, pos);
    if (rec) {
      const int row = pos % kBlock;
      *reinterpret_cast<uint32_t*>(rec + R::kKHi + row * R::kRow + ck * 4) = w_hi;
      if constexpr (kSplit) *reinterpret_cast<uint32_t*>(rec + R::kQ4KLo + row * R::kRow + ck * 4) = w_lo;
    }
  }
}

}  // namespace loopkv
