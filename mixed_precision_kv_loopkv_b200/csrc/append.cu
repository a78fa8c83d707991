// Quantise-append of new K/V tokens into a LoopKV cell (sm_100a).
//
// LoopKV: Loop-Aware KV Cache Compression for Serving Looped Transformers,
// Abstract: cells are stored 4-bit (as high and low 2-bit planes) or 2-bit.
// The quantiser is the library's reading of the open format: asymmetric, with
// bf16 scale and minimum; values per token over 32-channel groups, keys per
// channel over 32-token groups.  Every step of the quantiser is one correctly
// rounded fp32 operation (no contraction), so the integer codes are exactly
// reproducible on any IEEE machine.
//
// One CTA per (head, sequence):
//   1. each new value token: four warps quantise its 32-channel groups (one
//      lane per channel) and write its planes and the (scale, min) word;
//   2. every key group completed by this call (its 32nd token arrives):
//      quantised per channel (one lane per token) from the new tokens and the
//      exact ones waiting in the key residual; planes and meta written;
//   3. after a CTA barrier, the new tokens of the still-open group are copied
//      into the key residual (after step 2 read the residual).
#include "append_ops.cuh"
#include "kernels.h"

namespace loopkv {
namespace {

template <int KIND, int D>
__global__ void __launch_bounds__(128) append_kernel(const AppendParams p) {
  using R = Rec<KIND, D>;
  // Let the next kernel (a decode of this cell) launch and stream the cache
  // blocks this kernel does not write.
  pdl_allow_dependents();

  const int h = blockIdx.x, b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = p.T;
  // The start position and the block table are not written by the previous
  // kernel: read them (and the first new token's record) before waiting.
  const int start = p.start_pos[b];
  const int end = start + T;
  const bool in_range = start >= 0 && end <= p.max_blocks * kBlock;
  const CellRows cell{p.arena, p.block_table + static_cast<size_t>(b) * p.max_blocks, p.err, p.H, h,
                      p.max_blocks, p.num_blocks};
  uint8_t* const rec_first = in_range ? record_at<KIND, D>(cell, start) : nullptr;
  // then wait for the kernel before this one, which may produce the new tokens
  pdl_wait_prior_grid();
  if (start < 0) return;  // sequence not appended to in this call
  if (!in_range) {
    if (threadIdx.x == 0) flag_error(p.err, LOOPKV_DEVERR_SEQ_LEN);
    return;
  }
  const size_t tok_stride = static_cast<size_t>(p.H) * D;
  const __nv_bfloat16* kb = p.k_new + (static_cast<size_t>(b) * T * p.H + h) * D;
  const __nv_bfloat16* vb = p.v_new + (static_cast<size_t>(b) * T * p.H + h) * D;
  constexpr int kVecPerRow = D * 2 / 16;

  if constexpr (KIND == LOOPKV_CELL_BF16) {
    for (int i = threadIdx.x; i < T * kVecPerRow; i += blockDim.x) {
      const int t = i / kVecPerRow, c = i % kVecPerRow;
      const int pos = start + t;
      uint8_t* rec = t == 0 ? rec_first : record_at<KIND, D>(cell, pos);
      if (!rec) continue;
      const int row = pos % kBlock;
      reinterpret_cast<uint4*>(rec + R::kBfK + row * D * 2)[c] =
          reinterpret_cast<const uint4*>(kb + t * tok_stride)[c];
      reinterpret_cast<uint4*>(rec + R::kBfV + row * D * 2)[c] =
          reinterpret_cast<const uint4*>(vb + t * tok_stride)[c];
    }
    return;
  } else {
    constexpr int kVGroups = D / kGroup;

    // 1. values, one token and 32-channel group per warp iteration
    for (int item = warp; item < T * kVGroups; item += 4) {
      const int t = item / kVGroups, g = item % kVGroups;
      const int pos = start + t;
      const float x = __bfloat162float(vb[t * tok_stride + g * kGroup + lane]);
      uint8_t* rec = t == 0 ? rec_first : record_at<KIND, D>(cell, pos);
      store_value_group<KIND, D>(rec, pos % kBlock, g, x, lane);
    }

    // 2. key groups completed by this call: groups [start/32, end/32 - 1]
    __nv_bfloat16* res = p.residual + (static_cast<size_t>(b) * p.H + h) * kGroup * D;
    const int g_first = start / kGroup, g_last = end / kGroup - 1;
    for (int G = g_first; G <= g_last; ++G) {
      const int pos = G * kGroup + lane;  // this lane's token
      const __nv_bfloat16* src =
          pos >= start ? kb + static_cast<size_t>(pos - start) * tok_stride : res + lane * D;
      store_key_group<KIND, D>(cell, G, src, warp, lane, 4);
    }
    __syncthreads();

    // 3. new tokens of the still-open key group wait in the residual
    const int tail0 = max(start, (end / kGroup) * kGroup);
    for (int i = threadIdx.x; i < (end - tail0) * kVecPerRow; i += blockDim.x) {
      const int pos = tail0 + i / kVecPerRow, c = i % kVecPerRow;
      reinterpret_cast<uint4*>(res + (pos % kGroup) * D)[c] =
          reinterpret_cast<const uint4*>(kb + static_cast<size_t>(pos - start) * tok_stride)[c];
    }
  }
}

template <int KIND, int D>
cudaError_t launch_append_t(const AppendParams& p, int batch, cudaStream_t stream, bool pdl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.H, batch, 1);
  cfg.blockDim = dim3(128, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  if (pdl) {
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  return cudaLaunchKernelEx(&cfg, append_kernel<KIND, D>, p);
}

}  // namespace

cudaError_t launch_append(int kind, int head_dim, const AppendParams& p, int batch,
                          cudaStream_t stream, bool pdl) {
  if (batch == 0 || p.T == 0) return cudaSuccess;
  switch (kind * 1000 + head_dim) {
    case LOOPKV_CELL_Q4 * 1000 + 128: return launch_append_t<LOOPKV_CELL_Q4, 128>(p, batch, stream, pdl);
    case LOOPKV_CELL_Q4 * 1000 + 64: return launch_append_t<LOOPKV_CELL_Q4, 64>(p, batch, stream, pdl);
    case LOOPKV_CELL_Q2 * 1000 + 128: return launch_append_t<LOOPKV_CELL_Q2, 128>(p, batch, stream, pdl);
    case LOOPKV_CELL_Q2 * 1000 + 64: return launch_append_t<LOOPKV_CELL_Q2, 64>(p, batch, stream, pdl);
    case LOOPKV_CELL_BF16 * 1000 + 128: return launch_append_t<LOOPKV_CELL_BF16, 128>(p, batch, stream, pdl);
    case LOOPKV_CELL_BF16 * 1000 + 64: return launch_append_t<LOOPKV_CELL_BF16, 64>(p, batch, stream, pdl);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace loopkv
