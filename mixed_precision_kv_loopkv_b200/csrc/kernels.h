// Launch interface between the C-ABI layer and the kernels (internal).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace loopkv {

struct AppendParams {
  uint8_t* arena;                 // [num_blocks][H][record]
  __nv_bfloat16* residual;        // [max_batch][H][32][D], null for bf16 cells
  const __nv_bfloat16* k_new;     // [B][T][H][D]
  const __nv_bfloat16* v_new;     // [B][T][H][D]
  const int32_t* block_table;     // [B][max_blocks]
  const int32_t* start_pos;       // [B]
  int32_t* err;                   // optional
  int T, H, max_blocks, num_blocks;
};

struct DecodeParams {
  const uint8_t* arena;           // source cell arena
  const __nv_bfloat16* residual;  // source cell key residual (4/2-bit)
  const __nv_bfloat16* q;         // [B][H][D]
  const int32_t* block_table;     // [B][max_blocks]
  const int32_t* seq_lens;        // [B]
  __nv_bfloat16* out;             // [B][H][D]
  uint32_t* sel_mask;             // optional [B][H][mask_words]
  int32_t* sel_count;             // optional [B][H]
  int32_t* err;                   // optional
  int H, max_blocks, num_blocks, mask_words;
  int chunk_groups;               // capacity (32-token groups) of one split
  int max_seq_len;
  float tau;
  float sm_scale_log2;            // sm_scale * log2(e)
  int sel_unit;                   // low-plane selection unit: 1, 16 or 32 tokens
  // fused append (k_new non-null): seq_lens holds start positions; the
  // kernel first stores token start_pos[b] into the cell, then attends over
  // start_pos[b] + 1 tokens (negative start: sequence skipped)
  const __nv_bfloat16* k_new;     // [B][1][H][D]
  const __nv_bfloat16* v_new;     // [B][1][H][D]
  uint8_t* wr_arena;              // the same arena, writable
  __nv_bfloat16* wr_residual;     // the same key residual, writable
};

cudaError_t launch_append(int kind, int head_dim, const AppendParams& p, int batch,
                          cudaStream_t stream, bool pdl);

// Splits per (sequence, head) chosen for a decode launch.
int decode_splits(int kind, int head_dim, int batch, int heads, int max_seq_len);

cudaError_t launch_decode(int kind, int head_dim, const DecodeParams& p, int batch, int splits,
                          bool full_values, cudaStream_t stream, bool pdl);

}  // namespace loopkv
