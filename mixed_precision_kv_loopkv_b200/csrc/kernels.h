// Launch interface between the C-ABI layer and the kernels (internal).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "loopkv.h"

namespace loopkv {

struct AppendParams {              // H = KV heads here
  uint8_t* arena;                 // [num_blocks][H][record]
  __nv_bfloat16* residual;        // [max_batch][H][32][D], null for bf16 cells
  const __nv_bfloat16* k_new;     // [B][T][H][D]
  const __nv_bfloat16* v_new;     // [B][T][H][D]
  const int32_t* block_table;     // [B][max_blocks]
  const int32_t* start_pos;       // [B]
  int32_t* err;                   // optional
  int T, H, max_blocks, num_blocks;
};

struct DecodeParams {              // H = query heads, Hkv = KV heads
  const uint8_t* arena;           // source cell arena [num_blocks][Hkv][record]
  const __nv_bfloat16* residual;  // source cell key residual (4/2-bit) [max_batch][Hkv][32][D]
  const __nv_bfloat16* q;         // [B][H][D]
  const int32_t* block_table;     // [B][max_blocks]
  const int32_t* seq_lens;        // [B]
  __nv_bfloat16* out;             // [B][H][D]
  uint32_t* sel_mask;             // optional [B][H][mask_words]
  int32_t* sel_count;             // optional [B][H]
  int32_t* err;                   // optional
  int H, Hkv, g_log2, max_blocks, num_blocks, mask_words;  // H = Hkv << g_log2
  int chunk_groups;               // capacity (32-token groups) of one split
  int max_seq_len;
  float tau;
  float sm_scale_log2;            // sm_scale * log2(e)
  int sel_unit;                   // low-plane selection unit: 1, 16 or 32 tokens
  int pdl_early;                  // set by the launcher: signal dependents at kernel start (else after pass 1)
  // fused append (k_new non-null): seq_lens holds start positions; the
  // kernel first stores token start_pos[b] into the cell, then attends over
  // start_pos[b] + 1 tokens (negative start: sequence skipped)
  const __nv_bfloat16* k_new;     // [B][1][Hkv][D]
  const __nv_bfloat16* v_new;     // [B][1][Hkv][D]
  uint8_t* wr_arena;              // the same arena, writable
  __nv_bfloat16* wr_residual;     // the same key residual, writable
  // optional current token (k_cur non-null): its exact key and value join
  // the softmax after the seq_lens[b] stored tokens (no low plane)
  const __nv_bfloat16* k_cur;     // [B][Hkv][D]
  const __nv_bfloat16* v_cur;     // [B][Hkv][D]
};

cudaError_t launch_append(int kind, int head_dim, const AppendParams& p, int batch,
                          cudaStream_t stream, bool pdl);

// Query heads of one KV head whose CTAs share a cluster in a decode launch:
// G for 4-bit sources with tau > 0 (the union of their selections), else 1.
inline int head_cluster(int kind, int group, bool full_values) {
  return (kind == LOOPKV_CELL_Q4 && !full_values && group > 1) ? group : 1;
}

// Largest cluster: the portable size of 8 CTAs for splits alone, 16 (a
// non-portable size B200 supports) for splits x heads of grouped queries.
constexpr int kMaxClusterSplits = 8;
constexpr int kMaxClusterCtas = 16;

// Largest split count (a power of two) whose cluster of splits x hc CTAs
// stays within kMaxClusterCtas.
inline int max_splits(int hc) {
  int s = 1;
  while (s < kMaxClusterSplits && 2 * s * hc <= kMaxClusterCtas) s <<= 1;
  return s;
}

// Splits per (sequence, query head) chosen for a decode launch; hc as from
// head_cluster.
int decode_splits(int kind, int head_dim, int batch, int heads, int max_seq_len, int hc);

// Dynamic shared memory of one decode CTA whose split holds chunk_groups
// 32-token groups (0 for an unknown kind or head_dim).
size_t decode_smem_bytes(int kind, int head_dim, bool full_values, int chunk_groups);

cudaError_t launch_decode(int kind, int head_dim, const DecodeParams& p, int batch, int splits,
                          bool full_values, cudaStream_t stream, bool pdl);

}  // namespace loopkv
