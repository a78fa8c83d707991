// C ABI of the LoopKV decode path: argument validation, record sizes, plan
// resolution (a reuse cell reads the final loop's cell of its layer) and
// kernel dispatch.  See include/loopkv.h for the contract of every call.
#include <math.h>
#include <stdint.h>

#include "kernels.h"
#include "loopkv.h"

namespace {

constexpr int kMaxSeqLen = 65536;
constexpr size_t kMaxSmemPerCta = 227u * 1024u;  // opt-in dynamic shared memory of one CTA

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// KV heads of a config (0 in num_kv_heads: one per query head).
int kv_heads(const loopkv_config* cfg) { return cfg->num_kv_heads ? cfg->num_kv_heads : cfg->num_heads; }

bool stored_kind(int k) {
  return k == LOOPKV_CELL_Q4 || k == LOOPKV_CELL_Q2 || k == LOOPKV_CELL_BF16;
}

loopkv_status check_config(const loopkv_config* cfg) {
  if (!cfg || !cfg->plan) return LOOPKV_ERR_INVALID_ARG;
  if (cfg->num_loops <= 0 || cfg->num_layers <= 0 || cfg->num_heads <= 0 || cfg->num_blocks < 0 ||
      cfg->max_batch < 0 || cfg->max_blocks_per_seq <= 0)
    return LOOPKV_ERR_INVALID_ARG;
  if (cfg->num_kv_heads < 0 || cfg->num_heads % kv_heads(cfg) != 0) return LOOPKV_ERR_INVALID_ARG;
  const int group = cfg->num_heads / kv_heads(cfg);  // query heads per KV head: 1, 2, 4 or 8
  if (group != 1 && group != 2 && group != 4 && group != 8) return LOOPKV_ERR_UNSUPPORTED;
  if (cfg->head_dim != 64 && cfg->head_dim != 128) return LOOPKV_ERR_UNSUPPORTED;
  if (cfg->block_size != 16) return LOOPKV_ERR_UNSUPPORTED;
  if ((cfg->flags & LOOPKV_FLAG_SELECT_BLOCK) && (cfg->flags & LOOPKV_FLAG_SELECT_GROUP))
    return LOOPKV_ERR_INVALID_ARG;
  const int s = cfg->decode_splits;
  if (s != 0 && s != 1 && s != 2 && s != 4 && s != 8) return LOOPKV_ERR_INVALID_ARG;
  const int L = cfg->num_loops, N = cfg->num_layers;
  for (int c = 0; c < L * N; ++c) {
    const int k = cfg->plan[c];
    if (k != LOOPKV_CELL_REUSE && !stored_kind(k)) return LOOPKV_ERR_BAD_PLAN;
    if (k == LOOPKV_CELL_REUSE && c / N == L - 1) return LOOPKV_ERR_BAD_PLAN;
  }
  return LOOPKV_OK;
}

loopkv_status cell_index(const loopkv_config* cfg, int loop, int layer, int* cell) {
  if (loop < 0 || loop >= cfg->num_loops || layer < 0 || layer >= cfg->num_layers)
    return LOOPKV_ERR_INVALID_ARG;
  *cell = loop * cfg->num_layers + layer;
  return LOOPKV_OK;
}

}  // namespace

extern "C" {

size_t loopkv_record_bytes(int32_t head_dim, int32_t block_size, int32_t kind) {
  if ((head_dim != 64 && head_dim != 128) || block_size != 16) return 0;
  const size_t plane = static_cast<size_t>(block_size) * head_dim / 4;
  const size_t kmeta = static_cast<size_t>(head_dim / 2) * 4;
  const size_t vmeta = static_cast<size_t>(block_size) * (head_dim / 32) * 4;
  switch (kind) {
    case LOOPKV_CELL_Q4: return 4 * plane + kmeta + vmeta;
    case LOOPKV_CELL_Q2: return 2 * plane + kmeta + vmeta;
    case LOOPKV_CELL_BF16: return static_cast<size_t>(block_size) * head_dim * 4;
    default: return 0;
  }
}

size_t loopkv_arena_bytes(const loopkv_config* cfg, int32_t kind) {
  if (!cfg || cfg->num_blocks < 0 || cfg->num_heads <= 0 || cfg->num_kv_heads < 0) return 0;
  return static_cast<size_t>(cfg->num_blocks) * kv_heads(cfg) *
         loopkv_record_bytes(cfg->head_dim, cfg->block_size, kind);
}

size_t loopkv_residual_bytes(const loopkv_config* cfg) {
  if (!cfg || cfg->max_batch < 0 || cfg->num_heads <= 0 || cfg->num_kv_heads < 0) return 0;
  return static_cast<size_t>(cfg->max_batch) * kv_heads(cfg) * 32 * cfg->head_dim * 2;
}

loopkv_status loopkv_quantize_append(const loopkv_config* cfg, const loopkv_cells* cells,
                                     int32_t loop, int32_t layer, const void* k_new,
                                     const void* v_new, const int32_t* block_table,
                                     const int32_t* start_pos, int32_t batch, int32_t num_tokens,
                                     int32_t* err_flag, void* stream) {
  loopkv_status st = check_config(cfg);
  if (st != LOOPKV_OK) return st;
  int cell;
  if ((st = cell_index(cfg, loop, layer, &cell)) != LOOPKV_OK) return st;
  const int kind = cfg->plan[cell];
  if (kind == LOOPKV_CELL_REUSE) return LOOPKV_ERR_INVALID_ARG;  // reuse cells store nothing
  if (!cells || !cells->arena || !cells->key_residual) return LOOPKV_ERR_INVALID_ARG;
  if (batch < 0 || batch > cfg->max_batch || num_tokens < 0) return LOOPKV_ERR_INVALID_ARG;
  if (batch == 0 || num_tokens == 0) return LOOPKV_OK;
  void* arena = cells->arena[cell];
  void* residual = cells->key_residual[cell];
  if (!arena || !aligned16(arena)) return LOOPKV_ERR_INVALID_ARG;
  if (kind != LOOPKV_CELL_BF16 && (!residual || !aligned16(residual))) return LOOPKV_ERR_INVALID_ARG;
  if (!k_new || !v_new || !aligned16(k_new) || !aligned16(v_new) || !block_table || !start_pos)
    return LOOPKV_ERR_INVALID_ARG;

  loopkv::AppendParams p;
  p.arena = static_cast<uint8_t*>(arena);
  p.residual = static_cast<__nv_bfloat16*>(residual);
  p.k_new = static_cast<const __nv_bfloat16*>(k_new);
  p.v_new = static_cast<const __nv_bfloat16*>(v_new);
  p.block_table = block_table;
  p.start_pos = start_pos;
  p.err = err_flag;
  p.T = num_tokens;
  p.H = kv_heads(cfg);
  p.max_blocks = cfg->max_blocks_per_seq;
  p.num_blocks = cfg->num_blocks;
  const cudaError_t e = loopkv::launch_append(kind, cfg->head_dim, p, batch,
                                              static_cast<cudaStream_t>(stream),
                                              (cfg->flags & LOOPKV_FLAG_PDL) != 0);
  return e == cudaSuccess ? LOOPKV_OK : LOOPKV_ERR_CUDA;
}

int32_t loopkv_decode_splits(const loopkv_config* cfg, int32_t kind, int32_t batch,
                             int32_t max_seq_len) {
  if (check_config(cfg) != LOOPKV_OK || !stored_kind(kind) || batch < 0) return 0;
  const int cap = cfg->max_blocks_per_seq * cfg->block_size;
  const int len = max_seq_len == 0 ? cap : max_seq_len;
  if (len < 0 || len > cap || len > kMaxSeqLen) return 0;
  const int hc = loopkv::head_cluster(kind, cfg->num_heads / kv_heads(cfg), false);
  if (cfg->decode_splits) return cfg->decode_splits <= loopkv::max_splits(hc) ? cfg->decode_splits : 0;
  return loopkv::decode_splits(kind, cfg->head_dim, batch, cfg->num_heads, len, hc);
}

}  // extern "C"

namespace {

// Shared by the plain decode and the fused append + decode: validation,
// split choice and launch.  k_new == nullptr: plain decode over seq_lens;
// otherwise seq_lens holds start positions and the cell must be stored.
loopkv_status decode_common(const loopkv_config* cfg, const loopkv_cells* cells, int32_t loop, int32_t layer,
                            const void* k_new, const void* v_new, const void* q, const void* k_cur,
                            const void* v_cur, const int32_t* block_table,
                            const int32_t* seq_lens, int32_t batch, int32_t max_seq_len, float tau,
                            float sm_scale, void* out, uint32_t* sel_mask, int32_t* sel_count,
                            int32_t* err_flag, void* stream) {
  loopkv_status st = check_config(cfg);
  if (st != LOOPKV_OK) return st;
  int cell;
  if ((st = cell_index(cfg, loop, layer, &cell)) != LOOPKV_OK) return st;
  const bool fused = k_new != nullptr || v_new != nullptr;
  // a reuse cell reads the final loop's cell of the same layer with its own query
  if (fused && cfg->plan[cell] == LOOPKV_CELL_REUSE) return LOOPKV_ERR_INVALID_ARG;
  const int src = cfg->plan[cell] == LOOPKV_CELL_REUSE
                      ? (cfg->num_loops - 1) * cfg->num_layers + layer
                      : cell;
  const int kind = cfg->plan[src];
  if (!cells || !cells->arena || !cells->key_residual) return LOOPKV_ERR_INVALID_ARG;
  if (batch < 0 || batch > cfg->max_batch) return LOOPKV_ERR_INVALID_ARG;
  if (isnan(tau) || tau < 0.f || !isfinite(sm_scale)) return LOOPKV_ERR_INVALID_ARG;
  const int cap = cfg->max_blocks_per_seq * cfg->block_size;
  const int len = max_seq_len == 0 ? cap : max_seq_len;
  if (len < 0 || len > cap) return LOOPKV_ERR_INVALID_ARG;
  if (len > kMaxSeqLen) return LOOPKV_ERR_UNSUPPORTED;
  if (batch == 0) return LOOPKV_OK;
  void* arena = cells->arena[src];
  void* residual = cells->key_residual[src];
  if (!arena || !aligned16(arena)) return LOOPKV_ERR_INVALID_ARG;
  if (kind != LOOPKV_CELL_BF16 && (!residual || !aligned16(residual))) return LOOPKV_ERR_INVALID_ARG;
  if (!q || !aligned16(q) || !out || !block_table || !seq_lens) return LOOPKV_ERR_INVALID_ARG;
  if (fused && (!k_new || !v_new || !aligned16(k_new) || !aligned16(v_new))) return LOOPKV_ERR_INVALID_ARG;
  // the current token: both rows or neither
  if ((k_cur == nullptr) != (v_cur == nullptr)) return LOOPKV_ERR_INVALID_ARG;
  const int group = cfg->num_heads / kv_heads(cfg);  // query heads per KV head
  // grouped queries append through loopkv_quantize_append: in one launch the
  // other heads' CTAs would read the new token before its writer is done
  if (fused && group > 1) return LOOPKV_ERR_UNSUPPORTED;

  const bool full_values = kind == LOOPKV_CELL_Q4 && tau == 0.f;
  // splits are capped for every 4-bit source (also tau = 0) so that the
  // choice does not depend on tau; the launch clusters heads only for tau > 0
  const int hc = loopkv::head_cluster(kind, group, false);
  if (cfg->decode_splits > loopkv::max_splits(hc)) return LOOPKV_ERR_UNSUPPORTED;
  const int splits = cfg->decode_splits
                         ? cfg->decode_splits
                         : loopkv::decode_splits(kind, cfg->head_dim, batch, cfg->num_heads, len, hc);
  const int groups = (len + 31) / 32;
  loopkv::DecodeParams p;
  p.arena = static_cast<const uint8_t*>(arena);
  p.residual = static_cast<const __nv_bfloat16*>(residual);
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.block_table = block_table;
  p.seq_lens = seq_lens;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.sel_mask = sel_mask;
  p.sel_count = sel_count;
  p.err = err_flag;
  p.H = cfg->num_heads;
  p.Hkv = kv_heads(cfg);
  p.g_log2 = group == 8 ? 3 : group == 4 ? 2 : group == 2 ? 1 : 0;
  p.max_blocks = cfg->max_blocks_per_seq;
  p.num_blocks = cfg->num_blocks;
  p.mask_words = (cap + 31) / 32;
  p.chunk_groups = (groups + splits - 1) / splits;
  // one split's logits, block ids and selection words live in shared memory
  if (loopkv::decode_smem_bytes(kind, cfg->head_dim, full_values, p.chunk_groups) > kMaxSmemPerCta)
    return LOOPKV_ERR_UNSUPPORTED;
  p.max_seq_len = len;
  p.tau = tau;
  p.sm_scale_log2 = sm_scale * 1.4426950408889634f;
  p.sel_unit = (cfg->flags & LOOPKV_FLAG_SELECT_BLOCK) ? 16 : (cfg->flags & LOOPKV_FLAG_SELECT_GROUP) ? 32 : 1;
  p.k_new = static_cast<const __nv_bfloat16*>(k_new);
  p.v_new = static_cast<const __nv_bfloat16*>(v_new);
  p.wr_arena = fused ? static_cast<uint8_t*>(arena) : nullptr;
  p.wr_residual = fused ? static_cast<__nv_bfloat16*>(residual) : nullptr;
  p.k_cur = static_cast<const __nv_bfloat16*>(k_cur);
  p.v_cur = static_cast<const __nv_bfloat16*>(v_cur);
  const cudaError_t e = loopkv::launch_decode(kind, cfg->head_dim, p, batch, splits, full_values,
                                              static_cast<cudaStream_t>(stream),
                                              (cfg->flags & LOOPKV_FLAG_PDL) != 0);
  return e == cudaSuccess ? LOOPKV_OK : LOOPKV_ERR_CUDA;
}

}  // namespace

extern "C" {

loopkv_status loopkv_decode_attention(const loopkv_config* cfg, const loopkv_cells* cells,
                                      int32_t loop, int32_t layer, const void* q, const void* k_cur,
                                      const void* v_cur, const int32_t* block_table, const int32_t* seq_lens,
                                      int32_t batch, int32_t max_seq_len, float tau,
                                      float sm_scale, void* out, uint32_t* sel_mask,
                                      int32_t* sel_count, int32_t* err_flag, void* stream) {
  return decode_common(cfg, cells, loop, layer, nullptr, nullptr, q, k_cur, v_cur, block_table, seq_lens, batch,
                       max_seq_len, tau, sm_scale, out, sel_mask, sel_count, err_flag, stream);
}

loopkv_status loopkv_append_decode_attention(const loopkv_config* cfg, const loopkv_cells* cells,
                                             int32_t loop, int32_t layer, const void* k_new,
                                             const void* v_new, const void* q,
                                             const int32_t* block_table, const int32_t* start_pos,
                                             int32_t batch, int32_t max_seq_len, float tau,
                                             float sm_scale, void* out, uint32_t* sel_mask,
                                             int32_t* sel_count, int32_t* err_flag, void* stream) {
  if (!k_new || !v_new) return LOOPKV_ERR_INVALID_ARG;
  return decode_common(cfg, cells, loop, layer, k_new, v_new, q, nullptr, nullptr, block_table, start_pos, batch,
                       max_seq_len, tau, sm_scale, out, sel_mask, sel_count, err_flag, stream);
}

const char* loopkv_status_string(loopkv_status status) {
  switch (status) {
    case LOOPKV_OK: return "ok";
    case LOOPKV_ERR_INVALID_ARG: return "invalid argument";
    case LOOPKV_ERR_BAD_PLAN: return "bad plan";
    case LOOPKV_ERR_UNSUPPORTED: return "unsupported configuration";
    case LOOPKV_ERR_CUDA: return "CUDA launch failed";
    default: return "unknown status";
  }
}

}  // extern "C"
