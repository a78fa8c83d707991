/*
 * loopkv.h -- C ABI of the LoopKV decode path on B200 (sm_100a).
 *
 * LoopKV: Loop-Aware KV Cache Compression for Serving Looped Transformers
 * (Abstract): a looped transformer keeps one KV cell per (loop, layer); an
 * offline plan stores each cell as 4-bit, as 2-bit, or as a reuse of the
 * final loop's cell of the same layer.  A 4-bit value is stored as two
 * 2-bit planes (its top and bottom bits); a decode step reads the top plane
 * of every token and the bottom plane only of tokens that the cell's own
 * query weights heavily enough, and one kernel launch per cell carries out
 * its planned precision.
 *
 * The abstract leaves the storage format open.  This library fixes it:
 *   - asymmetric quantisation with bf16 scale and minimum; keys per channel
 *     over 32-token groups aligned at positions 0, 32, 64, ...; values per
 *     token over 32-channel groups;
 *   - key tokens of an unfinished group wait, exact, in a bf16 key residual;
 *   - a token takes its low plane when its fp32 softmax weight is >= tau;
 *     its high-plane-only value is the bucket midpoint min + s * (4 hi + 1.5).
 *
 * Paged storage (PagedAttention-style blocks, background from the same
 * pages' listing of serving papers): a stored cell owns one arena
 *   uint8 arena[num_blocks][Hkv][record]     (Hkv = KV heads, see loopkv_config)
 * addressed through a block table int32[batch][max_blocks_per_seq] that maps
 * logical block (token / block_size) to a physical block id.  One record holds
 * block_size (16) tokens of one head:
 *   4-bit : [K hi plane][K lo plane][K meta][V hi plane][V meta][V lo plane]
 *   2-bit : [K plane][K meta][V plane][V meta]
 *   bf16  : [K rows bf16][V rows bf16]
 * row-major plane (K planes, V lo plane) = 16 rows of D/4 bytes, one row per
 *              token; channel c of a row at byte c/4, bits 2*(c%4) and
 *              2*(c%4)+1 (least significant first);
 * column-major plane (V hi plane, 2-bit V plane) = the same bytes
 *              transposed: D/4 columns of 16 bytes, byte 16*(c/4) + t holds
 *              token t's channels 4*(c/4) .. 4*(c/4)+3 (same bit order), so
 *              that one 32-bit word holds one 4-channel column of 4 tokens;
 * K meta     = (scale, min) bf16 pairs (scale in the low half of each 32-bit
 *              word) of the 32-token key group: channels [0, D/2) in the
 *              group's even block, [D/2, D) in its odd block;
 * V meta     = (scale, min) per token row and 32-channel group, row-major.
 * At D = 128 a record is 2560 B (4-bit), 1536 B (2-bit) or 8192 B (bf16),
 * i.e. 160, 96 or 512 bytes per token and head.
 *
 * Conventions for every entry point:
 *   - pointers named "device" are caller-owned device memory; "host" ones are
 *     read during the call only;
 *   - the library allocates nothing, never synchronises, and enqueues its
 *     kernels on the caller's stream (a cudaStream_t passed as void*, NULL =
 *     the legacy default stream);
 *   - argument errors are returned synchronously and nothing is launched;
 *     LOOPKV_ERR_CUDA reports a failed launch;
 *   - faults found on the device (bad block id, sequence longer than its
 *     table or than max_seq_len, a bounded wait that gave up) are OR-ed into
 *     the optional device word *err_flag as LOOPKV_DEVERR_* bits and the
 *     affected (sequence, head) is skipped (decode writes zeros for it);
 *     kernels never trap;
 *   - the library's only global state is host-side launch settings: each
 *     kernel build's shared-memory limit and cluster permission are set once
 *     per device, and SM counts and occupancy answers are cached, all behind
 *     locks; concurrent calls from several host threads or on different
 *     streams are safe as long as they do not write the same cells.
 * Inputs must be finite; the fp32 key arithmetic assumes |q * scale * sm_scale|
 * below 2^40.  Value weights are carried in fixed point scaled per warp to
 * the largest value scale seen, so value scales have no limit of their own.
 */
#ifndef LOOPKV_H
#define LOOPKV_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LOOPKV_API __attribute__((visibility("default")))
#else
#define LOOPKV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LOOPKV_OK = 0,
  LOOPKV_ERR_INVALID_ARG = 1,  /* null pointer, bad size, bad tau, misaligned buffer */
  LOOPKV_ERR_BAD_PLAN = 2,     /* unknown kind, or a reuse cell in the final loop */
  LOOPKV_ERR_UNSUPPORTED = 3,  /* head_dim not 64/128, block_size not 16, too long */
  LOOPKV_ERR_CUDA = 4          /* a CUDA launch or attribute call failed */
} loopkv_status;

/* Plan entry of one (loop, layer) cell. */
typedef enum {
  LOOPKV_CELL_Q4 = 0,    /* 4-bit, split into high and low 2-bit planes */
  LOOPKV_CELL_Q2 = 1,    /* 2-bit */
  LOOPKV_CELL_REUSE = 2, /* reads the final loop's cell of the same layer */
  LOOPKV_CELL_BF16 = 3   /* unquantised bf16 (comparison runs) */
} loopkv_cell_kind;

/* Bits OR-ed into *err_flag by the kernels. */
#define LOOPKV_DEVERR_BLOCK_ID 0x1 /* block-table entry outside [0, num_blocks) */
#define LOOPKV_DEVERR_SEQ_LEN 0x2  /* length beyond the block table or max_seq_len */
#define LOOPKV_DEVERR_TIMEOUT 0x4  /* a bounded wait on the device gave up */
#define LOOPKV_DEVERR_RANGE 0x8    /* reserved (no longer raised: value scales
                                      have no limit) */

/* loopkv_config.flags */
#define LOOPKV_FLAG_PDL 0x1 /* programmatic dependent launch: a kernel may start
                               while the previous kernel on the stream drains.
                               The append kernel reads start_pos and the block
                               table before it waits, and touches nothing else
                               until then.  The decode kernel reads seq_lens and the
                               block table, and streams the cache blocks of the
                               32-token groups before the one holding token
                               seq_len - 1, before it waits: the previous kernel
                               must not write those (a decode step's append only
                               writes that last group and the key residual). */
#define LOOPKV_FLAG_SELECT_BLOCK 0x2 /* coarser low-plane selection: every token of
                               an aligned 16-token block takes its low plane when
                               the block's largest fp32 weight is >= tau */
#define LOOPKV_FLAG_SELECT_GROUP 0x4 /* the same over aligned 32-token groups
                               (at most one of the two selection flags) */

typedef struct {
  int32_t num_loops;          /* L */
  int32_t num_layers;         /* N (layers of the shared block) */
  int32_t num_heads;          /* query heads H */
  int32_t head_dim;           /* D: 64 or 128 */
  int32_t block_size;         /* tokens per paged block: 16 */
  int32_t num_blocks;         /* physical blocks in every stored cell's arena */
  int32_t max_batch;          /* sequences the key residuals hold */
  int32_t max_blocks_per_seq; /* columns of the block table */
  uint32_t flags;             /* LOOPKV_FLAG_* */
  int32_t decode_splits;      /* context splits per (sequence, head) for decode:
                                 0 = automatic, else 1, 2, 4 or 8 */
  const uint8_t* plan;        /* host [L*N] loopkv_cell_kind, cell = loop*N + layer */
  int32_t num_kv_heads;       /* KV heads Hkv; 0 = num_heads (MHA).  Grouped
                                 queries: num_heads = G * Hkv with G = 1, 2, 4
                                 or 8 query heads per KV head; query head h
                                 reads KV head h / G */
} loopkv_config;

typedef struct {
  /* host [L*N] arrays of device pointers, indexed like plan; NULL for reuse cells */
  void* const* arena;        /* uint8 [num_blocks][Hkv][record], 16-byte aligned */
  void* const* key_residual; /* bf16 [max_batch][Hkv][32][D] for 4/2-bit cells, else NULL */
} loopkv_cells;

/* Bytes of one (block, head) record of a stored cell kind (0 if unsupported). */
LOOPKV_API size_t loopkv_record_bytes(int32_t head_dim, int32_t block_size, int32_t kind);

/* Bytes of one stored cell's arena: num_blocks * Hkv * record. */
LOOPKV_API size_t loopkv_arena_bytes(const loopkv_config* cfg, int32_t kind);

/* Bytes of one key residual: max_batch * Hkv * 32 * head_dim * 2. */
LOOPKV_API size_t loopkv_residual_bytes(const loopkv_config* cfg);

/*
 * Append num_tokens new tokens to the cell (loop, layer) of every sequence b
 * at positions start_pos[b] .. start_pos[b] + num_tokens - 1.
 *
 * Values are quantised per token at once (4-bit: both planes); keys go to the
 * key residual and a 32-token key group is quantised per channel, and its
 * planes and meta written, when its last token arrives.  bf16 cells store the
 * rows unchanged.  A bulk append and the same tokens appended one at a time
 * produce identical arena bytes.
 *
 *   k_new, v_new : device bf16 [batch][num_tokens][Hkv][D]
 *   block_table  : device int32 [batch][max_blocks_per_seq]
 *   start_pos    : device int32 [batch]; a negative entry skips that sequence
 *   err_flag     : optional device int32 (LOOPKV_DEVERR_* bits)
 * Errors: INVALID_ARG for a reuse cell, null pointers, batch outside
 * [0, max_batch] or num_tokens < 0; BAD_PLAN / UNSUPPORTED as for the config.
 */
LOOPKV_API loopkv_status loopkv_quantize_append(const loopkv_config* cfg, const loopkv_cells* cells,
                                     int32_t loop, int32_t layer, const void* k_new,
                                     const void* v_new, const int32_t* block_table,
                                     const int32_t* start_pos, int32_t batch, int32_t num_tokens,
                                     int32_t* err_flag, void* stream);

/*
 * Fused decode attention of one query per (sequence, head) over the cell
 * (loop, layer), executing its plan entry: a reuse cell reads the final
 * loop's cell of the same layer with its own query.  Keys are dequantised at
 * the source cell's precision.  For 4-bit sources, every value contributes its
 * high-plane midpoint; tokens with fp32 softmax weight p >= tau then add their
 * low plane (tau = 0: all tokens, tau = +inf: none).
 * Grouped queries (G = H / Hkv > 1): the G query heads of a KV head each keep
 * their own softmax weights, and a token's low plane is fetched when any of
 * them selects it; it then serves all G heads (their values are full 4-bit
 * on the union of the heads' selections).  sel_mask and sel_count report
 * that union for every head of the group.
 * The current token (optional k_cur, v_cur): a looped model computes the
 * current token's K and V in every loop, but a reuse cell stores nothing and
 * the final loop's cell does not hold that token yet, so a reuse cell of an
 * earlier loop passes its own loop's rows here.  They join the softmax as one
 * more token after the seq_lens[b] stored ones, with their exact bf16 key and
 * value and no low plane; the stored tokens' weights, and so the low-plane
 * selection, are taken in that softmax (LoopKV abstract: a reuse cell reads
 * the final loop's KV; the current token's own entry is this library's
 * reading of causal attention in such a cell).
 *
 *   q           : device bf16 [batch][H][D]
 *   k_cur, v_cur: optional device bf16 [batch][Hkv][D] (both or neither)
 *   block_table : device int32 [batch][max_blocks_per_seq]
 *   seq_lens    : device int32 [batch], each in [0, max_seq_len]
 *   max_seq_len : host upper bound on seq_lens (sizes the split over the
 *                 context); 0 means max_blocks_per_seq * block_size
 *   tau         : >= 0 or +INF;  sm_scale: logit = sm_scale * q . k
 *   out         : device bf16 [batch][H][D]; zeros where seq_len = 0 and no
 *                 current token is given
 *   sel_mask    : optional device uint32 [batch][H][W], W = ceil(max_blocks_per_seq
 *                 * block_size / 32); bit t%32 of word t/32 = token t took its low
 *                 plane; words past ceil(seq_len/32) are not written
 *   sel_count   : optional device int32 [batch][H], number of selected tokens
 *                 (2-bit and bf16 sources have no low plane: zero words, zero
 *                 counts)
 *   err_flag    : optional device int32
 * Errors: INVALID_ARG for tau < 0 or NaN, null required pointers, only one of
 * k_cur / v_cur, batch outside [0, max_batch]; BAD_PLAN; UNSUPPORTED for
 * max_seq_len above 65536, for a 4-bit source with G x decode_splits above 16
 * (the CTAs of one KV head's query heads and splits form one thread-block
 * cluster), or for a context split too long for one CTA's shared memory.
 */
LOOPKV_API loopkv_status loopkv_decode_attention(const loopkv_config* cfg, const loopkv_cells* cells,
                                      int32_t loop, int32_t layer, const void* q, const void* k_cur,
                                      const void* v_cur, const int32_t* block_table,
                                      const int32_t* seq_lens, int32_t batch, int32_t max_seq_len, float tau,
                                      float sm_scale, void* out, uint32_t* sel_mask,
                                      int32_t* sel_count, int32_t* err_flag, void* stream);

/*
 * One decode step of a stored cell in a single launch: appends token
 * start_pos[b] (one new token per sequence) exactly as loopkv_quantize_append
 * with num_tokens = 1 would, then attends over start_pos[b] + 1 tokens exactly
 * as loopkv_decode_attention would with seq_lens = start_pos + 1.  This is
 * one launch per cell, as the LoopKV abstract describes its serving kernel,
 * with the store of the current token folded in: the split holding the new
 * token writes it before it reads that token's group.
 *
 *   k_new, v_new : device bf16 [batch][1][Hkv][D]
 *   start_pos    : device int32 [batch]; a negative entry skips that sequence
 *                  (nothing stored, zeros out)
 *   max_seq_len  : host upper bound on start_pos + 1; 0 means the capacity
 *   other arguments as for loopkv_decode_attention
 * Errors: as loopkv_decode_attention, INVALID_ARG for a reuse cell or
 * null k_new / v_new, and UNSUPPORTED with grouped queries (G > 1: append
 * with loopkv_quantize_append, then decode).  Device faults: LOOPKV_DEVERR_SEQ_LEN for start_pos + 1
 * above max_seq_len or the capacity, BLOCK_ID as for the append.
 */
LOOPKV_API loopkv_status loopkv_append_decode_attention(
    const loopkv_config* cfg, const loopkv_cells* cells, int32_t loop, int32_t layer, const void* k_new,
    const void* v_new, const void* q, const int32_t* block_table, const int32_t* start_pos, int32_t batch,
    int32_t max_seq_len, float tau, float sm_scale, void* out, uint32_t* sel_mask, int32_t* sel_count,
    int32_t* err_flag, void* stream);

/*
 * Offline plan of every (loop, layer) cell from a synthetic damage table
 * (host only, no GPU).  The LoopKV abstract describes a planner that picks
 * 4-bit, 2-bit or reuse per cell to minimise the bytes read per decoded
 * token under budgets on predicted (additive) damage and storage; the
 * formulation here is the library's reading:
 *   damage       : host int32 [L*N][3], the damage of cell (loop*N + layer)
 *                  stored 4-bit / 2-bit / as a reuse (column 2 of the final
 *                  loop is ignored: those cells cannot reuse); >= 0
 *   damage_budget: sum of the chosen damages must not exceed it
 *   storage_budget: sum of storage in 32-byte units per token-head
 *                  (4-bit 5, 2-bit 3, reuse 0) must not exceed it
 *   q4_read_bytes: bytes a 4-bit cell reads per token-head (128 plus the
 *                  expected low-plane share); 2-bit reads 96; a reuse cell
 *                  reads what its source (the final loop's cell) reads
 *   plan_out     : host uint8 [L*N], LOOPKV_CELL_Q4 / _Q2 / _REUSE
 *   reads_out    : optional host int64, total reads per token-head
 * The plan minimises total reads; among plans of equal reads it has the
 * least damage, then the least storage.  Exact (dynamic program over layers
 * with (damage, storage) states).  Errors: INVALID_ARG for bad sizes,
 * negative inputs or num_loops > 6; UNSUPPORTED when (damage_budget + 1) x
 * (storage_budget + 1) x num_layers exceeds 2^25 states; BAD_PLAN when no
 * plan meets the budgets (plan_out untouched).
 */
LOOPKV_API loopkv_status loopkv_plan_cells(int32_t num_loops, int32_t num_layers, const int32_t* damage,
                                           int32_t damage_budget, int32_t storage_budget,
                                           int32_t q4_read_bytes, uint8_t* plan_out, int64_t* reads_out);

/* Context splits (CTAs per sequence and query head) a decode call over a
 * source cell of the given kind would launch; 0 for invalid arguments or an
 * unsupported split. */
LOOPKV_API int32_t loopkv_decode_splits(const loopkv_config* cfg, int32_t kind, int32_t batch,
                             int32_t max_seq_len);

/*
 * Self-test of the device's bounded waits: one kernel waits on an mbarrier
 * whose phase never completes.  The wait gives up after the kernels' fixed
 * limit (2 s by the global timer), ORs LOOPKV_DEVERR_TIMEOUT into *err_flag
 * and the kernel exits; the context stays usable.  *elapsed_ns receives the
 * time the wait took.  Both pointers are device memory; the call returns at
 * once (the kernel runs on the stream).  Errors: INVALID_ARG for null
 * pointers, CUDA for a failed launch.
 */
LOOPKV_API loopkv_status loopkv_selftest_wait_timeout(int32_t* err_flag, uint64_t* elapsed_ns, void* stream);

/* Static text for a status code. */
LOOPKV_API const char* loopkv_status_string(loopkv_status status);

#ifdef __cplusplus
}
#endif

#endif /* LOOPKV_H */
