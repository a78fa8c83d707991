"""Algorithmic bytes of the LoopKV decode path (what a launch must move).

Per (cell, sequence, head) of n tokens, with the source cell's record
format (include/loopkv.h) at head width D:
  4-bit: complete key groups read both key planes (2 * D/4 per token) and the
         key meta (4 bytes per channel per 32 tokens); values read the high
         plane (D/4) and meta (4 bytes per 32 channels) of every token and the
         low plane (D/4) of the selected tokens;
  2-bit: one key plane and one value plane, both metas;
  bf16 : 2 * D bytes of key and of value per token;
plus the exact bf16 key tail of an unfinished group, one block-table entry per
16 tokens, the bf16 query and the bf16 output.  At D = 128 that is 128 B per
token-head (+32 per selected token) for 4-bit, 96 for 2-bit, 512 for bf16.
"""

from __future__ import annotations

GROUP = 32
BLOCK = 16


def decode_bytes(kind: str, d: int, n: int, n_selected: int = 0) -> int:
    fixed = 2 * d * 2 + 4 * (-(-n // BLOCK))
    if n == 0:
        return 2 * d * 2
    if kind == "bf16":
        return fixed + n * 4 * d
    full = (n // GROUP) * GROUP
    plane = d // 4
    k_meta = (n // GROUP) * d * 4
    tail = (n - full) * d * 2
    v_meta = n * (d // GROUP) * 4
    if kind == "q4":
        return fixed + full * 2 * plane + k_meta + tail + n * plane + v_meta + n_selected * plane
    if kind == "q2":
        return fixed + full * plane + k_meta + tail + n * plane + v_meta
    raise ValueError(kind)


def step_bytes(plan, num_layers: int, num_loops: int, d: int, heads: int, lens_stored, lens_reuse,
               selected=None, cells=None, group: int = 1, reuse_current: bool = False) -> int:
    """Bytes of one looped decode step: every cell decodes every (sequence,
    head); stored cells over lens_stored[b] tokens, reuse cells over the
    final loop's lens_reuse[b]; selected[cell][b][h] low-plane rows.

    ``group`` query heads share one KV head (``heads`` counts query heads):
    the KV head's cache, and the low-plane rows of the union of the group's
    selections (reported identically for every head of the group), are
    counted once per group; queries and outputs once per query head.
    ``reuse_current``: reuse cells also read the current token's exact bf16
    K and V row (4 * D bytes per sequence and KV head)."""
    total = 0
    for cell, kind in enumerate(plan):
        if cells is not None and cell not in cells:
            continue
        src = cell if kind != "reuse" else (num_loops - 1) * num_layers + cell % num_layers
        src_kind = plan[src]
        lens = lens_reuse if kind == "reuse" else lens_stored
        for b, n in enumerate(lens):
            for hk in range(heads // group):
                sel = 0 if selected is None else int(selected[cell][b][hk * group])
                total += decode_bytes(src_kind, d, int(n), sel) + (group - 1) * 2 * d * 2
                if reuse_current and kind == "reuse":
                    total += 4 * d
    return total
