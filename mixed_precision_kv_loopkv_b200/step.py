"""One looped decode step over every (loop, layer) cell.

LoopKV: Loop-Aware KV Cache Compression for Serving Looped Transformers
(Abstract): a looped transformer applies its shared block num_loops times per
token, and each application (loop) attends over its own KV cell per layer,
unless the plan lets it reuse the final loop's cell.  Within one decode step
the cells run in (loop, layer) order.  For the token being decoded at
position n:
  * a stored cell first appends the token's K/V at position n, then attends
    over n + 1 tokens;
  * a reuse cell of loop l < L-1 attends over the final loop's first n
    tokens (the final loop has not produced this token's K/V yet) plus the
    current token exactly as its own loop l computed it: the model projects
    K/V in every loop, a reuse cell just stores none of them, so its own row
    is passed to the kernel as one more, exact, token.
The model's projections and MLPs are not part of this path; each cell's query
and new K/V are given tensors.
"""

from __future__ import annotations

import torch

from .loopkv import (LOOPKV_CELL_REUSE, KVCells, loopkv_append_decode_attention, loopkv_decode_attention,
                     loopkv_quantize_append)


def prefill(kv: KVCells, loop: int, layer: int, k, v, block_table, lens, err_flag=None, stream=None):
    """Append the first lens[b] tokens of k, v (bf16 [B, n_max, Hkv, D]) to the
    cell, sequences of different lengths included: one append per distinct
    length, sequences already complete skipped (negative start position)."""
    lens = [int(x) for x in (lens.tolist() if hasattr(lens, "tolist") else lens)]
    prev = 0
    for cut in sorted(set(lens)):
        if cut <= prev:
            continue
        starts = [prev if n >= cut else -1 for n in lens]
        pos = torch.tensor(starts, dtype=torch.int32, device=k.device)
        loopkv_quantize_append(kv, loop, layer, k[:, prev:cut].contiguous(), v[:, prev:cut].contiguous(),
                               block_table, pos, err_flag=err_flag, stream=stream)
        prev = cut


class LoopedDecodeStep:
    """Sequences the per-cell kernels of one decode step (graph-capturable).

    pos    : device int32[B], current length n of every sequence (the new
             token's position); ``advance()`` moves it by one on the device.
    q      : per cell, bf16[B, H, D]  (H query heads)
    k_new, v_new : per cell, bf16[B, 1, Hkv, D]: the token's K/V as the cell's
             loop computed it (appended by stored cells, attended exactly by
             reuse cells; a reuse cell without an entry attends over the
             stored tokens only)
    out    : per cell, bf16[B, H, D] (written)
    sel_count : optional per cell int32[B, H] (written)
    fused  : a stored cell runs append and attention as one launch
             (loopkv_append_decode_attention); False: two launches.  Grouped
             queries (Hkv < H) always take two launches
    """

    def __init__(self, kv: KVCells, block_table, pos, q, k_new, v_new, out, tau: float,
                 sm_scale: float, max_seq_len: int, sel_count=None, err_flag=None, cells=None,
                 fused: bool = True):
        self.kv = kv
        self.fused = fused and kv.num_kv_heads == kv.num_heads
        self.cells = list(range(len(kv.plan_codes))) if cells is None else sorted(cells)
        self.block_table = block_table
        self.pos = pos
        self.pos_next = pos + 1
        self.q, self.out = q, out
        self.k_new, self.v_new = dict(k_new), dict(v_new)
        self.tau, self.sm_scale, self.max_seq_len = tau, sm_scale, max_seq_len
        self.sel_count = sel_count
        self.err_flag = err_flag

    def launches_per_step(self) -> int:
        stored = sum(1 for c in self.cells if self.kv.plan_codes[c] != LOOPKV_CELL_REUSE)
        return len(self.cells) + (0 if self.fused else stored)

    def run(self, stream=None):
        """Enqueue the step.  Re-running it at the same positions rewrites
        the same bytes, so a warm-up run before capture leaves the cache
        state unchanged."""
        kv = self.kv
        for cell in self.cells:
            kind = kv.plan_codes[cell]
            loop, layer = divmod(cell, kv.num_layers)
            sel = None if self.sel_count is None else self.sel_count[cell]
            if kind != LOOPKV_CELL_REUSE and self.fused:
                loopkv_append_decode_attention(kv, loop, layer, self.k_new[cell], self.v_new[cell], self.q[cell],
                                               self.block_table, self.pos, self.tau, self.sm_scale,
                                               out=self.out[cell], max_seq_len=self.max_seq_len,
                                               sel_count=sel, err_flag=self.err_flag, stream=stream)
                continue
            if kind != LOOPKV_CELL_REUSE:
                loopkv_quantize_append(kv, loop, layer, self.k_new[cell], self.v_new[cell],
                                       self.block_table, self.pos, err_flag=self.err_flag,
                                       stream=stream)
                lens = self.pos_next
            else:
                lens = self.pos
            cur_k = cur_v = None
            if kind == LOOPKV_CELL_REUSE and self.k_new.get(cell) is not None:
                cur_k, cur_v = self.k_new[cell], self.v_new[cell]
            loopkv_decode_attention(kv, loop, layer, self.q[cell], self.block_table, lens, self.tau,
                                    self.sm_scale, out=self.out[cell], max_seq_len=self.max_seq_len,
                                    sel_count=None if self.sel_count is None else self.sel_count[cell],
                                    err_flag=self.err_flag, stream=stream, k_cur=cur_k, v_cur=cur_v)

    def advance(self):
        self.pos.add_(1)
        self.pos_next.add_(1)

    def capture(self, steps_per_graph: int = 1) -> torch.cuda.CUDAGraph:
        """Capture ``steps_per_graph`` consecutive steps (run + advance)."""
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(steps_per_graph):
                self.run()
                self.advance()
        return g
