"""Seeded input generators (plans, lengths, block tables, K/V/q tensors).

Nothing here quantises or attends: these functions only draw the synthetic
inputs that both the CUDA path and the CPU oracle consume.

Recipe (one Ouro-1.4B-like stand-in, since the pages give no tensors):
  * K, V ~ N(0, 1) in fp32, cast to bf16; per (cell, head), ``outlier_channels``
    seeded key channels are multiplied by ``outlier_scale`` before the cast.
  * q ~ N(0, 1) * q_std * temperature, cast to bf16.
  * plan: ``round(frac_reuse * cells)`` reuse cells drawn uniformly among the
    non-final loops, then ``round(frac_q4 * cells)`` 4-bit cells among the
    rest; the remaining cells are 2-bit.
  * lengths: fixed, or uniform integers in ``ctx_range`` per sequence.
  * block tables: identity (sequence b owns a contiguous run of blocks) or a
    random permutation of a pool ``pool_factor`` times the blocks needed.
"""

from __future__ import annotations

import math

import numpy as np
import torch

from .configs import Workload

CELL_KINDS = ("q4", "q2", "reuse", "bf16")

_TAG_K, _TAG_V, _TAG_Q, _TAG_NEWK, _TAG_NEWV, _TAG_OUTLIER = 1, 2, 3, 4, 5, 6


def _seed(*parts: int) -> int:
    state = np.random.SeedSequence([int(p) & 0xFFFFFFFF for p in parts]).generate_state(2, np.uint64)
    return int(state[0] % np.uint64(2**62))


def _gen(device, *parts: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(_seed(*parts))
    return g


def make_plan(w: Workload) -> list:
    """Cell kinds in cell order (cell = loop * num_layers + layer)."""
    n = w.num_cells
    if w.all_bf16:
        return ["bf16"] * n
    rng = np.random.default_rng([w.seed, 0x504C414E])
    nonfinal = np.arange((w.num_loops - 1) * w.num_layers)
    n_reuse = int(round(w.frac_reuse * n))
    if n_reuse > nonfinal.size:
        raise ValueError("more reuse cells than non-final cells")
    reuse = rng.choice(nonfinal, size=n_reuse, replace=False) if n_reuse else np.array([], int)
    rest = np.setdiff1d(np.arange(n), reuse)
    n_q4 = min(int(round(w.frac_q4 * n)), rest.size)
    q4 = rng.choice(rest, size=n_q4, replace=False) if n_q4 else np.array([], int)
    plan = ["q2"] * n
    for c in q4:
        plan[int(c)] = "q4"
    for c in reuse:
        plan[int(c)] = "reuse"
    return plan


def seq_lens_for(w: Workload) -> np.ndarray:
    if w.ctx_range is None:
        return np.full(w.batch, w.context, dtype=np.int32)
    lo, hi = w.ctx_range
    rng = np.random.default_rng([w.seed, 0x4C454E53])
    return rng.integers(lo, hi + 1, size=w.batch, dtype=np.int64).astype(np.int32)


def block_table_for(w: Workload, capacity_tokens) -> tuple:
    """Return (block_table int32[B, max_blocks], num_blocks).

    ``capacity_tokens`` (int or per-sequence array) is how many token slots
    each sequence owns; unused table entries are -1.
    """
    cap = np.broadcast_to(np.asarray(capacity_tokens, dtype=np.int64), (w.batch,))
    bs = w.block_size
    nblk = (cap + bs - 1) // bs
    max_blocks = int(nblk.max()) if w.batch else 0
    table = np.full((w.batch, max_blocks), -1, dtype=np.int32)
    if w.paging == "identity":
        for b in range(w.batch):
            table[b, : nblk[b]] = b * max_blocks + np.arange(nblk[b])
        return table, w.batch * max_blocks
    if w.paging != "shuffled":
        raise ValueError(w.paging)
    total = int(nblk.sum())
    pool = int(math.ceil(w.pool_factor * total))
    rng = np.random.default_rng([w.seed, 0x424C4B53])
    ids = rng.permutation(pool)[:total].astype(np.int32)
    off = 0
    for b in range(w.batch):
        table[b, : nblk[b]] = ids[off: off + nblk[b]]
        off += nblk[b]
    return table, pool


def _outlier_scale(w: Workload, loop: int, layer: int) -> torch.Tensor:
    rng = np.random.default_rng([w.seed, loop, layer, _TAG_OUTLIER])
    scale = np.ones((w.kv_heads, w.head_dim), dtype=np.float32)
    for h in range(w.kv_heads):
        ch = rng.choice(w.head_dim, size=min(w.outlier_channels, w.head_dim), replace=False)
        scale[h, ch] = w.outlier_scale
    return torch.from_numpy(scale)


def cell_kv(w: Workload, loop: int, layer: int, device="cpu", n: int | None = None):
    """K, V bf16[B, n, Hkv, D] of one stored cell (n defaults to max_context)."""
    n = w.max_context if n is None else n
    shape = (w.batch, n, w.kv_heads, w.head_dim)
    k = torch.randn(shape, generator=_gen(device, w.seed, loop, layer, _TAG_K), device=device)
    k.mul_(_outlier_scale(w, loop, layer).to(device))
    v = torch.randn(shape, generator=_gen(device, w.seed, loop, layer, _TAG_V), device=device)
    return k.to(torch.bfloat16), v.to(torch.bfloat16)


def cell_new_token(w: Workload, loop: int, layer: int, device="cpu", step: int = 0):
    """K, V bf16[B, 1, Hkv, D] of the token appended at decode step ``step``."""
    shape = (w.batch, 1, w.kv_heads, w.head_dim)
    k = torch.randn(shape, generator=_gen(device, w.seed, loop, layer, _TAG_NEWK, step), device=device)
    k.mul_(_outlier_scale(w, loop, layer).to(device))
    v = torch.randn(shape, generator=_gen(device, w.seed, loop, layer, _TAG_NEWV, step), device=device)
    return k.to(torch.bfloat16), v.to(torch.bfloat16)


def cell_query(w: Workload, loop: int, layer: int, device="cpu", temperature: float | None = None):
    """q bf16[B, H, D] of one cell."""
    t = w.temperature if temperature is None else temperature
    shape = (w.batch, w.num_heads, w.head_dim)
    q = torch.randn(shape, generator=_gen(device, w.seed, loop, layer, _TAG_Q), device=device)
    return (q * (w.q_std * t)).to(torch.bfloat16)
