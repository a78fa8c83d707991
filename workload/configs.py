"""The five synthetic workloads of the LoopKV decode path.

LoopKV: Loop-Aware KV Cache Compression for Serving Looped Transformers,
Abstract: the method serves a looped model (Ouro-1.4B) whose KV cache has one
cell per (loop, layer); each cell is 4-bit, 2-bit or a reuse of the final
loop's cell; contexts reach 16K tokens.  The pages print no model shape, so
the shapes below are an Ouro-1.4B-like stand-in: 4 loops x 24 layers, 16 MHA
heads of width 128, paged KV blocks of 16 tokens.
"""

from __future__ import annotations

from dataclasses import dataclass, replace


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    num_loops: int
    num_layers: int
    num_heads: int
    head_dim: int
    context: int                      # fixed context length of every sequence
    ctx_range: tuple | None           # (lo, hi) inclusive: per-sequence uniform lengths
    frac_q4: float                    # fraction of all cells stored 4-bit
    frac_reuse: float                 # fraction of all cells that reuse the final loop
    tau: float                        # low-plane threshold on the softmax weight
    paging: str                       # "identity" or "shuffled"
    pool_factor: float                # physical pool size / blocks needed (shuffled)
    seed: int
    temperature: float = 1.0          # multiplies q (flat -> peaky attention)
    all_bf16: bool = False            # every cell stored as bf16 (comparison run)
    block_size: int = 16
    outlier_channels: int = 4         # key channels per (cell, head) scaled up
    outlier_scale: float = 10.0
    q_std: float = 0.125              # q ~ N(0, 1) / 8, already carrying its scale
    sm_scale: float = 1.0
    num_kv_heads: int = 0             # KV heads (0: one per query head, MHA)

    @property
    def kv_heads(self) -> int:
        return self.num_kv_heads or self.num_heads

    @property
    def num_cells(self) -> int:
        return self.num_loops * self.num_layers

    @property
    def max_context(self) -> int:
        return self.ctx_range[1] if self.ctx_range else self.context

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    # correctness-only case
    "tiny": Workload(
        name="tiny", batch=1, num_loops=1, num_layers=2, num_heads=2, head_dim=64,
        context=256, ctx_range=None, frac_q4=1.0, frac_reuse=0.0, tau=0.02,
        paging="identity", pool_factor=1.0, seed=0),
    # one looped decode step of an Ouro-1.4B-like model
    "ouro_step": Workload(
        name="ouro_step", batch=8, num_loops=4, num_layers=24, num_heads=16, head_dim=128,
        context=2048, ctx_range=None, frac_q4=0.5, frac_reuse=0.2, tau=0.01,
        paging="identity", pool_factor=1.0, seed=1),
    # large batch, memory-lean plan, blocks shuffled in a 1.5x pool
    "throughput": Workload(
        name="throughput", batch=64, num_loops=4, num_layers=24, num_heads=16, head_dim=128,
        context=8192, ctx_range=None, frac_q4=0.3, frac_reuse=0.3, tau=0.01,
        paging="shuffled", pool_factor=1.5, seed=2),
    # ragged long contexts, 1K..16K tokens
    "long_context": Workload(
        name="long_context", batch=16, num_loops=4, num_layers=24, num_heads=16, head_dim=128,
        context=16384, ctx_range=(1024, 16384), frac_q4=0.4, frac_reuse=0.25, tau=0.005,
        paging="shuffled", pool_factor=1.0, seed=3),
    # threshold sweep: all cells 4-bit so tau acts everywhere
    "tau_sweep": Workload(
        name="tau_sweep", batch=32, num_loops=4, num_layers=24, num_heads=16, head_dim=128,
        context=4096, ctx_range=None, frac_q4=1.0, frac_reuse=0.0, tau=0.01,
        paging="identity", pool_factor=1.0, seed=4),
}

TAU_SWEEP = (0.0, 1e-3, 1e-2, 5e-2, float("inf"))
TEMPERATURE_SWEEP = (0.5, 1.0, 4.0)


def get_workload(name: str) -> Workload:
    try:
        return WORKLOADS[name]
    except KeyError:
        raise KeyError(f"unknown workload {name!r}; known: {sorted(WORKLOADS)}") from None
