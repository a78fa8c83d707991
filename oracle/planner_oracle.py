"""Brute-force oracle of the cell planner (TEST INFRASTRUCTURE ONLY).

LoopKV: Loop-Aware KV Cache Compression for Serving Looped Transformers
(Abstract): every (loop, layer) cell is stored 4-bit, 2-bit or reuses the
final loop's cell of its layer; a planner picks the choices that minimise
bytes read per decoded token under budgets on predicted damage (additive over
cells) and storage.  This module enumerates every admissible plan of a small
model and keeps the best one under the library's reading of that problem:
  * damage = sum of damage[loop][layer][choice] (choice 0: 4-bit, 1: 2-bit,
    2: reuse), at most the damage budget;
  * storage in 32-byte units per token-head: 4-bit 5, 2-bit 3, reuse 0, at
    most the storage budget;
  * reads per token-head: 4-bit q4_read_bytes, 2-bit 96, a reuse cell the
    reads of the final loop's cell of its layer;
  * the final loop never reuses;
  * minimal reads, then minimal damage, then minimal storage.
"""

from __future__ import annotations

import itertools

STORAGE = (5, 3, 0)


def plan_cost(damage, plan, q4_read_bytes: int):
    """(reads, damage, storage) of a plan given as choices[loop][layer]."""
    L, N = len(plan), len(plan[0])
    reads = dmg = sto = 0
    for l in range(L):
        for j in range(N):
            c = plan[l][j]
            dmg += damage[l][j][c]
            sto += STORAGE[c]
            src = plan[L - 1][j] if c == 2 else c
            reads += q4_read_bytes if src == 0 else 96
    return reads, dmg, sto


def plan_brute_force(damage, damage_budget: int, storage_budget: int, q4_read_bytes: int):
    """Best (reads, damage, storage) and a plan achieving it, or None."""
    L, N = len(damage), len(damage[0])
    choices = [(0, 1, 2) if l < L - 1 else (0, 1) for l in range(L) for _ in range(N)]
    best = None
    for flat in itertools.product(*choices):
        plan = [list(flat[l * N:(l + 1) * N]) for l in range(L)]
        r, d, s = plan_cost(damage, plan, q4_read_bytes)
        if d > damage_budget or s > storage_budget:
            continue
        if best is None or (r, d, s) < best[0]:
            best = ((r, d, s), plan)
    return best
