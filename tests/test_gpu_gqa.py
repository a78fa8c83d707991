"""GPU parity of grouped-query decode (G query heads per KV head) against the
oracle's grouped form, through the C ABI: every head's output within
|gpu - oracle| <= 2e-3 + 1e-2 |oracle|, and the union of the heads'
low-plane selections, reported for every head of the group, exact except
where some head's weight lies within 1e-6 of tau."""

import math

import pytest
import torch

from loopkv_testlib import check_cell, mask_buffers, query_for
from workload import block_table_for, cell_kv
from workload.configs import Workload

pytestmark = pytest.mark.gpu

LENS = [0, 1, 31, 33, 100, 513, 1000, 2048]


def _workload(kind, d, lens, hq, hkv, seed):
    return Workload(name="gqa", batch=len(lens), num_loops=1, num_layers=1, num_heads=hq, num_kv_heads=hkv,
                    head_dim=d, context=max(lens), ctx_range=None, frac_q4=1.0 if kind == "q4" else 0.0,
                    frac_reuse=0.0, tau=0.01, paging="shuffled", pool_factor=1.2, seed=seed,
                    all_bf16=kind == "bf16")


def _store(kind, d, lens, hq, hkv, seed=41, splits=0):
    """One cell of KV heads hkv, every sequence appended to its own length."""
    from mixed_precision_kv_loopkv_b200 import KVCells, loopkv_quantize_append
    w = _workload(kind, d, lens, hq, hkv, seed)
    table, nblocks = block_table_for(w, [max(n, 1) for n in lens])
    kv = KVCells([kind], 1, 1, hq, d, nblocks, w.batch, table.shape[1], decode_splits=splits, num_kv_heads=hkv)
    k, v = cell_kv(w, 0, 0, device="cuda", n=max(max(lens), 1))
    table_d = torch.from_numpy(table).cuda()
    for b, n in enumerate(lens):
        if n == 0:
            continue
        starts = torch.full((w.batch,), -1, dtype=torch.int32, device="cuda")
        starts[b] = 0
        loopkv_quantize_append(kv, 0, 0, k[:, :n].contiguous(), v[:, :n].contiguous(), table_d, starts)
    lens_d = torch.tensor(lens, dtype=torch.int32, device="cuda")
    return w, kv, {0: (k, v)}, table_d, lens_d


def _decode(kv, q, table, lens, tau, max_seq_len=0):
    from mixed_precision_kv_loopkv_b200 import loopkv_decode_attention
    sm, sc = mask_buffers(kv, q.shape[0])
    out = loopkv_decode_attention(kv, 0, 0, q, table, lens, tau, 1.0, max_seq_len=max_seq_len,
                                  sel_mask=sm, sel_count=sc)
    torch.cuda.synchronize()
    return out, sm, sc


def _pairs(w):
    return [(b, h) for b in range(w.batch) for h in range(w.num_heads)]


@pytest.mark.parametrize("g", [2, 4, 8])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("tau", [0.0, 0.01, 0.05, math.inf])
def test_grouped_q4(g, d, tau):
    w, kv, data, table, lens = _store("q4", d, LENS, 2 * g, 2)
    for temp in (1.0, 6.0):
        q = query_for(w, 0, temperature=temp)
        out, sm, sc = _decode(kv, q, table, lens, tau)
        check_cell(kv, ["q4"], 0, data, q, table, lens, tau, 1.0, _pairs(w), out=out, sel_mask=sm, sel_count=sc)
        # the union is reported for every head of a group
        for hk in range(2):
            grp = sm[:, hk * g:(hk + 1) * g]
            assert torch.equal(grp, grp[:, :1].expand_as(grp))
        if 0 < tau < math.inf and temp > 1:
            assert int(sc.sum()) > 0


@pytest.mark.parametrize("kind", ["q2", "bf16"])
@pytest.mark.parametrize("g", [2, 8])
def test_grouped_other_kinds(kind, g):
    w, kv, data, table, lens = _store(kind, 128, LENS, 2 * g, 2)
    q = query_for(w, 0, temperature=4.0)
    out, sm, sc = _decode(kv, q, table, lens, 0.01)
    check_cell(kv, [kind], 0, data, q, table, lens, 0.01, 1.0, _pairs(w), out=out, sel_mask=sm, sel_count=sc)
    assert int(sc.sum()) == 0


@pytest.mark.parametrize("unit", [16, 32])
def test_grouped_selection_units(unit):
    from mixed_precision_kv_loopkv_b200 import LOOPKV_FLAG_SELECT_BLOCK, LOOPKV_FLAG_SELECT_GROUP
    w, kv, data, table, lens = _store("q4", 128, LENS, 8, 2, seed=43)
    kv.flags = LOOPKV_FLAG_SELECT_BLOCK if unit == 16 else LOOPKV_FLAG_SELECT_GROUP
    q = query_for(w, 0, temperature=4.0)
    out, sm, sc = _decode(kv, q, table, lens, 0.01)
    check_cell(kv, ["q4"], 0, data, q, table, lens, 0.01, 1.0, _pairs(w), out=out, sel_mask=sm, sel_count=sc,
               unit=unit)
    assert int(sc.sum()) > 0


@pytest.mark.parametrize("g,splits", [(2, 1), (2, 2), (2, 4), (2, 8), (4, 1), (4, 2), (4, 4), (8, 1), (8, 2)])
def test_grouped_explicit_splits(g, splits):
    """Every cluster shape of splits x heads up to 16 CTAs."""
    w, kv, data, table, lens = _store("q4", 128, [7, 255, 777, 3000], 2 * g, 2, seed=44, splits=splits)
    q = query_for(w, 0, temperature=4.0)
    out, sm, sc = _decode(kv, q, table, lens, 0.01)
    check_cell(kv, ["q4"], 0, data, q, table, lens, 0.01, 1.0, _pairs(w), out=out, sel_mask=sm, sel_count=sc)


def test_identical_queries_match_one_query_per_head():
    """G copies of one query per KV head give exactly the one-query result
    (same splits): the union of identical selections is that selection, and
    every head reads its KV head's cache."""
    from mixed_precision_kv_loopkv_b200 import KVCells, loopkv_decode_attention
    lens = [500, 1500, 64]
    w, kv, data, table, lens_d = _store("q4", 128, lens, 8, 2, seed=45, splits=2)
    q1 = query_for(w.with_(num_heads=2, num_kv_heads=0), 0, temperature=5.0)   # [B, 2, D]
    q = q1.repeat_interleave(4, dim=1).contiguous()                           # heads 4j..4j+3 = q1[:, j]
    out, sm, sc = _decode(kv, q, table, lens_d, 0.01)
    mha = KVCells(["q4"], 1, 1, 2, 128, kv.num_blocks, w.batch, kv.max_blocks_per_seq, decode_splits=2)
    mha.arenas[0].copy_(kv.arenas[0])
    mha.residuals[0].copy_(kv.residuals[0])
    sm1, sc1 = mask_buffers(mha, w.batch)
    out1 = loopkv_decode_attention(mha, 0, 0, q1, table, lens_d, 0.01, 1.0, sel_mask=sm1, sel_count=sc1)
    torch.cuda.synchronize()
    assert torch.equal(out, out1.repeat_interleave(4, dim=1))
    assert torch.equal(sm, sm1.repeat_interleave(4, dim=1))
    assert torch.equal(sc, sc1.repeat_interleave(4, dim=1))
    assert int(sc.sum()) > 0


def test_grouped_long_context_two_splits():
    """Eight heads per KV head leave two splits per cluster of 16 CTAs: a
    16K-token context is two chunks of 256 groups."""
    from mixed_precision_kv_loopkv_b200 import loopkv_decode_splits
    lens = [16384, 9000]
    w, kv, data, table, lens_d = _store("q4", 128, lens, 16, 2, seed=46)
    assert loopkv_decode_splits(kv, "q4", 2, 16384) == 2
    q = query_for(w, 0, temperature=6.0)
    out, sm, sc = _decode(kv, q, table, lens_d, 0.01)
    check_cell(kv, ["q4"], 0, data, q, table, lens_d, 0.01, 1.0, [(b, h) for b in range(2) for h in (0, 7, 8, 15)],
               out=out, sel_mask=sm, sel_count=sc)


def test_grouped_looped_step():
    """A captured looped decode step (PDL, CUDA graph, reuse cells included)
    with four query heads per KV head: appends run as their own launches."""
    from loopkv_testlib import step_parity
    w = Workload(name="gqa_step", batch=4, num_loops=2, num_layers=3, num_heads=8, num_kv_heads=2, head_dim=128,
                 context=0, ctx_range=(100, 900), frac_q4=0.5, frac_reuse=0.2, tau=0.01, paging="shuffled",
                 pool_factor=1.3, seed=47, temperature=4.0)
    rep = step_parity(w, nseq=4)
    assert len(rep) == 6


def test_grouped_maximum_context():
    """The largest context the ABI accepts (65536 tokens) with eight query
    heads per KV head: two splits of 1024 groups, one CTA's shared memory
    holding 128 KB of logits; sampled heads against the oracle."""
    lens = [65536, 777]
    w, kv, data, table, lens_d = _store("q4", 128, lens, 8, 1, seed=48)
    q = query_for(w, 0, temperature=6.0)
    out, sm, sc = _decode(kv, q, table, lens_d, 0.01, max_seq_len=65536)
    check_cell(kv, ["q4"], 0, data, q, table, lens_d, 0.01, 1.0, [(0, 0), (0, 5), (1, 3)],
               out=out, sel_mask=sm, sel_count=sc)
    assert int(sc[0, 0]) > 0
