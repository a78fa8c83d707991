"""GPU parity of loopkv_decode_attention against the CPU oracle (through the
C ABI): outputs within |gpu - oracle| <= 2e-3 + 1e-2 |oracle|, the low-plane
selection set exact except where the oracle's weight lies within 1e-6 of tau,
and selection counts consistent with the masks."""

import math

import numpy as np
import pytest
import torch

from loopkv_testlib import (build_store, check_cell, mask_buffers, query_for, sample_pairs, step_parity)
from workload import block_table_for, cell_kv, get_workload
from workload.configs import Workload

pytestmark = pytest.mark.gpu


def _decode(kv, cell, q, table, lens, tau, sm_scale=1.0, max_seq_len=0, masks=True, err=None):
    from mixed_precision_kv_loopkv_b200 import loopkv_decode_attention
    loop, layer = divmod(cell, kv.num_layers)
    sel_mask, sel_count = mask_buffers(kv, q.shape[0]) if masks else (None, None)
    out = loopkv_decode_attention(kv, loop, layer, q, table, lens, tau, sm_scale, max_seq_len=max_seq_len,
                                  sel_mask=sel_mask, sel_count=sel_count, err_flag=err)
    torch.cuda.synchronize()
    return out, sel_mask, sel_count


def test_tiny_workload_all_cells():
    w = get_workload("tiny")
    kv, plan, table, lens, data = build_store(w)
    pairs = [(b, h) for b in range(w.batch) for h in range(w.num_heads)]
    for cell in range(w.num_cells):
        q = query_for(w, cell)
        out, sm, sc = _decode(kv, cell, q, table, lens, w.tau)
        check_cell(kv, plan, cell, data, q, table, lens, w.tau, w.sm_scale, pairs, out=out,
                   sel_mask=sm, sel_count=sc)


def _custom(kind, d, lens, heads=2, seed=11, paging="shuffled"):
    return Workload(name="custom", batch=len(lens), num_loops=1, num_layers=1, num_heads=heads,
                    head_dim=d, context=max(lens), ctx_range=None, frac_q4=1.0, frac_reuse=0.0,
                    tau=0.01, paging=paging, pool_factor=1.2, seed=seed)


def _store_ragged(kind, d, lens, heads=2, seed=11, splits=0):
    from mixed_precision_kv_loopkv_b200 import KVCells, loopkv_quantize_append
    w = _custom(kind, d, lens, heads, seed)
    table, nblocks = block_table_for(w, [max(n, 1) for n in lens])
    kv = KVCells([kind], 1, 1, heads, d, nblocks, w.batch, table.shape[1], decode_splits=splits)
    k, v = cell_kv(w, 0, 0, device="cuda", n=max(max(lens), 1))
    table_d = torch.from_numpy(table).cuda()
    # append each sequence's own length: full prefix, then skip finished ones
    have = [0] * len(lens)
    for cut in sorted(set(lens)):
        T = cut - min(h for h, n in zip(have, lens) if n >= cut)
        starts = []
        kr, vr = torch.zeros_like(k[:, :T]), torch.zeros_like(v[:, :T])
        for b, n in enumerate(lens):
            if n >= cut and cut - have[b] == T and T > 0:
                kr[b], vr[b] = k[b, have[b]:cut], v[b, have[b]:cut]
                starts.append(have[b])
                have[b] = cut
            else:
                starts.append(-1)
        if T > 0:
            loopkv_quantize_append(kv, 0, 0, kr.contiguous(), vr.contiguous(), table_d,
                                   torch.tensor(starts, dtype=torch.int32, device="cuda"))
    assert have == lens
    lens_d = torch.tensor(lens, dtype=torch.int32, device="cuda")
    return w, kv, {0: (k, v)}, table_d, lens_d


RAGGED = [0, 1, 31, 32, 33, 100, 513, 1000]


@pytest.mark.parametrize("kind", ["q4", "q2", "bf16"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("tau", [0.0, 0.01, 0.05, math.inf])
def test_ragged_lengths(kind, d, tau):
    w, kv, data, table, lens = _store_ragged(kind, d, RAGGED, heads=2)
    pairs = [(b, h) for b in range(w.batch) for h in range(2)]
    for temp in (1.0, 6.0):
        q = query_for(w, 0, temperature=temp)
        out, sm, sc = _decode(kv, 0, q, table, lens, tau)
        check_cell(kv, [kind], 0, data, q, table, lens, tau, 1.0, pairs, out=out, sel_mask=sm, sel_count=sc)
        if kind == "q4" and 0 < tau < math.inf and temp > 1:
            assert int(sc.sum()) > 0
        if kind == "q4" and tau == 0.0:
            assert int(sc[2, 0]) == 31


@pytest.mark.parametrize("kind", ["q4", "q2", "bf16"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("splits", [1, 2, 4, 8])
def test_explicit_splits(kind, d, splits):
    """Every split count of a cluster (a 4-bit cell's two-barrier combine, and
    the single-barrier combine of 2-bit and bf16 cells, where each owner
    rescales every split's channel sums), D 64 and 128."""
    w, kv, data, table, lens = _store_ragged(kind, d, [7, 255, 777, 2048], heads=3, seed=3,
                                             splits=splits)
    q = query_for(w, 0, temperature=4.0)
    out, sm, sc = _decode(kv, 0, q, table, lens, 0.01)
    check_cell(kv, [kind], 0, data, q, table, lens, 0.01, 1.0,
               [(b, h) for b in range(4) for h in range(3)], out=out, sel_mask=sm, sel_count=sc)


def test_reuse_equals_source_with_own_query():
    from mixed_precision_kv_loopkv_b200 import loopkv_decode_attention
    w = get_workload("tiny").with_(num_loops=2, num_layers=2, frac_q4=0.5, frac_reuse=0.25, seed=7)
    kv, plan, table, lens, data = build_store(w)
    reuse = [c for c, k in enumerate(plan) if k == "reuse"]
    assert reuse
    for cell in reuse:
        src = kv.source_cell(cell)
        q = query_for(w, cell)
        out_r, sm_r, sc_r = _decode(kv, cell, q, table, lens, w.tau)
        loop, layer = divmod(src, w.num_layers)
        out_s = loopkv_decode_attention(kv, loop, layer, q, table, lens, w.tau)
        torch.cuda.synchronize()
        assert torch.equal(out_r, out_s)
        check_cell(kv, plan, cell, data, q, table, lens, w.tau, 1.0,
                   [(0, h) for h in range(w.num_heads)], out=out_r, sel_mask=sm_r, sel_count=sc_r)


@pytest.mark.parametrize("kind", ["q4", "q2", "bf16"])
def test_bad_block_in_one_split_zeroes_the_whole_row(kind):
    """A bad block id in one split of four: every split's owner learns of it
    through the exchanged tables (both combines), the sequence-head's whole
    output row is zero and the error bit is set; the other sequence is
    unaffected."""
    from mixed_precision_kv_loopkv_b200 import LOOPKV_DEVERR_BLOCK_ID
    w, kv, data, table, lens = _store_ragged(kind, 128, [2048, 2048], heads=2, splits=4)
    bad = table.clone()
    bad[1, 70] = kv.num_blocks + 3          # block 70 of 128: the third split's chunk
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    q = query_for(w, 0)
    out, _, _ = _decode(kv, 0, q, bad, lens, 0.01, err=err)
    assert int(err) & LOOPKV_DEVERR_BLOCK_ID
    assert not out[1].any()
    check_cell(kv, [kind], 0, data, q, table, lens, 0.01, 1.0, [(0, 0), (0, 1)], out=out)


def test_bad_block_id_and_length_are_flagged():
    from mixed_precision_kv_loopkv_b200 import LOOPKV_DEVERR_BLOCK_ID, LOOPKV_DEVERR_SEQ_LEN
    w, kv, data, table, lens = _store_ragged("q4", 64, [64, 64], heads=1)
    bad = table.clone()
    bad[1, 1] = kv.num_blocks + 5
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    q = query_for(w, 0)
    out, _, _ = _decode(kv, 0, q, bad, lens, 0.01, err=err)
    assert int(err) & LOOPKV_DEVERR_BLOCK_ID
    assert not out[1].any() and out[0].abs().sum() > 0
    err.zero_()
    long = torch.tensor([64, 65], dtype=torch.int32, device="cuda")
    out, _, _ = _decode(kv, 0, q, table, long, 0.01, max_seq_len=64, err=err)
    assert int(err) & LOOPKV_DEVERR_SEQ_LEN
    assert not out[1].any()


def test_pdl_flag_matches_plain_launch():
    from mixed_precision_kv_loopkv_b200 import LOOPKV_FLAG_PDL
    w, kv, data, table, lens = _store_ragged("q4", 128, [300, 1234, 2047], heads=4)
    q = query_for(w, 0, temperature=3.0)
    a, _, _ = _decode(kv, 0, q, table, lens, 0.01)
    kv.flags = LOOPKV_FLAG_PDL
    b, _, _ = _decode(kv, 0, q, table, lens, 0.01)
    assert torch.equal(a, b)


@pytest.mark.parametrize("fused", [True, False])
def test_ouro_step_captured_with_pdl(fused):
    rep = step_parity(get_workload("ouro_step"), nseq=2, fused=fused)
    assert len(rep) == 96


@pytest.mark.parametrize("name,cells", [("throughput", None), ("long_context", None)])
def test_full_size_sampled(name, cells):
    """Full-size shapes of the throughput (64 x 8192, blocks shuffled in a
    1.5x pool) and long-context (16 sequences of 1K..16K) workloads on a
    subset of cells: every kind present, reuse included."""
    w = get_workload(name)
    from workload import make_plan
    plan = make_plan(w)
    L, N = w.num_loops, w.num_layers
    pick = []
    for kind in ("q4", "q2", "reuse"):
        pick += [c for c, k in enumerate(plan) if k == kind][:2]
    kv, plan, table, lens, data = build_store(w, cells=pick)
    pairs = sample_pairs(w, 3, seed=1)
    for cell in pick:
        q = query_for(w, cell)
        out, sm, sc = _decode(kv, cell, q, table, lens, w.tau, max_seq_len=int(lens.max()))
        check_cell(kv, plan, cell, data, q, table, lens, w.tau, 1.0, pairs, out=out, sel_mask=sm, sel_count=sc)
    del kv, data
    torch.cuda.empty_cache()


@pytest.mark.parametrize("temperature", [0.5, 1.0, 4.0])
def test_tau_sweep_sampled(temperature):
    w = get_workload("tau_sweep")
    kv, plan, table, lens, data = build_store(w, cells=[0, 50])
    pairs = sample_pairs(w, 2, seed=2)
    for cell in (0, 50):
        q = query_for(w, cell, temperature=temperature)
        for tau in (0.0, 1e-3, 1e-2, 5e-2, math.inf):
            out, sm, sc = _decode(kv, cell, q, table, lens, tau)
            check_cell(kv, plan, cell, data, q, table, lens, tau, 1.0, pairs, out=out, sel_mask=sm,
                       sel_count=sc)


def test_bf16_cells_full_shape_sampled():
    w = get_workload("tau_sweep").with_(all_bf16=True, batch=8)
    kv, plan, table, lens, data = build_store(w, cells=[3])
    q = query_for(w, 3)
    out, sm, sc = _decode(kv, 3, q, table, lens, 0.01)
    check_cell(kv, plan, 3, data, q, table, lens, 0.01, 1.0, sample_pairs(w, 2), out=out, sel_mask=sm,
               sel_count=sc)


@pytest.mark.parametrize("unit", [16, 32])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("tau", [0.01, 0.05])
def test_coarser_selection_units(unit, d, tau):
    """Low-plane selection by 16-token block or 32-token group (the
    granularity variant): any token of the unit at or above tau upgrades the
    whole unit."""
    from mixed_precision_kv_loopkv_b200 import LOOPKV_FLAG_SELECT_BLOCK, LOOPKV_FLAG_SELECT_GROUP
    w, kv, data, table, lens = _store_ragged("q4", d, RAGGED, heads=2, seed=13)
    kv.flags = LOOPKV_FLAG_SELECT_BLOCK if unit == 16 else LOOPKV_FLAG_SELECT_GROUP
    pairs = [(b, h) for b in range(w.batch) for h in range(2)]
    q = query_for(w, 0, temperature=4.0)
    out, sm, sc = _decode(kv, 0, q, table, lens, tau)
    check_cell(kv, ["q4"], 0, data, q, table, lens, tau, 1.0, pairs, out=out, sel_mask=sm, sel_count=sc,
               unit=unit)
    assert int(sc.sum()) > 0
    kv.flags = 0
    out1, sm1, sc1 = _decode(kv, 0, q, table, lens, tau)
    assert int(sc.sum()) >= int(sc1.sum())


@pytest.mark.parametrize("kind", ["q4", "q2"])
def test_maximum_context(kind):
    """The largest context the ABI accepts (65536 tokens after the step:
    2048 groups, 8 splits of 256 groups, the most the split rule produces),
    with a ragged partner sequence, on the fused decode step."""
    from mixed_precision_kv_loopkv_b200 import (KVCells, loopkv_append_decode_attention, loopkv_decode_splits,
                                                prefill)
    lens = [65535, 40000]
    w = _custom(kind, 128, [n + 1 for n in lens], heads=2, seed=17)
    table, nblocks = block_table_for(w, [n + 1 for n in lens])
    kv = KVCells([kind], 1, 1, 2, 128, nblocks, 2, table.shape[1])
    k, v = cell_kv(w, 0, 0, device="cuda", n=65536)
    table_d = torch.from_numpy(table).cuda()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    prefill(kv, 0, 0, k, v, table_d, lens, err_flag=err)
    assert loopkv_decode_splits(kv, kind, 2, 65536) == 8
    kn = torch.stack([k[0, 65535], k[1, 40000]]).unsqueeze(1).contiguous()
    vn = torch.stack([v[0, 65535], v[1, 40000]]).unsqueeze(1).contiguous()
    q = query_for(w, 0, temperature=4.0)
    sm, sc = mask_buffers(kv, 2)
    start = torch.tensor(lens, dtype=torch.int32, device="cuda")
    out = loopkv_append_decode_attention(kv, 0, 0, kn, vn, q, table_d, start, 0.01, max_seq_len=65536,
                                         sel_mask=sm, sel_count=sc, err_flag=err)
    torch.cuda.synchronize()
    assert int(err) == 0
    check_cell(kv, [kind], 0, {0: (k, v)}, q, table_d, start + 1, 0.01, 1.0, [(0, 0), (0, 1), (1, 0)],
               out=out, sel_mask=sm, sel_count=sc)


@pytest.mark.parametrize("B", [48, 64, 70])
def test_ragged_batch_order(B):
    """Batches are dispatched longest first (a rank of each sequence by
    length, ties by index, over up to 64 sequences: both halves of a warp's
    ranking for 33..64; beyond 64 the identity order): every sequence of a
    ragged batch with repeated lengths is decoded exactly once, into its own
    output row."""
    from loopkv_testlib import seeded_bf16, store_tensors
    rng = np.random.default_rng(B)
    lens = rng.integers(1, 200, size=B)
    lens[::7] = 96                                # ties
    k = seeded_bf16((B, int(lens.max()), 2, 64), 60)
    v = seeded_bf16((B, int(lens.max()), 2, 64), 61)
    kv, table, lens_d = store_tensors("q4", k, v, lens.tolist())
    q = seeded_bf16((B, 2, 64), 62, 0.5)
    from mixed_precision_kv_loopkv_b200 import loopkv_decode_attention
    sm, sc = mask_buffers(kv, B)
    out = loopkv_decode_attention(kv, 0, 0, q, table, lens_d, 0.01, 1.0, sel_mask=sm, sel_count=sc)
    torch.cuda.synchronize()
    check_cell(kv, ["q4"], 0, {0: (k, v)}, q, table, lens_d, 0.01, 1.0,
               [(b, h) for b in range(B) for h in range(2)], out=out, sel_mask=sm, sel_count=sc)
