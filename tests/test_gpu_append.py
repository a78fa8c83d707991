"""GPU parity of loopkv_quantize_append: packed bytes bit-exact against the
oracle's own record writer, on seeded ragged inputs (through the C ABI)."""

import numpy as np
import pytest
import torch

import oracle as O
from workload import block_table_for, cell_kv
from workload.configs import Workload

pytestmark = pytest.mark.gpu


def _small(d, lens, paging="shuffled", seed=5, heads=3):
    return Workload(name="append_test", batch=len(lens), num_loops=1, num_layers=1, num_heads=heads,
                    head_dim=d, context=max(lens), ctx_range=None, frac_q4=1.0, frac_reuse=0.0,
                    tau=0.01, paging=paging, pool_factor=1.3, seed=seed)


def _ragged_append(kv, k, v, lens, table_d, rounds):
    """Append so that sequence b ends with lens[b] tokens, in several calls
    whose start positions differ per sequence (negative = skipped): at every
    cut, sequences that still lack tokens take a common chunk T."""
    from mixed_precision_kv_loopkv_b200 import loopkv_quantize_append
    B = k.shape[0]
    have = [0] * B
    for cut in rounds:
        while True:
            takes = [min(cut, lens[b]) - have[b] for b in range(B)]
            pos = [t for t in takes if t > 0]
            if not pos:
                break
            T = min(pos)
            starts, kr, vr = [], torch.zeros_like(k[:, :T]), torch.zeros_like(v[:, :T])
            for b in range(B):
                if takes[b] > 0:
                    starts.append(have[b])
                    kr[b] = k[b, have[b]: have[b] + T]
                    vr[b] = v[b, have[b]: have[b] + T]
                    have[b] += T
                else:
                    starts.append(-1)
            st = torch.tensor(starts, dtype=torch.int32, device=k.device)
            loopkv_quantize_append(kv, 0, 0, kr.contiguous(), vr.contiguous(), table_d, st)
    return have


def _check_records(kv, kind, k, v, lens, table):
    arena = kv.arena_view(0).cpu().numpy()
    res = kv.residuals[0]
    res_h = None if res is None else res.view(torch.int16).cpu().numpy()
    for b, n in enumerate(lens):
        for h in range(kv.num_heads):
            kk = k[b, :n, h].float().cpu().numpy()
            vv = v[b, :n, h].float().cpu().numpy()
            want, resid = O.sequence_records(kind, kk, vv)
            got = arena[table[b, : want.shape[0]], h]
            if not np.array_equal(got, want):
                blk, byte = np.argwhere(got != want)[0]
                raise AssertionError(f"{kind} b={b} h={h} n={n}: block {blk} byte {byte} "
                                     f"gpu {got[blk, byte]} oracle {want[blk, byte]}")
            if resid is not None:
                for p in range(32 * (n // 32), n):
                    row = res_h[b, h, p % 32]
                    exp = k[b, p, h].view(torch.int16).cpu().numpy()
                    assert np.array_equal(row, exp), (kind, b, h, p)


@pytest.mark.parametrize("kind", ["q4", "q2", "bf16"])
@pytest.mark.parametrize("d", [64, 128])
def test_append_bytes_bit_exact(kind, d):
    from mixed_precision_kv_loopkv_b200 import KVCells
    lens = [70, 75, 87, 32, 1]
    w = _small(d, lens)
    table, nblocks = block_table_for(w, lens)
    kv = KVCells([kind], 1, 1, w.num_heads, d, nblocks, w.batch, table.shape[1])
    k, v = cell_kv(w, 0, 0, device="cuda")
    table_d = torch.from_numpy(table).cuda()
    got = _ragged_append(kv, k, v, lens, table_d, rounds=[1, 33, 70, 76, 100])
    assert got == lens
    torch.cuda.synchronize()
    _check_records(kv, kind, k, v, lens, table)


@pytest.mark.parametrize("kind", ["q4", "q2", "bf16"])
def test_incremental_append_equals_bulk(kind):
    from mixed_precision_kv_loopkv_b200 import KVCells, loopkv_quantize_append
    lens = [97, 97]
    w = _small(128, lens, paging="identity", seed=9, heads=2)
    table, nblocks = block_table_for(w, lens)
    table_d = torch.from_numpy(table).cuda()
    k, v = cell_kv(w, 0, 0, device="cuda")
    bulk = KVCells([kind], 1, 1, 2, 128, nblocks, 2, table.shape[1])
    loopkv_quantize_append(bulk, 0, 0, k, v, table_d, torch.zeros(2, dtype=torch.int32, device="cuda"))
    inc = KVCells([kind], 1, 1, 2, 128, nblocks, 2, table.shape[1])
    for t in range(97):
        pos = torch.full((2,), t, dtype=torch.int32, device="cuda")
        loopkv_quantize_append(inc, 0, 0, k[:, t: t + 1].contiguous(), v[:, t: t + 1].contiguous(),
                               table_d, pos)
    torch.cuda.synchronize()
    assert torch.equal(bulk.arenas[0], inc.arenas[0])
    if bulk.residuals[0] is not None:
        live = slice(0, 97 % 32)
        assert torch.equal(bulk.residuals[0][:, :, live], inc.residuals[0][:, :, live])
    _check_records(inc, kind, k, v, lens, table)


def test_append_flags_bad_block_and_overflow():
    from mixed_precision_kv_loopkv_b200 import (LOOPKV_DEVERR_BLOCK_ID, LOOPKV_DEVERR_SEQ_LEN, KVCells,
                                                loopkv_quantize_append)
    kv = KVCells(["q4"], 1, 1, 2, 64, 4, 2, 2)
    table = torch.tensor([[0, 1], [2, 99]], dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    k = torch.randn(2, 20, 2, 64, device="cuda").to(torch.bfloat16)
    loopkv_quantize_append(kv, 0, 0, k, k, table, torch.zeros(2, dtype=torch.int32, device="cuda"),
                           err_flag=err)
    assert int(err) & LOOPKV_DEVERR_BLOCK_ID
    err.zero_()
    loopkv_quantize_append(kv, 0, 0, k, k, table, torch.tensor([20, 0], dtype=torch.int32, device="cuda"),
                           err_flag=err)
    assert int(err) & LOOPKV_DEVERR_SEQ_LEN


def test_large_value_scales_need_no_flag():
    """Value scales have no limit: a 32-channel range of 5000 (scale 333 at
    4 bits) is stored without any device error."""
    from mixed_precision_kv_loopkv_b200 import KVCells, loopkv_quantize_append
    kv = KVCells(["q4"], 1, 1, 1, 64, 2, 1, 2)
    table = torch.tensor([[0, 1]], dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    k = torch.randn(1, 4, 1, 64, device="cuda").to(torch.bfloat16)
    v = k.clone()
    v[0, 3, 0, 7] = 5000.0
    loopkv_quantize_append(kv, 0, 0, k, v, table, torch.zeros(1, dtype=torch.int32, device="cuda"), err_flag=err)
    torch.cuda.synchronize()
    assert int(err) == 0
