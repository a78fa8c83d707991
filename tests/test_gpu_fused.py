"""GPU parity of loopkv_append_decode_attention (one launch: store the new
token, then attend over it): arena and residual bytes bit-exact against the
oracle's record writer for the extended sequences and identical to the
two-launch path (append, then decode), outputs identical to that path and
within tolerance of the oracle, selection exact outside the 1e-6 window."""

import math

import numpy as np
import pytest
import torch

import oracle as O
from loopkv_testlib import check_cell, mask_buffers, query_for
from workload import block_table_for, cell_kv
from workload.configs import Workload

pytestmark = pytest.mark.gpu

# lengths before the step: the new token lands at position n; 31 and 63
# complete a key group, 32 starts one, 0 is a first token
LENS = [0, 1, 30, 31, 32, 63, 100, 511]


def _store(kind, d, lens, heads=2, seed=21):
    from mixed_precision_kv_loopkv_b200 import KVCells, prefill
    w = Workload(name="fused", batch=len(lens), num_loops=1, num_layers=1, num_heads=heads, head_dim=d,
                 context=max(lens) + 1, ctx_range=None, frac_q4=1.0, frac_reuse=0.0, tau=0.01,
                 paging="shuffled", pool_factor=1.3, seed=seed)
    table, nblocks = block_table_for(w, [n + 1 for n in lens])
    k, v = cell_kv(w, 0, 0, device="cuda", n=max(lens) + 1)
    table_d = torch.from_numpy(table).cuda()
    cells = []
    for _ in range(2):  # one for the fused path, one for the two-launch path
        kv = KVCells([kind], 1, 1, heads, d, nblocks, w.batch, table.shape[1])
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        prefill(kv, 0, 0, k, v, table_d, lens, err_flag=err)
        assert int(err) == 0
        cells.append(kv)
    idx = torch.tensor(lens, device="cuda")
    kn = k[torch.arange(len(lens), device="cuda"), idx].unsqueeze(1).contiguous()
    vn = v[torch.arange(len(lens), device="cuda"), idx].unsqueeze(1).contiguous()
    return w, cells, k, v, kn, vn, table_d, table


def _records_match_oracle(kv, kind, k, v, lens, table):
    arena = kv.arena_view(0).cpu().numpy()
    res = kv.residuals[0]
    res_h = None if res is None else res.view(torch.int16).cpu().numpy()
    for b, n in enumerate(lens):
        for h in range(kv.num_heads):
            want, _ = O.sequence_records(kind, k[b, :n, h].float().cpu().numpy(),
                                         v[b, :n, h].float().cpu().numpy())
            got = arena[table[b, : want.shape[0]], h]
            assert np.array_equal(got, want), (kind, b, h, n)
            if res_h is not None:
                for pos in range(32 * (n // 32), n):
                    assert np.array_equal(res_h[b, h, pos % 32], k[b, pos, h].view(torch.int16).cpu().numpy())


@pytest.mark.parametrize("kind", ["q4", "q2", "bf16"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("tau", [0.0, 0.01, math.inf])
def test_fused_step_matches_two_launches_and_oracle(kind, d, tau):
    from mixed_precision_kv_loopkv_b200 import (loopkv_append_decode_attention, loopkv_decode_attention,
                                                loopkv_quantize_append)
    w, (kv_f, kv_u), k, v, kn, vn, table_d, table = _store(kind, d, LENS)
    start = torch.tensor(LENS, dtype=torch.int32, device="cuda")
    lens1 = start + 1
    q = query_for(w, 0, temperature=4.0)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    sm_f, sc_f = mask_buffers(kv_f, w.batch)
    out_f = loopkv_append_decode_attention(kv_f, 0, 0, kn, vn, q, table_d, start, tau, sel_mask=sm_f,
                                           sel_count=sc_f, err_flag=err)
    loopkv_quantize_append(kv_u, 0, 0, kn, vn, table_d, start)
    sm_u, sc_u = mask_buffers(kv_u, w.batch)
    out_u = loopkv_decode_attention(kv_u, 0, 0, q, table_d, lens1, tau, sel_mask=sm_u, sel_count=sc_u)
    torch.cuda.synchronize()
    assert int(err) == 0
    assert torch.equal(kv_f.arenas[0], kv_u.arenas[0])
    if kv_f.residuals[0] is not None:
        for b, n in enumerate(LENS):
            live = slice(0, (n + 1) % 32)
            assert torch.equal(kv_f.residuals[0][b, :, live], kv_u.residuals[0][b, :, live])
    assert torch.equal(out_f, out_u)
    assert torch.equal(sm_f, sm_u) and torch.equal(sc_f, sc_u)
    new_lens = [n + 1 for n in LENS]
    _records_match_oracle(kv_f, kind, k, v, new_lens, table)
    pairs = [(b, h) for b in range(w.batch) for h in range(w.num_heads)]
    check_cell(kv_f, [kind], 0, {0: (k, v)}, q, table_d, lens1, tau, 1.0, pairs, out=out_f,
               sel_mask=sm_f, sel_count=sc_f)


def test_fused_skips_negative_start_and_flags_overflow():
    from mixed_precision_kv_loopkv_b200 import LOOPKV_DEVERR_SEQ_LEN, loopkv_append_decode_attention
    w, (kv, _), k, v, kn, vn, table_d, table = _store("q4", 128, [40, 70])
    before = kv.arenas[0].clone()
    q = query_for(w, 0)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    start = torch.tensor([-1, 70], dtype=torch.int32, device="cuda")
    out = loopkv_append_decode_attention(kv, 0, 0, kn, vn, q, table_d, start, 0.01, err_flag=err)
    torch.cuda.synchronize()
    assert int(err) == 0
    assert not out[0].any() and out[1].abs().sum() > 0
    # sequence 0 untouched: only sequence 1's new row changed
    changed = (kv.arenas[0] != before).nonzero().numel()
    assert changed > 0
    rec = kv.record_bytes("q4")
    view = kv.arenas[0].view(kv.num_blocks, kv.num_heads, rec)
    before_v = before.view(kv.num_blocks, kv.num_heads, rec)
    for blk in table[0][: (40 + 15) // 16]:
        assert torch.equal(view[blk], before_v[blk])
    # start + 1 beyond max_seq_len: flagged, nothing attended
    err.zero_()
    start = torch.tensor([40, 70], dtype=torch.int32, device="cuda")
    out = loopkv_append_decode_attention(kv, 0, 0, kn, vn, q, table_d, start, 0.01, max_seq_len=64, err_flag=err)
    torch.cuda.synchronize()
    assert int(err) & LOOPKV_DEVERR_SEQ_LEN
    assert not out[1].any()
