"""Shared helpers of the GPU parity tests: build cells through the C ABI on
seeded inputs and compare them, output by output, with the CPU oracle."""

from __future__ import annotations

import math

import numpy as np
import torch

import oracle as O
from workload import block_table_for, cell_kv, cell_query, make_plan, seq_lens_for

# Output tolerance of the attention result: |gpu - oracle| <= ATOL + RTOL*|oracle|
ATOL, RTOL = 2e-3, 1e-2
# Selection may differ only where the oracle's weight is this close to tau
SEL_WINDOW = 1e-6


def build_store(w, cells=None, capacity=None, device="cuda", flags=0, splits=0, prefill=True):
    """Allocate the cells of workload ``w`` and bulk-append its seeded K/V.

    ``cells`` limits which cells get storage and data (reuse cells always
    need their final-loop source).  Returns (kv, plan, table, lens, kvdata)
    with kvdata[cell] = (K, V) bf16 [B, n_max, Hkv, D] on the device.
    """
    from mixed_precision_kv_loopkv_b200 import KVCells, prefill as prefill_cell

    plan = make_plan(w)
    lens = seq_lens_for(w)
    cap = lens if capacity is None else capacity
    table, num_blocks = block_table_for(w, cap)
    want = set(range(len(plan))) if cells is None else set(cells)
    for c in list(want):
        if plan[c] == "reuse":
            want.add((w.num_loops - 1) * w.num_layers + c % w.num_layers)
    kv = KVCells(plan, w.num_loops, w.num_layers, w.num_heads, w.head_dim, num_blocks,
                 w.batch, table.shape[1], device=device, flags=flags, decode_splits=splits,
                 allocate=want, num_kv_heads=w.num_kv_heads)
    table_d = torch.from_numpy(table).to(device)
    lens_d = torch.from_numpy(lens).to(device)
    data = {}
    if prefill:
        err = torch.zeros(1, dtype=torch.int32, device=device)
        for c in sorted(want):
            if plan[c] == "reuse":
                continue
            loop, layer = divmod(c, w.num_layers)
            k, v = cell_kv(w, loop, layer, device=device)
            prefill_cell(kv, loop, layer, k, v, table_d, lens, err_flag=err)
            data[c] = (k, v)
        assert int(err) == 0, f"prefill flagged device error {int(err)}"
    return kv, plan, table_d, lens_d, data


def _np(t):
    return None if t is None else t.float().cpu().numpy()


def oracle_pair(kind, k, v, q, tau, sm_scale, unit=1, k_cur=None, v_cur=None):
    """Oracle decode of one (cell, sequence, head) from bf16 tensors (and the
    exact current token k_cur, v_cur when given)."""
    seq = O.StoredSequence(kind, k.float().cpu().numpy(), v.float().cpu().numpy())
    return seq.attend(q.float().cpu().numpy(), tau, sm_scale, unit, k_cur=_np(k_cur), v_cur=_np(v_cur))


def oracle_group(kind, k, v, qs, tau, sm_scale, unit=1, k_cur=None, v_cur=None):
    """Oracle decode of the query heads qs [G, D] sharing one KV head."""
    seq = O.StoredSequence(kind, k.float().cpu().numpy(), v.float().cpu().numpy())
    return seq.attend_grouped(qs.float().cpu().numpy(), tau, sm_scale, unit, k_cur=_np(k_cur), v_cur=_np(v_cur))


def undecided(p_heads, tau: float) -> bool:
    """Whether the low-plane bit of a token may legitimately differ between
    GPU (fp32 weights) and oracle (fp64): the union over heads is decided as
    soon as one head's weight is at least tau + window (selected), or every
    head's weight is below tau - window (not selected)."""
    p_heads = np.asarray(p_heads, np.float64)
    if np.any(p_heads >= tau + SEL_WINDOW):
        return False
    return bool(np.any(np.abs(p_heads - tau) < SEL_WINDOW))


def unpack_mask(words: torch.Tensor, n: int) -> np.ndarray:
    w = words.cpu().numpy().astype(np.int64) & 0xFFFFFFFF
    bits = ((w[:, None] >> np.arange(32)) & 1).astype(bool).reshape(-1)
    return bits[:n]


def check_cell(kv, plan, cell, data, q, table, lens, tau, sm_scale, pairs, out=None,
               sel_mask=None, sel_count=None, report=None, unit=1, current=None, atol=ATOL):
    """Compare one decoded cell with the oracle on the given (b, h) pairs
    (h: query head; with grouped queries the oracle decodes every head of
    h's KV head together, for the union of their selections).  current:
    optional (k_cur, v_cur) bf16 [B, Hkv, D], the exact current token the
    kernel attended after the stored ones."""
    src = kv.source_cell(cell)
    kind = plan[src]
    k_all, v_all = data[src]
    lens_h = lens.cpu().numpy()
    out_h = out.float().cpu()
    G = kv.num_heads // kv.num_kv_heads
    groups = {}
    worst = 0.0
    mism = 0
    for (b, h) in pairs:
        n = int(lens_h[b])
        hk = h // G
        kc, vc = (None, None) if current is None else (current[0][b, hk], current[1][b, hk])
        if G == 1:
            o, sel, p = oracle_pair(kind, k_all[b, :n, hk], v_all[b, :n, hk], q[b, h], tau, sm_scale, unit,
                                    k_cur=kc, v_cur=vc)
            p = p[None, :n]
        else:
            if (b, hk) not in groups:
                groups[(b, hk)] = oracle_group(kind, k_all[b, :n, hk], v_all[b, :n, hk],
                                               q[b, hk * G:(hk + 1) * G], tau, sm_scale, unit, k_cur=kc, v_cur=vc)
            og, sel, p = groups[(b, hk)]
            o = og[h - hk * G]
            p = p[:, :n]
        got = out_h[b, h].numpy().astype(np.float64)
        err = np.abs(got - o) - (atol + RTOL * np.abs(o))
        worst = max(worst, float(np.max(np.abs(got - o))) if n else 0.0)
        if np.any(err > 0):
            i = int(np.argmax(err))
            raise AssertionError(f"cell {cell} ({kind}) b={b} h={h} n={n}: channel {i} "
                                 f"gpu {got[i]:.6g} oracle {o[i]:.6g}")
        if sel_mask is not None and n:
            g = unpack_mask(sel_mask[b, h], n)
            diff = np.nonzero(g != sel)[0]
            # with coarser units a token follows its unit's largest weight;
            # with grouped queries, the union over the group's heads.  A token
            # is undecided (a mismatch is excused) only when no head is clearly
            # at or above tau and at least one head lies within the window.
            pu = p if unit == 1 else np.stack([[ph[(t // unit) * unit: (t // unit + 1) * unit].max()
                                                for t in range(n)] for ph in p])
            bad = [t for t in diff if not undecided(pu[:, t], tau)]
            if bad:
                t = bad[0]
                raise AssertionError(f"cell {cell} b={b} h={h}: token {t} selected gpu={g[t]} "
                                     f"oracle={sel[t]} p={p[:, t]} tau={tau}")
            mism += len(diff)
        if sel_count is not None:
            want = int(sel.sum())
            got_c = int(sel_count[b, h])
            if sel_mask is not None:
                want = int(unpack_mask(sel_mask[b, h], n).sum()) if n else 0
            assert got_c == want, (cell, b, h, got_c, want)
    if report is not None:
        report.append({"cell": cell, "kind": kind, "max_abs_err": worst, "sel_mismatch_in_window": mism})
    return worst, mism


def query_for(w, cell, device="cuda", temperature=None):
    loop, layer = divmod(cell, w.num_layers)
    return cell_query(w, loop, layer, device=device, temperature=temperature)


def sample_pairs(w, nseq, seed=0):
    rng = np.random.default_rng(seed)
    seqs = sorted(rng.choice(w.batch, size=min(nseq, w.batch), replace=False).tolist())
    return [(b, h) for b in seqs for h in range(w.num_heads)]


def mask_buffers(kv, batch, device="cuda"):
    words = math.ceil(kv.max_blocks_per_seq * kv.block_size / 32)
    return (torch.zeros((batch, kv.num_heads, words), dtype=torch.int32, device=device),
            torch.zeros((batch, kv.num_heads), dtype=torch.int32, device=device))


def step_parity(w, nseq, cells=None, extra=32, fused=True):
    """One captured looped decode step (append + attend per cell, PDL,
    CUDA graph) exactly as the benchmark runs it, checked on sampled
    sequences of every cell against the oracle."""
    from mixed_precision_kv_loopkv_b200 import LOOPKV_FLAG_PDL, LoopedDecodeStep
    from workload import cell_new_token, seq_lens_for
    kv, plan, table, lens, data = build_store(w, cells=cells, capacity=seq_lens_for(w) + extra,
                                              flags=LOOPKV_FLAG_PDL)
    run_cells = sorted(range(w.num_cells) if cells is None else
                       set(cells) | {kv.source_cell(c) for c in cells})
    q, kn, vn, out = {}, {}, {}, {}
    for c in run_cells:
        q[c] = query_for(w, c)
        out[c] = torch.zeros_like(q[c])
        # every cell's loop computes the token's K/V: stored cells append it,
        # reuse cells attend it exactly
        kn[c], vn[c] = cell_new_token(w, *divmod(c, w.num_layers), device="cuda")
    pos = lens.clone()
    max_len = int(lens.max()) + extra
    step = LoopedDecodeStep(kv, table, pos, q, kn, vn, out, w.tau, w.sm_scale, max_len, cells=run_cells,
                            fused=fused)
    step.run()                      # eager warm-up; idempotent at the same position
    torch.cuda.synchronize()
    for c in run_cells:
        out[c].zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step.run()
    g.replay()
    torch.cuda.synchronize()
    # oracle view: stored cells hold the new token at position n
    full = {}
    for c, (k, v) in data.items():
        if plan[c] == "reuse":
            continue
        kk = torch.cat([k, torch.zeros_like(k[:, :1])], dim=1)
        vv = torch.cat([v, torch.zeros_like(v[:, :1])], dim=1)
        for b in range(w.batch):
            n = int(lens[b])
            kk[b, n], vv[b, n] = kn[c][b, 0], vn[c][b, 0]
        full[c] = (kk, vv)
    pairs = sample_pairs(w, nseq)
    report = []
    for cell in run_cells:
        reuse = plan[cell] == "reuse"
        lc = lens if reuse else lens + 1
        cur = (kn[cell][:, 0], vn[cell][:, 0]) if reuse else None
        check_cell(kv, plan, cell, full, q[cell], table, lc, w.tau, w.sm_scale, pairs, out=out[cell],
                   report=report, current=cur)
    del g
    return report


def store_tensors(kind, k, v, lens, heads=None, splits=0, seed=5, pool_factor=1.3):
    """A one-cell store of kind ``kind`` holding the first lens[b] tokens of
    the given bf16 K, V [B, n_max, Hkv, D] (blocks shuffled in a larger
    pool); returns (kv, table, lens_d).  heads: query heads (default Hkv)."""
    from mixed_precision_kv_loopkv_b200 import KVCells, prefill as prefill_cell
    B, _, hkv, d = k.shape
    rng = np.random.default_rng(seed)
    need = [max(-(-int(n) // 16), 1) for n in lens]
    mb = max(need)
    pool = int(B * mb * pool_factor) + 1
    ids = rng.permutation(pool)[: B * mb].reshape(B, mb).astype(np.int32)
    kv = KVCells([kind], 1, 1, heads or hkv, d, pool, B, mb, decode_splits=splits, num_kv_heads=hkv)
    table = torch.from_numpy(ids).cuda()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    prefill_cell(kv, 0, 0, k, v, table, [int(n) for n in lens], err_flag=err)
    torch.cuda.synchronize()
    assert int(err) == 0, int(err)
    return kv, table, torch.tensor([int(n) for n in lens], dtype=torch.int32, device="cuda")


def seeded_bf16(shape, seed, scale=1.0, device="cuda"):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return (torch.randn(shape, generator=g, device=device) * scale).to(torch.bfloat16)
