"""The low-plane selection set against the oracle on every workload (tiny,
ouro_step, throughput, long_context, tau_sweep), with the count of tokens
whose GPU and oracle selection differ inside the allowed window
|p - tau| < 1e-6 (GPU weights are fp32, the oracle's fp64).  Outside the
window any difference fails.  The counts are printed (pytest -s) and, when
LOOPKV_SELECTION_REPORT names a file, written there as JSON."""

import json
import math
import os

import pytest
import torch

from loopkv_testlib import build_store, check_cell, mask_buffers, query_for, sample_pairs
from workload import get_workload, make_plan

pytestmark = pytest.mark.gpu

_REPORT = {}


def _cells(w, n_q4=2):
    plan = make_plan(w)
    L, N = w.num_loops, w.num_layers
    q4 = [c for c, k in enumerate(plan) if k == "q4"][:n_q4]
    reuse_q4 = [c for c, k in enumerate(plan)
                if k == "reuse" and plan[(L - 1) * N + c % N] == "q4"][:1]
    return q4 + reuse_q4


def _count(w, cells, nseq, taus, temperatures, seed=3):
    from mixed_precision_kv_loopkv_b200 import loopkv_decode_attention
    kv, plan, table, lens, data = build_store(w, cells=cells)
    pairs = sample_pairs(w, nseq, seed=seed)
    mism = selected = checked = 0
    for cell in cells:
        for temp in temperatures:
            q = query_for(w, cell, temperature=temp)
            for tau in taus:
                sm, sc = mask_buffers(kv, w.batch)
                loop, layer = divmod(cell, w.num_layers)
                out = loopkv_decode_attention(kv, loop, layer, q, table, lens, tau, w.sm_scale, sel_mask=sm,
                                              sel_count=sc, max_seq_len=int(lens.max()))
                torch.cuda.synchronize()
                _, m = check_cell(kv, plan, cell, data, q, table, lens, tau, w.sm_scale, pairs, out=out,
                                  sel_mask=sm, sel_count=sc)
                mism += m
                selected += int(sum(int(sc[b, h]) for b, h in pairs))
                checked += sum(int(lens[b]) for b, _ in pairs)
    del kv, data
    torch.cuda.empty_cache()
    return {"cells": cells, "sequence_heads": len(pairs) * len(cells) * len(taus) * len(temperatures),
            "tokens_checked": checked, "selected": selected, "mismatches_in_window": mism}


CASES = {
    "tiny": dict(nseq=1, taus=None, temperatures=(1.0,)),
    "ouro_step": dict(nseq=4, taus=None, temperatures=(1.0,)),
    "throughput": dict(nseq=2, taus=None, temperatures=(1.0,)),
    "long_context": dict(nseq=2, taus=None, temperatures=(1.0,)),
    "tau_sweep": dict(nseq=2, taus=(1e-3, 1e-2, 5e-2), temperatures=(0.5, 1.0, 4.0)),
}


@pytest.mark.parametrize("name", list(CASES))
def test_selection_window_count(name):
    w = get_workload(name)
    c = CASES[name]
    cells = list(range(w.num_cells)) if name == "tiny" else _cells(w, 1 if name == "tau_sweep" else 2)
    taus = c["taus"] or (w.tau,)
    rep = _count(w, cells, c["nseq"], taus, c["temperatures"])
    rep["tau"] = [t if math.isfinite(t) else "inf" for t in taus]
    _REPORT[name] = rep
    print(f"\nselection window {name}: {json.dumps(rep)}")
    assert rep["selected"] > 0
    path = os.environ.get("LOOPKV_SELECTION_REPORT")
    if path:
        with open(path, "w") as f:
            json.dump(_REPORT, f, indent=1)
