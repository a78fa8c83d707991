#!/usr/bin/env python3
"""Benchmark of the LoopKV decode path on B200.

Metric: decode-attention KV GB/s (algorithmic bytes the decode kernels must
move, over device time) and microseconds per looped decode step.

One step = every (loop, layer) cell of the Ouro-1.4B-like workload in order:
stored cells append the current token and attend over n + 1 tokens in one
launch (loopkv_append_decode_attention; --no-fuse: append kernel, then decode
kernel), reuse cells attend over the final loop's n tokens
(loopkv_decode_attention).  The step is captured once in a CUDA graph (kernels
launched with programmatic dependent launch) and replayed.  Every step
decodes at the same position (the append rewrites the same token), so the
context stays at the workload's length however many steps are timed.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Multi-GPU (torchrun, one process per GPU): every rank holds its own batch
(sequence data parallelism, no collective on the data path); the timed
region is bracketed by barriers and the slowest rank's time is used.
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode-attention KV GB/s (% of B200 HBM peak) and µs per looped decode step"
# what the decode kernel computes in: fp32 logits from the 2/4-bit key codes
# (packed fp32 FMAs), values as u16 fixed-point weights x 2-bit codes (dp2a,
# exact 32-bit integer group sums) accumulated in fp32
DTYPE = "f32 logits; u16 weights x u2 codes (dp2a) values, f32 accumulate"
FALLBACK_HBM_GBS = 6650.0


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="mine", choices=["mine", "reference"])
    ap.add_argument("--workload", default="throughput")
    ap.add_argument("--splits", type=int, default=0, help="decode splits override (0 = automatic)")
    ap.add_argument("--no-pdl", action="store_true")
    ap.add_argument("--select-unit", type=int, default=1, choices=[1, 16, 32],
                    help="low-plane selection unit in tokens (1: per token, the method's rule)")
    ap.add_argument("--no-fuse", action="store_true",
                    help="stored cells append and attend in two launches instead of one")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="CPU-baseline sample budget")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--batch", type=int, default=0,
                    help="override the workload's batch (a smaller case of the same kernel)")
    ap.add_argument("--cells", type=int, default=0,
                    help="run only the first N cells (and their reuse sources): a small case for ncu")
    ap.add_argument("--tau", type=float, default=None,
                    help="override the workload's low-plane threshold (tau sweep; 'inf' for none)")
    ap.add_argument("--temperature", type=float, default=None,
                    help="override the query temperature (tau sweep: flat 0.5 .. peaky 4)")
    ap.add_argument("--all-bf16", action="store_true",
                    help="store every cell as bf16 (the unquantised comparison run of the tau sweep)")
    ap.add_argument("--kv-heads", type=int, default=0,
                    help="KV heads (grouped queries: the workload's query heads share them; 0 = one per head)")
    ap.add_argument("--ingest-ncu", default=None, metavar="CSV",
                    help="write profiles/decode_attention_<workload>.json from an ncu --csv launch log, then exit")
    ap.add_argument("--ncu-scale", type=float, default=1.0,
                    help="with --ingest-ncu: factor from the captured launches to the workload's full launch")
    ap.add_argument("--ncu-command", default="", help="with --ingest-ncu: the command that made the capture")
    return ap.parse_args(argv)


def apply_overrides(w, args):
    """The workload with the command line's batch / tau / temperature / bf16 overrides."""
    kw = {}
    if args.batch:
        kw["batch"] = args.batch
    if args.tau is not None:
        kw["tau"] = args.tau
    if args.temperature is not None:
        kw["temperature"] = args.temperature
    if args.all_bf16:
        kw["all_bf16"] = True
    if args.kv_heads:
        kw["num_kv_heads"] = args.kv_heads
    return w.with_(**kw) if kw else w


# ----------------------------------------------------------------- ranks

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world, local, backend="nccl"):
    if world <= 1:
        return
    import torch.distributed as dist
    kw = dict(backend=backend, timeout=datetime.timedelta(seconds=120))
    if backend == "nccl":
        kw["device_id"] = torch.device(f"cuda:{local}")
    dist.init_process_group(**kw)


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Largest value of x over all ranks (the slowest rank's time)."""
    if world <= 1:
        return float(x)
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_value(bytes_per_rank: float, world: int, seconds_max: float) -> float:
    """Whole-job GB/s: bytes all ranks moved over the slowest rank's time."""
    return bytes_per_rank * world / seconds_max / 1e9


# ----------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and clock-event reasons of one GPU (NVML) while the
    timed region runs.  Reads only; changes no GPU setting."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index: int, period_s: float = 0.02):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period = period_s
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(device_index)
            try:
                self._h = pynvml.nvmlDeviceGetHandleByUUID(f"GPU-{props.uuid}")
            except Exception:
                bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
                self._h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            self._nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # no NVML: report no clocks
            self._nv, self.error = None, str(e)

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                bits = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for mask, name in self.REASONS.items():
                    if bits & mask:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self._nv is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread:
            self._thread.join()

    def summary(self):
        if self._nv is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "NVML unavailable"}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ----------------------------------------------------------------- peaks, profile

def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def decode_source_hash() -> str:
    h = hashlib.sha256()
    for f in ("decode.cu", "device_common.cuh"):
        with open(os.path.join(ROOT, "mixed_precision_kv_loopkv_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_fields(workload: str) -> dict:
    """Machine-written fields of the committed ncu summary of the decode
    kernel (profiles/decode_attention_<workload>.json, written by
    --ingest-ncu); empty unless it was taken on the current kernel source."""
    path = os.path.join(ROOT, "profiles", f"decode_attention_{workload}.json")
    try:
        with open(path) as f:
            fields = json.load(f)
        return fields if fields.get("source_sha256") == decode_source_hash() else {}
    except Exception:
        return {}


def profiled_traffic(workload: str):
    """Per-launch DRAM bytes of the decode kernel from the committed ncu summary."""
    try:
        return float(profiled_fields(workload)["dram_bytes_per_launch"])
    except (KeyError, ValueError, TypeError):
        return None


KIND_OF_TEMPLATE = {"0": "q4", "1": "q2", "3": "bf16"}


def parse_ncu_csv(path: str):
    """Per-launch metrics of the decode kernel from an ncu --csv log:
    [(source kind, {metric: value})] in launch order."""
    import csv
    import re
    rows, hdr = [], None
    with open(path) as f:
        for r in csv.reader(f):
            if r and r[0] == "ID":
                hdr = r
                continue
            if hdr and len(r) == len(hdr):
                rows.append(dict(zip(hdr, r)))
    launches = {}
    for d in rows:
        if "decode_kernel" not in d["Kernel Name"]:
            continue
        m = re.search(r"decode_kernel<(\d+),", d["Kernel Name"])
        kind = KIND_OF_TEMPLATE.get(m.group(1), "?") if m else "?"
        ent = launches.setdefault(d["ID"], (kind, {}))
        try:
            ent[1][d["Metric Name"]] = float(d["Metric Value"].replace(",", ""))
        except ValueError:
            pass
    return [launches[k] for k in sorted(launches, key=int)]


def ingest_ncu(csv_path: str, workload: str, scale: float = 1.0, command: str = "") -> dict:
    """Plan-weighted per-launch DRAM bytes and warp instructions of the
    decode kernel for a workload, from the launches of an ncu capture
    (scaled by ``scale`` when the capture ran a smaller batch); written to
    profiles/decode_attention_<workload>.json with the kernel source hash."""
    from workload import get_workload, make_plan
    w = get_workload(workload)
    plan = make_plan(w)
    L, N = w.num_loops, w.num_layers
    src_kind = [plan[c] if plan[c] != "reuse" else plan[(L - 1) * N + c % N] for c in range(len(plan))]
    per_kind = {}
    for kind, m in parse_ncu_csv(csv_path):
        per_kind.setdefault(kind, []).append(m)
    out = {"source_sha256": decode_source_hash(), "workload": workload, "capture_scale": scale,
           "command": command, "per_kind": {}}
    tot_dram = tot_inst = 0.0
    weight = 0
    for kind in sorted(set(src_kind)):
        ms = per_kind.get(kind)
        if not ms:
            raise ValueError(f"no captured launch of a {kind} source")
        dram = [(m.get("dram__bytes_read.sum", 0) + m.get("dram__bytes_write.sum", 0)) * scale for m in ms]
        inst = [m.get("smsp__inst_executed.sum", 0) * scale for m in ms]
        dur = [m.get("gpu__time_duration.sum", 0) * scale for m in ms]
        cnt = src_kind.count(kind)
        out["per_kind"][kind] = {"launches_captured": len(ms), "launches_per_step": cnt,
                                 "dram_bytes_per_launch": sum(dram) / len(ms),
                                 "warp_instructions_per_launch": sum(inst) / len(ms),
                                 "duration_ns_per_launch": sum(dur) / len(ms)}
        tot_dram += cnt * sum(dram) / len(ms)
        tot_inst += cnt * sum(inst) / len(ms)
        weight += cnt
    out["dram_bytes_per_launch"] = tot_dram / weight
    out["warp_instructions_per_launch"] = tot_inst / weight
    path = os.path.join(ROOT, "profiles", f"decode_attention_{workload}.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
        f.write("\n")
    return out


# ----------------------------------------------------------------- workload setup

def setup(w, pdl: bool, splits: int, extra: int = 64, ncells: int = 0, fused: bool = True, unit: int = 1):
    from mixed_precision_kv_loopkv_b200 import (LOOPKV_FLAG_PDL, LOOPKV_FLAG_SELECT_BLOCK, LOOPKV_FLAG_SELECT_GROUP,
                                                KVCells, LoopedDecodeStep, prefill)
    from workload import block_table_for, cell_kv, cell_new_token, cell_query, make_plan, seq_lens_for

    plan = make_plan(w)
    lens = seq_lens_for(w)
    table_np, num_blocks = block_table_for(w, lens + extra)
    C = len(plan)
    run = list(range(C))
    if ncells:
        src = lambda c: c if plan[c] != "reuse" else (w.num_loops - 1) * w.num_layers + c % w.num_layers
        run = sorted(set(range(ncells)) | {src(c) for c in range(ncells)})
    kv = KVCells(plan, w.num_loops, w.num_layers, w.num_heads, w.head_dim, num_blocks, w.batch,
                 table_np.shape[1], num_kv_heads=w.num_kv_heads,
                 flags=(LOOPKV_FLAG_PDL if pdl else 0) | {1: 0, 16: LOOPKV_FLAG_SELECT_BLOCK,
                                                          32: LOOPKV_FLAG_SELECT_GROUP}[unit],
                 decode_splits=splits,
                 allocate=set(run))
    table = torch.from_numpy(table_np).cuda()
    stored = [c for c in run if plan[c] != "reuse"]
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    for c in stored:
        loop, layer = divmod(c, w.num_layers)
        k, v = cell_kv(w, loop, layer, device="cuda")
        prefill(kv, loop, layer, k, v, table, lens, err_flag=err)
        del k, v
    if int(err):
        raise RuntimeError(f"prefill flagged device error {int(err)}")
    q_all = torch.stack([cell_query(w, *divmod(c, w.num_layers), device="cuda") for c in range(C)])
    # the current token's K/V of every cell's loop: stored cells append it,
    # reuse cells attend it exactly after the final loop's tokens
    kn_all = torch.empty((len(run), w.batch, 1, w.kv_heads, w.head_dim), dtype=torch.bfloat16,
                         device="cuda")
    vn_all = torch.empty_like(kn_all)
    for i, c in enumerate(run):
        kn_all[i], vn_all[i] = cell_new_token(w, *divmod(c, w.num_layers), device="cuda")
    out_all = torch.zeros_like(q_all)
    sel_all = torch.zeros((C, w.batch, w.num_heads), dtype=torch.int32, device="cuda")
    slot = {c: i for i, c in enumerate(run)}
    pos = torch.from_numpy(lens).cuda()
    step = LoopedDecodeStep(
        kv, table, pos, [q_all[c] for c in range(C)],
        {c: kn_all[slot[c]] for c in run}, {c: vn_all[slot[c]] for c in run},
        [out_all[c] for c in range(C)], w.tau, w.sm_scale, int(lens.max()) + 1,
        sel_count=[sel_all[c] for c in range(C)], cells=run, fused=fused)
    torch.cuda.synchronize()
    return dict(plan=plan, lens=lens, kv=kv, step=step, q_all=q_all, kn_all=kn_all, vn_all=vn_all,
                out_all=out_all, sel_all=sel_all)


def time_end_to_end(g, S, steps):
    """Device time (ms) of ``steps`` steps fed from and drained to pinned
    host memory: every step copies its queries and new tokens in from the
    host and its outputs back out.  The copies run on a second stream
    through two sets of staging buffers, one step ahead of (inputs) and one
    behind (outputs) the step's kernels, so transfers overlap computation;
    the step itself only adds two device-to-device copies.  The timed region
    spans the first host-to-device copy to the last device-to-host copy.
    Returns (ms, host-to-device bytes per step, device-to-host bytes per step)."""
    ins = [S["q_all"], S["kn_all"], S["vn_all"]]
    out = S["out_all"]
    host_in = [t.cpu().pin_memory() for t in ins]
    host_out = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    stage_in = [[torch.empty_like(t) for t in ins] for _ in range(2)]
    stage_out = [torch.empty_like(out) for _ in range(2)]
    comp, copy = torch.cuda.current_stream(), torch.cuda.Stream()
    in_ready, in_free, out_ready, out_free = ([torch.cuda.Event() for _ in range(2)] for _ in range(4))
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(comp)
    for e in in_free + out_free:
        e.record(comp)
    copy.wait_stream(comp)

    def h2d(i):
        k = i % 2
        with torch.cuda.stream(copy):
            copy.wait_event(in_free[k])
            for st, h in zip(stage_in[k], host_in):
                st.copy_(h, non_blocking=True)
            in_ready[k].record(copy)

    h2d(0)
    for i in range(steps):
        k = i % 2
        if i + 1 < steps:
            h2d(i + 1)
        comp.wait_event(in_ready[k])
        for t, st in zip(ins, stage_in[k]):
            t.copy_(st, non_blocking=True)
        in_free[k].record(comp)
        g.replay()
        comp.wait_event(out_free[k])
        stage_out[k].copy_(out, non_blocking=True)
        out_ready[k].record(comp)
        with torch.cuda.stream(copy):
            copy.wait_event(out_ready[k])
            host_out[k].copy_(stage_out[k], non_blocking=True)
            out_free[k].record(copy)
    comp.wait_stream(copy)
    b.record(comp)
    b.synchronize()
    if not torch.equal(host_out[(steps - 1) % 2], out.cpu()):
        raise RuntimeError("end-to-end outputs differ from the device result")
    h2d_bytes = sum(h.numel() * h.element_size() for h in host_in)
    d2h_bytes = out.numel() * out.element_size()
    return a.elapsed_time(b), h2d_bytes, d2h_bytes


class DecodeOnly:
    """The decode launches of a step without the appends (roofline timing)."""

    def __init__(self, step):
        self.s = step

    def run(self):
        from mixed_precision_kv_loopkv_b200 import LOOPKV_CELL_REUSE, loopkv_decode_attention
        s, kv = self.s, self.s.kv
        for cell in s.cells:
            loop, layer = divmod(cell, kv.num_layers)
            reuse = kv.plan_codes[cell] == LOOPKV_CELL_REUSE
            lens = s.pos if reuse else s.pos_next
            loopkv_decode_attention(kv, loop, layer, s.q[cell], s.block_table, lens, s.tau, s.sm_scale,
                                    out=s.out[cell], max_seq_len=s.max_seq_len,
                                    sel_count=s.sel_count[cell], k_cur=s.k_new.get(cell) if reuse else None,
                                    v_cur=s.v_new.get(cell) if reuse else None)


def capture(fn):
    fn()                     # eager warm-up (idempotent at a fixed position)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


def time_replays(g, n: int) -> float:
    """Device milliseconds of n back-to-back replays (events on this stream)."""
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(n):
        g.replay()
    b.record()
    b.synchronize()
    return a.elapsed_time(b)


# ----------------------------------------------------------------- CPU oracle

def oracle_sample(w, plan, lens, n_pairs: int, seed: int = 0):
    """A seeded sample of (cell, sequence, head) decodes for the CPU oracle:
    the same inputs as the GPU run, built into the oracle's own stored form."""
    import oracle as O
    from workload import cell_kv, cell_query
    rng = np.random.default_rng(seed)
    C = len(plan)
    cells = rng.choice(C, size=min(n_pairs, C), replace=False)
    items = []
    for cell in cells:
        cell = int(cell)
        src = cell if plan[cell] != "reuse" else (w.num_loops - 1) * w.num_layers + cell % w.num_layers
        g = w.num_heads // w.kv_heads
        b, hk = int(rng.integers(w.batch)), int(rng.integers(w.kv_heads))
        n = int(lens[b])
        # the GPU arm's inputs come from the CUDA generator; without a GPU the
        # CPU generator gives inputs of the same distribution
        dev = "cuda" if torch.cuda.is_available() else "cpu"
        k, v = cell_kv(w, *divmod(src, w.num_layers), device=dev)
        kk = k[b, :n, hk].float().cpu().numpy()
        vv = v[b, :n, hk].float().cpu().numpy()
        del k, v
        # the query heads of KV head hk (one head without grouped queries)
        q = cell_query(w, *divmod(cell, w.num_layers), device=dev)[b, hk * g:(hk + 1) * g].float().cpu().numpy()
        items.append((plan[src], O.StoredSequence(plan[src], kk, vv), q, n))
    torch.cuda.empty_cache()
    return items


def oracle_decode(seq, q, w):
    """The oracle's decode of one sampled item: q [G, D] holds the query heads
    of one KV head (G = 1 without grouped queries).  Returns the selection."""
    if len(q) == 1:
        return seq.attend(q[0], w.tau, w.sm_scale)[1]
    return seq.attend_grouped(q, w.tau, w.sm_scale)[1]


def byte_accounting():
    """The package's byte-accounting module, loaded from its file: the CPU
    legs must not import the package, whose import maps the CUDA library."""
    import importlib.util
    name = "_loopkv_accounting"
    if name in sys.modules:
        return sys.modules[name]
    path = os.path.join(ROOT, "mixed_precision_kv_loopkv_b200", "accounting.py")
    spec = importlib.util.spec_from_file_location(name, path)
    mod = importlib.util.module_from_spec(spec)
    sys.modules[name] = mod
    spec.loader.exec_module(mod)
    return mod


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


_POOL_ITEMS, _POOL_W = None, None


def _oracle_worker_init(items, w):
    global _POOL_ITEMS, _POOL_W
    _POOL_ITEMS, _POOL_W = items, w
    from threadpoolctl import threadpool_limits
    threadpool_limits(limits=1)       # one BLAS thread per worker process


def _oracle_item_bytes(kind, n, sel, g, d):
    return byte_accounting().decode_bytes(kind, d, n, int(sel.sum())) + (g - 1) * 4 * d


def _oracle_worker_budget(args):
    """Round robin over the sample from a worker-specific start for
    budget_s seconds; returns (bytes, decodes, seconds)."""
    start, budget_s = args
    items, w = _POOL_ITEMS, _POOL_W
    total, i = 0, start
    t0 = time.perf_counter()
    while True:
        kind, seq, q, n = items[i % len(items)]
        sel = oracle_decode(seq, q, w)
        total += _oracle_item_bytes(kind, n, sel, len(q), w.head_dim)
        i += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            return total, i - start, el


def _oracle_worker_one(index):
    items, w = _POOL_ITEMS, _POOL_W
    kind, seq, q, n = items[index % len(items)]
    sel = oracle_decode(seq, q, w)
    return _oracle_item_bytes(kind, n, sel, len(q), w.head_dim)


def oracle_pool(items, w, workers: int):
    """A pool of oracle worker processes (spawned, so that it is safe after
    the GPU arm has initialised CUDA), one per host core."""
    import multiprocessing as mp
    return mp.get_context("spawn").Pool(workers, initializer=_oracle_worker_init, initargs=(items, w))


def run_oracle_budget(items, w, budget_s: float, workers: int):
    """Every worker decodes sampled items for budget_s seconds, all at once;
    returns (GB/s over all workers, seconds, decodes run)."""
    with oracle_pool(items, w, workers) as pool:
        pool.map(_oracle_worker_one, range(workers))          # warm-up: imports, first decode
        res = pool.map(_oracle_worker_budget, [(k, budget_s) for k in range(workers)])
    total = sum(r[0] for r in res)
    secs = max(r[2] for r in res)
    return total / secs / 1e9, secs, sum(r[1] for r in res)


def run_oracle_steps(items, w, steps: int, warmup: int, workers: int):
    """Steps of one decode per worker, all workers at once; each step is
    timed by the host clock.  Returns (GB/s, seconds, decodes run)."""
    with oracle_pool(items, w, workers) as pool:
        for s in range(max(warmup, 1)):
            pool.map(_oracle_worker_one, range(s * workers, (s + 1) * workers))
        total = 0
        t0 = time.perf_counter()
        for s in range(steps):
            total += sum(pool.map(_oracle_worker_one, range(s * workers, (s + 1) * workers)))
        secs = time.perf_counter() - t0
    return total / secs / 1e9, secs, steps * workers


# ----------------------------------------------------------------- arms

def workload_config(w, world):
    frac = f"{round(w.frac_q4 * 100)}/{round((1 - w.frac_q4 - w.frac_reuse) * 100)}/{round(w.frac_reuse * 100)}"
    plan = "all bf16" if w.all_bf16 else f"plan {frac} 4b/2b/reuse"
    ctx = f"{w.ctx_range[0]}..{w.ctx_range[1]}" if w.ctx_range else str(w.context)
    temp = "" if w.temperature == 1.0 else f", q temperature {w.temperature}"
    heads = (f"{w.num_heads} MHA heads" if w.kv_heads == w.num_heads
             else f"{w.num_heads} query heads on {w.kv_heads} KV heads")
    return {
        "workload": (f"{w.name}: batch {w.batch}, {w.num_loops} loops x {w.num_layers} layers, "
                     f"{heads} x {w.head_dim}, context {ctx}, {plan}, "
                     f"tau {w.tau}{temp}, paged 16-token blocks ({w.paging})"),
        "batch_per_gpu": w.batch, "context": ctx, "cells": w.num_cells,
        "tau": w.tau if math.isfinite(w.tau) else "inf", "temperature": w.temperature,
        "l2": "inputs larger than L2 (whole step streams the cache once)",
        "parallelism": f"dp{world} (sequences)",
    }


def reference_arm(args, world, rank):
    """The oracle as it stands on the host cores: every step, one sampled
    (cell, sequence, head) decode per host core, all cores at once."""
    from workload import get_workload, make_plan, seq_lens_for
    if rank != 0:
        return
    w = apply_overrides(get_workload(args.workload), args)
    plan, lens = make_plan(w), seq_lens_for(w)
    items = oracle_sample(w, plan, lens, n_pairs=16)
    cores = host_cores()
    gbs, secs, n_run = run_oracle_steps(items, w, steps=args.steps, warmup=args.warmup, workers=cores)
    line = {
        "impl": "reference", "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / max(args.steps, 1) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w, 1),
        "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": f"one (cell, sequence, head) decode per host core per step ({cores} worker "
                                   f"processes, one BLAS thread each), round robin over 16 seeded pairs of "
                                   f"the {w.name} workload"},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main_arm(args, world, rank, local):
    from mixed_precision_kv_loopkv_b200.accounting import step_bytes
    from workload import get_workload

    torch.cuda.set_device(local)
    init_dist(world, local)
    w = apply_overrides(get_workload(args.workload), args)
    S = setup(w, pdl=not args.no_pdl, splits=args.splits, ncells=args.cells, fused=not args.no_fuse,
              unit=args.select_unit)
    step, plan, lens = S["step"], S["plan"], S["lens"]
    dev = torch.device(f"cuda:{local}")

    g = capture(step.run)
    for _ in range(max(args.warmup, 3)):
        g.replay()
    torch.cuda.synchronize()
    barrier(world)
    with ClockSampler(local) as clocks:
        ms = time_replays(g, args.steps)
    barrier(world)
    ms_max = max_over_ranks(ms, world, dev)

    sel = S["sel_all"].cpu().numpy()
    bytes_step = step_bytes(plan, w.num_layers, w.num_loops, w.head_dim, w.num_heads, lens + 1, lens, sel,
                            group=w.num_heads // w.kv_heads,
                            cells=step.cells, reuse_current=True)
    value = aggregate_value(bytes_step * args.steps, world, ms_max / 1e3)
    us_step = ms_max / args.steps * 1e3

    # dominant kernel: the decode launches alone, same state
    gd = capture(DecodeOnly(step).run)
    reps = max(20, args.steps // 4)
    ms_dec = time_replays(gd, reps)
    launches = len(step.cells)
    per_launch_s = ms_dec / 1e3 / (reps * launches)
    achieved = bytes_step / launches / per_launch_s / 1e9
    peak, peak_kind = hbm_peak()
    # the committed ncu counters describe the workload as defined; any
    # override of its shape or launch options leaves them unused
    as_profiled = not (args.batch or args.cells or args.splits or args.kv_heads or args.all_bf16 or args.no_fuse
                       or args.no_pdl or args.select_unit != 1 or args.tau is not None
                       or args.temperature is not None)
    traffic = profiled_traffic(w.name) if as_profiled else None
    try:
        inst_per_launch = float(profiled_fields(w.name)["warp_instructions_per_launch"]) if as_profiled else None
    except (KeyError, ValueError):
        inst_per_launch = None

    # end to end: inputs of every step copied in from pinned host memory,
    # outputs copied back, inside the timed region
    e2e_steps = max(3, args.steps // 4)
    barrier(world)
    e2e_ms, h2d, d2h = time_end_to_end(g, S, e2e_steps)
    e2e_ms = max_over_ranks(e2e_ms, world, dev)
    e2e_value = aggregate_value(bytes_step * e2e_steps, world, e2e_ms / 1e3)

    cpu = None
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        items = oracle_sample(w, plan, lens, n_pairs=12)
        cores = host_cores()
        gbs, secs, n_run = run_oracle_budget(items, w, budget_s=args.cpu_seconds, workers=cores)
        unit = "head" if w.kv_heads == w.num_heads else f"KV head with its {w.num_heads // w.kv_heads} query heads"
        cpu = {"value": gbs, "unit": "GB/s", "cores": cores, "kind": "oracle",
               "sample": f"{n_run} (cell, sequence, {unit}) decodes over {secs:.1f} s on {cores} worker "
                         f"processes (one per host core, numpy fp64, one BLAS thread each), round robin over "
                         f"12 seeded pairs of the {w.name} workload"}

    if rank == 0:
        cfg = workload_config(w, world)
        if args.cells:
            cfg["cells_run"] = len(step.cells)
        cfg.update({"pdl": not args.no_pdl, "fused_append": not args.no_fuse, "select_unit": args.select_unit,
                    "splits": args.splits or "auto", "cuda_graph": True,
                    "algorithmic_bytes_per_step": bytes_step,
                    "selected_low_plane_rows_per_step": int(sel.sum())})
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": us_step / 1e3, "us_per_step": us_step,
            "pct_of_hbm_peak": value / world / peak * 100, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": DTYPE, "data": "synthetic", "config": cfg,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": traffic,
                         "kernel": "decode_kernel (all decode launches of one step, timed alone)",
                         "per_launch_us": per_launch_s * 1e6,
                         "bytes_per_launch": bytes_step / launches,
                         "peak_source": f"{peak_kind} hbm_gbs"},
            # the launches are bound by instruction issue: warp instructions per
            # second (ncu count per launch / measured launch time) against the
            # SMs' issue peak (4 schedulers x SMs x the sampled SM clock)
            "issue_roofline": None if inst_per_launch is None or not clocks.summary().get("sm_mhz") else {
                "achieved": inst_per_launch / per_launch_s,
                "peak": 4 * torch.cuda.get_device_properties(dev).multi_processor_count
                        * clocks.summary()["sm_mhz"] * 1e6,
                "unit": "warp instructions / s",
                "frac": inst_per_launch / per_launch_s / (
                    4 * torch.cuda.get_device_properties(dev).multi_processor_count
                    * clocks.summary()["sm_mhz"] * 1e6),
                "warp_instructions_per_launch": inst_per_launch},
            "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "us_per_step": e2e_ms / e2e_steps * 1e3},
            "gpu_launches": args.steps * step.launches_per_step(),
            "clocks": clocks.summary(),
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    del g, gd
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def main(argv=None):
    args = parse_args(argv)
    if args.ingest_ncu:
        print(json.dumps(ingest_ncu(args.ingest_ncu, args.workload, args.ncu_scale, args.ncu_command), indent=1))
        return
    world, rank, local = dist_env()
    if args.impl == "reference":
        reference_arm(args, world, rank)
        return
    main_arm(args, world, rank, local)


if __name__ == "__main__":
    main()
