"""Host logic of bench.py on CPU: the slowest-rank reduction and the
whole-job aggregate over world_size 2 gloo ranks, plus the reference arm's
bookkeeping."""

import json
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    bench.init_dist(world, rank, backend="gloo")
    ms = [12.5, 20.0][rank]
    slowest = bench.max_over_ranks(ms, world)
    bench.barrier(world)
    value = bench.aggregate_value(1e9, world, slowest / 1e3)
    q.put((rank, slowest, value))
    import torch.distributed as dist
    dist.destroy_process_group()


def test_two_rank_max_and_aggregate():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, slowest, value in res:
        assert slowest == 20.0
        assert value == pytest.approx(2 * 1e9 / 0.020 / 1e9)


def test_single_rank_helpers():
    assert bench.max_over_ranks(3.0, 1) == 3.0
    assert bench.aggregate_value(2e9, 1, 1.0) == 2.0


def test_profiled_traffic_requires_matching_source(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "decode_attention_demo.json").write_text(json.dumps(
        {"source_sha256": bench.decode_source_hash(), "dram_bytes_per_launch": 1234}))
    csrc = tmp_path / "mixed_precision_kv_loopkv_b200" / "csrc"
    csrc.mkdir(parents=True)
    for f in ("decode.cu", "device_common.cuh"):
        src = os.path.join(bench.ROOT, "mixed_precision_kv_loopkv_b200", "csrc", f)
        (csrc / f).write_bytes(open(src, "rb").read())
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic("demo") == 1234.0
    (csrc / "decode.cu").write_text("// changed\n")
    assert bench.profiled_traffic("demo") is None


def test_ingest_ncu_weights_launches_by_plan(tmp_path, monkeypatch):
    """The ncu launch log is parsed per source kind and weighted by the
    plan's launches of each kind."""
    from workload import get_workload, make_plan
    hdr = ['"ID"', '"Kernel Name"', '"Metric Name"', '"Metric Value"']
    lines = [",".join(hdr)]
    vals = {("0", "q4"): (100.0, 1000.0), ("1", "q2"): (60.0, 600.0), ("2", "q4"): (300.0, 3000.0)}
    for (lid, kind), (dram, inst) in vals.items():
        t = {"q4": 0, "q2": 1}[kind]
        name = f"void loopkv::decode_kernel<{t}, 128, 0, 1, 4, 0>(loopkv::DecodeParams)"
        for metric, v in (("dram__bytes_read.sum", dram), ("dram__bytes_write.sum", 0.0),
                          ("smsp__inst_executed.sum", inst), ("gpu__time_duration.sum", 5.0)):
            lines.append(",".join(f'"{x}"' for x in (lid, name, metric, v)))
    csv_path = tmp_path / "launches.csv"
    csv_path.write_text("\n".join(lines) + "\n")
    (tmp_path / "profiles").mkdir()
    for f in ("decode.cu", "device_common.cuh"):
        d = tmp_path / "mixed_precision_kv_loopkv_b200" / "csrc"
        d.mkdir(parents=True, exist_ok=True)
        (d / f).write_bytes(open(os.path.join(bench.ROOT, "mixed_precision_kv_loopkv_b200", "csrc", f), "rb").read())
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    out = bench.ingest_ncu(str(csv_path), "ouro_step", scale=2.0)
    w = get_workload("ouro_step")
    plan = make_plan(w)
    L, N = w.num_loops, w.num_layers
    src = [plan[c] if plan[c] != "reuse" else plan[(L - 1) * N + c % N] for c in range(len(plan))]
    n4, n2 = src.count("q4"), src.count("q2")
    assert out["per_kind"]["q4"]["dram_bytes_per_launch"] == 2 * 200.0
    assert out["dram_bytes_per_launch"] == pytest.approx((n4 * 400.0 + n2 * 120.0) / (n4 + n2))
    assert out["warp_instructions_per_launch"] == pytest.approx((n4 * 4000.0 + n2 * 1200.0) / (n4 + n2))
    assert bench.profiled_traffic("ouro_step") == pytest.approx(out["dram_bytes_per_launch"])


def test_sweep_overrides_and_strict_json():
    """The tau sweep's overrides reach the workload, and the config stays
    strict JSON for tau = +inf."""
    import json
    import math
    from workload import get_workload
    args = bench.parse_args(["--workload", "tau_sweep", "--tau", "inf", "--temperature", "4", "--all-bf16",
                             "--batch", "2"])
    w = bench.apply_overrides(get_workload(args.workload), args)
    assert math.isinf(w.tau) and w.temperature == 4.0 and w.all_bf16 and w.batch == 2
    cfg = bench.workload_config(w, 1)
    text = json.dumps(cfg, allow_nan=False)
    assert '"tau": "inf"' in text and "all bf16" in cfg["workload"] and "temperature 4.0" in cfg["workload"]
    plain = bench.apply_overrides(get_workload("ouro_step"), bench.parse_args([]))
    assert plain == get_workload("ouro_step")


def test_reference_arm_maps_no_product_library(tmp_path):
    """The oracle arm (all host cores) runs without importing the package,
    so the CUDA library never enters its process."""
    import subprocess
    import sys
    code = (
        "import sys, json; sys.argv = ['bench.py', '--impl', 'reference', '--workload', 'tiny', '--steps', '2', "
        "'--warmup', '1']\n"
        "import bench; bench.main()\n"
        "maps = open('/proc/self/maps').read()\n"
        "print('LOADED' if 'libloopkv' in maps or 'mixed_precision_kv_loopkv_b200' in sys.modules else 'CLEAN')\n")
    res = subprocess.run([sys.executable, "-c", code], cwd=bench.ROOT, capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = res.stdout.strip().splitlines()
    assert lines[-1] == "CLEAN", res.stdout
    line = json.loads(lines[-2])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["cores"] == bench.host_cores()


def test_oracle_budget_on_all_cores():
    """The CPU baseline's worker pool decodes on every host core and counts
    its bytes with the package's own accounting."""
    from workload import get_workload, make_plan, seq_lens_for
    w = get_workload("tiny")
    items = bench.oracle_sample(w, make_plan(w), seq_lens_for(w), n_pairs=2)
    gbs, secs, n_run = bench.run_oracle_budget(items, w, budget_s=0.5, workers=2)
    assert gbs > 0 and secs >= 0.5 and n_run >= 2
