"""Host-side logic of bench.py, on CPU: the reference arm's JSON line, its
behaviour on ranks other than 0, and the multi-rank aggregation (max over
ranks, whole-job throughput) over a world_size-2 gloo process group."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def run_bench(args, rank=0, world=1):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, env=env, cwd=ROOT,
                          capture_output=True, text=True, timeout=600)


def test_reference_arm_prints_one_json_line():
    r = run_bench(["--impl", "reference", "--steps", "2", "--warmup", "1", "--workload", "tiny"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["value"] > 0 and d["unit"] == "TFLOP/s" and d["higher_is_better"] is True
    assert d["steps"] == 2 and d["warmup"] == 1 and d["n_gpus"] == 1
    assert d["vs_baseline"] is None and d["dtype"] == "f64" and d["data"] == "synthetic"
    assert d["config"]["workload"].startswith("tiny")
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_do_no_work():
    r = run_bench(["--impl", "reference", "--steps", "2", "--warmup", "1", "--workload", "tiny"], rank=1, world=2)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""


def test_replica_throughput():
    # 2 replicas x 10 steps x 1e12 FLOP in 4 s (the slowest rank) = 5 TFLOP/s
    assert bench.replica_tflops(2, 10, 1e12, 4000.0) == pytest.approx(5.0)
    assert bench.replica_tflops(1, 10, 1e12, 4000.0) == pytest.approx(2.5)
    assert bench.all_max(3.0, 1) == 3.0


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        t_rank = [1200.0, 1500.0][rank]          # this rank's summed step time, ms
        bench.barrier(world)
        t_max = bench.all_max(t_rank, world)
        out[rank] = (t_max, bench.replica_tflops(world, 10, 1e12, t_max))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo():
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    for rank in range(world):
        t_max, value = res[rank]
        assert t_max == 1500.0                   # every rank sees the slowest rank's time
        assert value == pytest.approx(world * 10 * 1e12 / 1.5 / 1e12)


def test_measured_traffic_follows_the_kernel_sources(tmp_path, monkeypatch):
    """The roofline's DRAM traffic comes from the committed ncu record only
    while the kernel's sources hash to the value stored with it, and only for
    the workload it was captured on."""
    import hashlib
    from flashattention_bf16_fwd_b200.workloads import WORKLOADS
    src = tmp_path / "flashattention_bf16_fwd_b200" / "csrc"
    src.mkdir(parents=True)
    (src / "a.cuh").write_text("kernel A\n")
    (src / "b.cuh").write_text("helpers\n")
    digest = hashlib.sha256(b"kernel A\nhelpers\n").hexdigest()
    (tmp_path / "profiles").mkdir()
    rec = {"fa_bwd_kernel": {"sources": ["a.cuh", "b.cuh"], "csrc_sha256": digest,
                             "per_workload": {"gpt2s": {"dram_bytes_per_launch": 1234}}}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_traffic("fa_bwd_kernel", WORKLOADS["gpt2s"]) == 1234
    assert bench.measured_traffic("fa_bwd_kernel", WORKLOADS["gpt2m"]) is None
    assert bench.measured_traffic("fa_fwd_kernel", WORKLOADS["gpt2s"]) is None
    (src / "b.cuh").write_text("helpers, changed\n")
    assert bench.measured_traffic("fa_bwd_kernel", WORKLOADS["gpt2s"]) is None
