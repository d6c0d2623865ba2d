#!/usr/bin/env python
"""Benchmark: BF16 attention forward + backward on B200, repeated-max fix on.

One step = fa_fwd + fa_bwd (the whole hot path) over one batch of synthetic
input of the chosen workload (default: GPT-2 small attention, B=8 H=12 N=1024
d=64, causal).  Prints ONE JSON line on rank 0.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   # the FP64 CPU oracle, timed on host cores

Timing: CUDA events on the launching stream around every step (fa_fwd then
fa_bwd, the library's public calls, which launch four kernels back to back
with programmatic dependent launch); the L2 is flushed (a 512 MiB write)
before each step, outside the events.  A second pass of the same number of
steps calls the backward's three launches one by one with events between all
four kernels: it gives the per-kernel times and the roofline of the dominant
kernel.  A third pass repeats the first without the flush (L2-warm).

The line's headline is the chosen workload.  Its ``per_config`` block repeats
the same three passes for each workload of ``--configs`` (default: GPT-2
small, GPT-2 medium, the long-context shape and the Llama-2-7B shape), each
over a step count sized to about a second: median step time flushed and
warm, TFLOP/s, percent of peak, per-kernel times and the dominant kernel's
roofline fraction, and at d = 64 the bound the MUFU exponentials put on the
throughput.

Multi-GPU runs are independent replicas (attention over (B, H) has no
exchange step): each rank runs the full workload on its own GPU, and the
slowest rank's time is used.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from flashattention_bf16_fwd_b200.workloads import WORKLOADS, make_inputs, visible_pairs, workload_flops  # noqa: E402

METRIC = "BF16 attn fwd+bwd TFLOP/s (% of B200 BF16 peak), fix on; max err vs FP64 oracle"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
DATASHEET_BF16_TFLOPS = 2250.0
L2_FLUSH_BYTES = 512 << 20


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="gpt2s")
    ap.add_argument("--fix-mode", type=int, default=1)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="budget of the oracle CPU baseline")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--configs", default="gpt2s,gpt2m,long,llama7b",
                    help="workloads measured into the line's per_config block (comma list, or none)")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def all_max(x: float, world: int) -> float:
    """The largest of the ranks' values (every rank gets it): the slowest rank's time."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_tflops(world: int, steps: int, flops_per_step: float, t_max_ms: float) -> float:
    """Whole-job throughput of `world` replicas that each ran `steps` steps: the
    work of all ranks divided by the slowest rank's time."""
    return world * steps * flops_per_step / (t_max_ms * 1e-3) / 1e12


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the GPU is busy."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None
        self.t0 = self.t1 = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "50", "-f", self.path], stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def mark(self, begin: bool):
        if begin:
            self.t0 = time.time()
        else:
            self.t1 = time.time()

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.12)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9 and parts[1].replace(".", "").isdigit():
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows]
        busy = [s for s, r in zip(sm, rows) if float(r[3]) > 150.0] or sm
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return {"sm_mhz": float(np.median(busy)), "sm_max_mhz": float(rows[0][2]), "reasons": reasons,
                "samples": len(rows), "power_w_max": max(float(r[3]) for r in rows)}


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max([i.get("num_threads", 1) for i in info] or [1])
    except Exception:
        return os.cpu_count() or 1


def oracle_sample(x, w, budget_s, seed=0, gpu_out=None):
    """Time the FP64 oracle (forward + backward) on seeded heads until the budget is spent.

    Returns (algorithmic FLOPs done, seconds, heads, errors vs the GPU outputs of the same heads).
    """
    from flashattention_bf16_fwd_b200.stats import lse_rel_err, max_rel_err, normwise_rel_err
    from oracle import attention_bwd, attention_fwd

    rng = np.random.default_rng(seed)
    order = rng.permutation(w.B * w.H)
    per_head = workload_flops(1, 1, w.N, w.d, w.causal)["total"]
    flops = secs = 0.0
    heads = []
    errs = {"o_max_abs": 0.0, "o_max_rel": 0.0, "lse_rel": 0.0, "dq_rel": 0.0, "dk_rel": 0.0, "dv_rel": 0.0}
    for idx in order:
        b, h = divmod(int(idx), w.H)
        sl = (slice(b, b + 1), slice(h, h + 1))
        xs = {n: x[n][sl] for n in ("q", "k", "v", "do")}
        t0 = time.perf_counter()
        o_ref, lse_ref = attention_fwd(xs["q"], xs["k"], xs["v"], w.causal, w.scale)
        grads = attention_bwd(xs["q"], xs["k"], xs["v"], xs["do"], w.causal, w.scale)
        secs += time.perf_counter() - t0
        flops += per_head
        heads.append((b, h))
        if gpu_out is not None:
            g = {n: t[sl].float().cpu().numpy() for n, t in gpu_out.items()}
            errs["o_max_abs"] = max(errs["o_max_abs"], float(np.abs(g["o"] - o_ref).max()))
            errs["o_max_rel"] = max(errs["o_max_rel"], max_rel_err(g["o"], o_ref))
            errs["lse_rel"] = max(errs["lse_rel"], lse_rel_err(g["lse"], lse_ref))
            for n, r in zip(("dq", "dk", "dv"), grads):
                errs[f"{n}_rel"] = max(errs[f"{n}_rel"], normwise_rel_err(g[n], r))
        if secs >= budget_s:
            break
    return flops, secs, heads, (errs if gpu_out is not None else None)


def run_reference(args, rank, world):
    """The FP64 CPU oracle as the reference arm, on bounded samples of the workload."""
    if rank != 0:
        return
    w = WORKLOADS[args.workload]
    x = make_inputs(w, seed=args.seed)
    per_step_budget = max(0.5, 60.0 / max(args.steps + args.warmup, 1))
    for _ in range(args.warmup):
        oracle_sample(x, w, per_step_budget / 4, seed=args.seed)
    flops = secs = 0.0
    heads = 0
    for i in range(args.steps):
        f, s, hs, _ = oracle_sample(x, w, per_step_budget, seed=args.seed + 1 + i)
        flops, secs, heads = flops + f, secs + s, heads + len(hs)
    value = flops / secs / 1e12
    cores = cpu_threads()
    sample = (f"{heads} (batch, head) pairs of {args.workload} over {args.steps} steps, "
              f"fwd+bwd FP64 NumPy oracle, ~{per_step_budget:.1f} s per step")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w, args),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(w, args):
    return {"workload": f"{w.name}: B={w.B} H={w.H} N={w.N} d={w.d} {'causal' if w.causal else 'full'}, "
                        f"{w.structure} inputs, fix_mode={args.fix_mode}",
            "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal, "fix_mode": args.fix_mode,
            "parallelism": "replicas", "l2": "flushed before every step (512 MiB write, outside the events)"}


KERNELS = ["fa_fwd_kernel", "fa_bwd_pre_kernel", "fa_bwd_kernel", "fa_bwd_dq_kernel"]
# nominal MUFU ex2 throughput of one SM (results per clock), for the bound the
# exponentials put on the d = 64 configurations
MUFU_EX2_PER_CLK_PER_SM = 16


def computed_tiles(N: int, causal: bool) -> int:
    """128 x 128 score tiles a head computes (causal: the key tiles up to the
    diagonal of each query tile, the diagonal's masked half included)."""
    n = (N + 127) // 128
    return n * (n + 1) // 2 if causal else n * n


def mufu_bound(w, sm_mhz: float, n_sms: int) -> dict:
    """TFLOP/s the exponentials allow if MUFU ex2 were the only limit: one
    exponential per computed score in the forward, one in the backward."""
    exps = computed_tiles(w.N, w.causal) * 128 * 128 * w.B * w.H
    rate = MUFU_EX2_PER_CLK_PER_SM * n_sms * sm_mhz * 1e6
    fl = workload_flops(w.B, w.H, w.N, w.d, w.causal)
    return {"fwd_tflops": fl["fwd"] / (exps / rate) / 1e12, "fwd_bwd_tflops": fl["total"] / (2 * exps / rate) / 1e12,
            "ex2_per_clk_per_sm": MUFU_EX2_PER_CLK_PER_SM, "sm_mhz": sm_mhz, "exps_per_pass": exps,
            "basis": "nominal MUFU rate x the SM clock sampled during the run"}


class Problem:
    """One workload's inputs and outputs resident on the device."""

    def __init__(self, fa, w, seed, dev, stream):
        self.fa, self.w, self.stream = fa, w, stream
        self.x = make_inputs(w, seed=seed)
        self.q, self.k, self.v, self.do = (self.x[n].to(dev) for n in ("q", "k", "v", "do"))
        self.o, self.dq, self.dk, self.dv = (torch.empty_like(self.q) for _ in range(4))
        self.lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
        self.ws = torch.empty(fa.fa_bwd_workspace_size(w.B, w.H, w.N, w.d), dtype=torch.uint8, device=dev)

    def step_api(self, fix):
        fa, w = self.fa, self.w
        check(fa.fa_fwd(self.q, self.k, self.v, self.o, self.lse, w.causal, w.scale, fix, self.stream), "fa_fwd")
        check(fa.fa_bwd(self.q, self.k, self.v, self.o, self.lse, self.do, self.dq, self.dk, self.dv, self.ws,
                        w.causal, w.scale, self.stream), "fa_bwd")

    def step_split(self, fix, ev):
        fa, w, s = self.fa, self.w, self.stream
        ev[0].record(s)
        check(fa.fa_fwd(self.q, self.k, self.v, self.o, self.lse, w.causal, w.scale, fix, s), "fa_fwd")
        ev[1].record(s)
        check(fa.fa_bwd_preprocess(self.o, self.do, self.ws, s), "fa_bwd_preprocess")
        ev[2].record(s)
        check(fa.fa_bwd_main(self.q, self.k, self.v, self.lse, self.do, self.dk, self.dv, self.ws, w.causal,
                             w.scale, s), "fa_bwd_main")
        ev[3].record(s)
        check(fa.fa_bwd_finish(self.dq, self.ws, w.scale, s), "fa_bwd_finish")
        ev[4].record(s)

    def free(self):
        for n in ("q", "k", "v", "do", "o", "dq", "dk", "dv", "lse", "ws"):
            setattr(self, n, None)


def check(rc, what):
    if rc != 0:
        from flashattention_bf16_fwd_b200 import fa
        raise RuntimeError(f"{what}: {fa.fa_status_string(rc)}")


def time_steps(pb, fix, steps, flush, stream):
    """Per-step times (ms): one event pair around fa_fwd + fa_bwd on the
    launching stream; with `flush`, a write larger than the L2 before each
    step, outside the events."""
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
    for i in range(steps):
        if flush is not None:
            flush.zero_()
        ev[i][0].record(stream)
        pb.step_api(fix)
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    return np.array([a.elapsed_time(b) for a, b in ev])


def time_kernels(pb, fix, steps, flush, stream):
    """Per-kernel times (ms, [steps, 4]): events between the four launches."""
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        pb.step_split(fix, ev[i])
    torch.cuda.synchronize()
    return np.array([[ev[i][j].elapsed_time(ev[i][j + 1]) for j in range(4)] for i in range(steps)])


def kernel_table(w, kern_ms, peaks, peak_kind):
    """Per-kernel times, rates and the roofline of the dominant kernel."""
    flops = workload_flops(w.B, w.H, w.N, w.d, w.causal)
    rows = w.B * w.H * w.N
    elem = rows * w.d
    work = {
        "fa_fwd_kernel": ("tensor", flops["fwd"]),
        "fa_bwd_pre_kernel": ("hbm", 2 * elem * 2 + rows * 4 + elem * 4),
        "fa_bwd_kernel": ("tensor", flops["bwd"]),
        "fa_bwd_dq_kernel": ("hbm", elem * 4 + elem * 2),
    }
    kernels = {}
    for name, ms in zip(KERNELS, kern_ms):
        bound, amount = work[name]
        rate = amount / (ms * 1e-3)
        kernels[name] = {"ms": float(ms), "share": float(ms / kern_ms.sum()),
                         ("TFLOP/s" if bound == "tensor" else "GB/s"): rate / (1e12 if bound == "tensor" else 1e9)}
    dom = KERNELS[int(np.argmax(kern_ms))]
    bound, amount = work[dom]
    ms = kern_ms[KERNELS.index(dom)]
    if bound == "tensor":
        achieved, peak, unit = amount / (ms * 1e-3) / 1e12, peaks["bf16_tflops"], "TFLOP/s"
    else:
        achieved, peak, unit = amount / (ms * 1e-3) / 1e9, peaks["hbm_gbs"], "GB/s"
    roofline = {"kernel": dom, "bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
                "frac": achieved / peak, "traffic": measured_traffic(dom, w), "peak_source": f"{peak_kind} burst",
                "algorithmic": amount,
                "timing": "mean of the kernel's event-bracketed launches in the per-kernel pass"}
    return kernels, roofline


def run_ours(args, rank, world, local):
    from flashattention_bf16_fwd_b200 import fa

    w = WORKLOADS[args.workload]
    dev = torch.device("cuda", local if world > 1 else 0)
    stream = torch.cuda.current_stream(dev)
    n_sms = torch.cuda.get_device_properties(dev).multi_processor_count
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    fix = args.fix_mode
    pb = Problem(fa, w, args.seed + rank, dev, stream)

    warm = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
    for _ in range(max(args.warmup, 0)):
        flush.zero_()
        pb.step_api(fix)
        flush.zero_()
        pb.step_split(fix, warm)
    torch.cuda.synchronize()
    check(fa.fa_check_device_error(), "warm-up")

    sampler = ClockSampler(local if world > 1 else 0)
    sampler.start()
    time.sleep(0.2)
    # timed pass: one event pair per step, the kernels of a step back to back
    outer = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    barrier(world)
    torch.cuda.synchronize()
    sampler.mark(True)
    outer[0].record(stream)
    step_ms = time_steps(pb, fix, args.steps, flush, stream)
    outer[1].record(stream)
    torch.cuda.synchronize()
    per = time_kernels(pb, fix, args.steps, flush, stream)
    warm_ms = time_steps(pb, fix, args.steps, None, stream)
    barrier(world)
    check(fa.fa_check_device_error(), "timed steps")

    t_rank = float(step_ms.sum())
    t_max = all_max(t_rank, world)
    outer_ms = all_max(outer[0].elapsed_time(outer[1]), world)
    flops = workload_flops(w.B, w.H, w.N, w.d, w.causal)
    value = replica_tflops(world, args.steps, flops["total"], t_max)
    peaks, peak_kind = load_peaks()
    kernels, roofline = kernel_table(w, per.mean(axis=0), peaks, peak_kind)

    # every other workload of the configuration list, same procedure
    per_config = {}
    names = [] if args.configs == "none" else [c for c in args.configs.split(",") if c]
    for name in names:
        if name == w.name:
            res = {"step_ms_flushed": float(np.median(step_ms)), "step_ms_warm": float(np.median(warm_ms)),
                   "steps": args.steps, "kern_ms": per.mean(axis=0), "workload": w}
        else:
            res = measure_config(fa, WORKLOADS[name], args, rank, dev, stream, flush)
        per_config[name] = res
    sampler.mark(False)
    clocks = sampler.stop()
    check(fa.fa_check_device_error(), "configurations")
    sm_mhz = clocks.get("sm_mhz") or 1965.0
    for name, res in per_config.items():
        cw = res.pop("workload")
        kern_ms = res.pop("kern_ms")
        fl = workload_flops(cw.B, cw.H, cw.N, cw.d, cw.causal)["total"]
        ktab, kroof = kernel_table(cw, kern_ms, peaks, peak_kind)
        res.update({
            "shape": f"B={cw.B} H={cw.H} N={cw.N} d={cw.d} {'causal' if cw.causal else 'full'}, {cw.structure}",
            "tflops_flushed": fl / (res["step_ms_flushed"] * 1e-3) / 1e12,
            "tflops_warm": fl / (res["step_ms_warm"] * 1e-3) / 1e12,
        })
        res["pct_of_measured_peak_flushed"] = res["tflops_flushed"] / peaks["bf16_tflops"] * 100.0
        res["pct_of_datasheet_peak_flushed"] = res["tflops_flushed"] / DATASHEET_BF16_TFLOPS * 100.0
        res["kernels"] = ktab
        res["roofline"] = kroof
        if cw.d == 64:
            res["mufu_bound"] = mufu_bound(cw, sm_mhz, n_sms)

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(fa, pb.x, w, args, dev, stream, flops["total"], world)

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": t_max / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": workload_config(w, args),
        "pct_of_peak": {"measured_burst": value / world / peaks["bf16_tflops"] * 100.0,
                        "datasheet": value / world / DATASHEET_BF16_TFLOPS * 100.0, "peak_source": peak_kind},
        "ms_per_step_bracket": outer_ms / args.steps,
        "ms_per_step_warm_l2": float(np.median(warm_ms)),
        "ms_per_step_kernel_sum": float(per.sum(axis=1).mean()),
        "roofline": roofline, "kernels": kernels, "gpu_launches": len(KERNELS) * args.steps,
        "clocks": clocks,
    }
    if w.d == 64:
        line["mufu_bound"] = mufu_bound(w, sm_mhz, n_sms)
    if per_config:
        line["per_config"] = per_config
    if e2e is not None:
        line["e2e"] = e2e
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        gout = {"o": pb.o, "lse": pb.lse, "dq": pb.dq, "dk": pb.dk, "dv": pb.dv}
        fl, secs, heads, errs = oracle_sample(pb.x, w, args.cpu_seconds, seed=args.seed, gpu_out=gout)
        line["cpu_baseline"] = {"value": fl / secs / 1e12, "unit": "TFLOP/s", "cores": cpu_threads(),
                                "kind": "oracle",
                                "sample": f"{len(heads)} of {w.B * w.H} (batch, head) pairs, FP64 NumPy "
                                          f"fwd+bwd, {secs:.1f} s; errors measured on the same heads"}
        line["max_err"] = errs
    if rank == 0:
        print(json.dumps(line), flush=True)


def measure_config(fa, w, args, rank, dev, stream, flush):
    """Median step time of workload w with the L2 flushed and warm, and its
    per-kernel times, each over a step count sized to about a second."""
    pb = Problem(fa, w, args.seed + rank, dev, stream)
    warm = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
    for _ in range(max(args.warmup, 3)):
        flush.zero_()
        pb.step_api(args.fix_mode)
        flush.zero_()
        pb.step_split(args.fix_mode, warm)
    torch.cuda.synchronize()
    est = max(warm[0].elapsed_time(warm[4]), 1e-3)
    steps = int(min(args.steps, max(10, 1000.0 / est)))
    flushed = time_steps(pb, args.fix_mode, steps, flush, stream)
    per = time_kernels(pb, args.fix_mode, steps, flush, stream)
    warm_ms = time_steps(pb, args.fix_mode, steps, None, stream)
    pb.free()
    torch.cuda.empty_cache()
    return {"step_ms_flushed": float(np.median(flushed)), "step_ms_warm": float(np.median(warm_ms)),
            "steps": steps, "kern_ms": per.mean(axis=0), "workload": w}


def measured_traffic(kernel, w):
    """DRAM bytes per launch from the committed ncu capture of this workload, if it matches this kernel build."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    import hashlib
    with open(path) as f:
        rec = json.load(f).get(kernel)
    if not rec:
        return None
    # the hash covers the sources the kernel is compiled from (all of csrc/
    # when the record names none)
    src = os.path.join(ROOT, "flashattention_bf16_fwd_b200", "csrc")
    files = rec.get("sources") or sorted(os.listdir(src))
    h = hashlib.sha256()
    for fn in files:
        with open(os.path.join(src, fn), "rb") as f:
            h.update(f.read())
    if rec.get("csrc_sha256") != h.hexdigest():
        return None
    per = rec.get("per_workload", {}).get(w.name)
    return per.get("dram_bytes_per_launch") if per else None


def run_e2e(fa, x, w, args, dev, stream, flops_total, world):
    """Same metric end to end through the C ABI: every step copies its inputs
    from pinned host memory to the device, runs fa_fwd + fa_bwd, and copies
    its outputs (O, LSE, dQ, dK, dV) back to pinned host memory.

    The steps are pipelined the way a training loop with a data loader runs:
    two device slots, the host-to-device copy of step k+1 on one stream and
    the device-to-host copy of step k-1 on another while step k's kernels run
    on the compute stream (PCIe carries both directions at once).  Every
    step's copies are inside the timed region; the clock runs from the first
    input copy to the last output copy."""
    # Each step's inputs sit in one pinned host buffer (q, k, v, dO back to
    # back, as a data loader would stage them) and its outputs (O, dQ, dK, dV,
    # LSE) in another, so that each direction is one copy.
    shape = (w.B, w.H, w.N, w.d)
    in_names = ("q", "k", "v", "do")
    out_names = ("o", "dq", "dk", "dv", "lse")
    nb = w.B * w.H * w.N * w.d * 2                   # bytes of one bf16 tensor (a multiple of 16)
    lse_bytes = w.B * w.H * w.N * 4

    def views(buf, names):
        out = {}
        for idx, n in enumerate(names):
            if n == "lse":
                out[n] = buf[idx * nb: idx * nb + lse_bytes].view(torch.float32).view(w.B, w.H, w.N)
            else:
                out[n] = buf[idx * nb:(idx + 1) * nb].view(torch.bfloat16).view(shape)
        return out

    host_in_buf = torch.empty(4 * nb, dtype=torch.uint8).pin_memory()
    host_in = views(host_in_buf, in_names)
    for n in in_names:
        host_in[n].copy_(x[n])
    slots = []
    for _ in range(2):
        dev_in = torch.empty(4 * nb, dtype=torch.uint8, device=dev)
        dev_out = torch.empty(4 * nb + lse_bytes, dtype=torch.uint8, device=dev)
        host_out = torch.empty(4 * nb + lse_bytes, dtype=torch.uint8).pin_memory()
        slots.append({
            "in_buf": dev_in, "in": views(dev_in, in_names),
            "out_buf": dev_out, "out": views(dev_out, out_names), "host_buf": host_out,
            "h2d": torch.cuda.Event(), "comp": torch.cuda.Event(), "d2h": torch.cuda.Event(),
            "used": False,
        })
    ws = torch.empty(fa.fa_bwd_workspace_size(*shape), dtype=torch.uint8, device=dev)
    h2d_stream = torch.cuda.Stream(device=dev)
    d2h_stream = torch.cuda.Stream(device=dev)

    def one(k):
        sl = slots[k % 2]
        with torch.cuda.stream(h2d_stream):
            if sl["used"]:
                h2d_stream.wait_event(sl["comp"])       # step k-2 has finished reading this slot's inputs
            sl["in_buf"].copy_(host_in_buf, non_blocking=True)
            sl["h2d"].record(h2d_stream)
        stream.wait_event(sl["h2d"])
        if sl["used"]:
            stream.wait_event(sl["d2h"])                # step k-2's outputs have left this slot
        i, o = sl["in"], sl["out"]
        rc = fa.fa_fwd(i["q"], i["k"], i["v"], o["o"], o["lse"], w.causal, w.scale, args.fix_mode, stream)
        rc |= fa.fa_bwd(i["q"], i["k"], i["v"], o["o"], o["lse"], i["do"], o["dq"], o["dk"], o["dv"], ws,
                        w.causal, w.scale, stream)
        if rc != 0:
            raise RuntimeError("e2e step failed")
        sl["comp"].record(stream)
        with torch.cuda.stream(d2h_stream):
            d2h_stream.wait_event(sl["comp"])
            sl["host_buf"].copy_(sl["out_buf"], non_blocking=True)
            sl["d2h"].record(d2h_stream)
        sl["used"] = True

    for k in range(4):
        one(k)
    torch.cuda.synchronize()
    # enough steps that the pipeline's fill (the first input copy alone) and
    # drain (the last output copy alone) weigh little against the steady state
    # (60 steps, about 75 ms, whatever --steps asks of the kernel timing)
    steps = 60
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    t0.record(h2d_stream)
    for k in range(steps):
        one(k)
    t1.record(d2h_stream)
    torch.cuda.synchronize()
    t = all_max(t0.elapsed_time(t1), world)
    h2d = host_in_buf.numel()
    d2h = slots[0]["host_buf"].numel()
    return {"value": replica_tflops(world, steps, flops_total, t), "unit": "TFLOP/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "ms_per_step": t / steps,
            "pipelining": "two device slots; step k+1's input copy and step k-1's output copy overlap step k; "
                          "one copy per direction (inputs and outputs each in one pinned buffer)"}


def main():
    args = parse_args()
    if args.impl == "reference":
        # the oracle runs on rank 0's host cores only; other ranks have no work
        run_reference(args, int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")))
        return
    rank, world, local = dist_setup(args.gpus)
    try:
        run_ours(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
