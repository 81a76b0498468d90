#!/usr/bin/env python
"""Benchmark of the exact-attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one pass of the whole path over one batch of synthetic input:
the forward (O, LSE) and the recompute backward (D preprocess, dQ/dK/dV) on
the large-head causal workload B=4, H=16, N=4096, d=128, bf16 (unless
--workload picks another; forward-only workloads time the forward alone).
The metric is algorithmic TFLOP/s: forward 4*B*H*N^2*d, backward
10*B*H*N^2*d (five contractions including the S recompute), both halved
under the causal mask; fwd+bwd is 14*B*H*N^2*d (halved).

Under torchrun each rank runs its own full workload instance (weak scaling,
no collective on the data path: every head is independent); the value is the
sum of all ranks' work over the slowest rank's device time.

``--impl reference`` times the fp64 CPU oracle (the only reference this path
has) on a bounded sample of the same workload, on the host cores.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from io_aware_exact_30_b200 import synth  # noqa: E402

WORKLOADS = {
    # name: (B, H, N, d, causal, dtype, sigma, passes)
    "tiny": (1, 2, 256, 64, False, "bf16", 1.0, "fwd"),
    "bert_large": (8, 16, 512, 64, False, "bf16", 1.0, "fwd"),
    "gpt2_causal": (8, 12, 1024, 64, True, "bf16", 1.0, "fwdbwd"),
    "long_day": (1, 12, 23400, 64, True, "fp16", 0.5, "fwd"),
    "large_head": (4, 16, 4096, 128, True, "bf16", 1.0, "fwdbwd"),
}
DESCRIPTION = {
    "tiny": "tiny exact attention fwd B=1 H=2 N=256 d=64 non-causal bf16",
    "bert_large": "BERT-large-shaped fwd B=8 H=16 N=512 d=64 non-causal bf16",
    "gpt2_causal": "GPT-2-shaped causal fwd+bwd B=8 H=12 N=1024 d=64 bf16",
    "long_day": "long single-sequence causal fwd B=1 H=12 N=23400 d=64 fp16 sigma=0.5",
    "large_head": "large-head causal fwd+bwd B=4 H=16 N=4096 d=128 bf16",
}
METRIC = "attention fwd and fwd+bwd TFLOP/s on 1 B200; % of dense BF16 tensor peak"
L2_BYTES = 126 * 1024 * 1024


def flops(B, H, N, d, causal):
    f = 4.0 * B * H * N * N * d
    if causal:
        f /= 2
    return f, 2.5 * f  # forward, backward


def kernel_traffic(kernels):
    """DRAM bytes per launch, summed over `kernels`, from profiles/traffic.json; None
    when any of them is missing or its sources have changed since those counters
    were taken."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        table = json.load(f)
    total = 0
    for kernel in kernels:
        entry = table.get(kernel)
        if not entry:
            return None
        m = hashlib.sha1()
        for src in entry["sources"]:
            with open(os.path.join(ROOT, src), "rb") as f:
                m.update(f.read())
        if m.hexdigest() != entry["source_sha1"]:
            return None
        total += entry["dram_bytes_read"] + entry["dram_bytes_write"]
    return total


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return j["bf16_tflops"], j["bf16_tflops_sustained"], j["hbm_gbs"], "measured"
    return 1590.0, 1400.0, 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons around the timed region."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.proc = None
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.file, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.5)

    def mark(self, begin):
        if begin:
            self.t0 = time.time()
        else:
            self.t1 = time.time()

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.2)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        text = self.file.read()
        os.unlink(self.file.name)
        return parse_clock_samples(text, self.t0, self.t1)


def parse_clock_samples(text, t0, t1):
    """Summary of `nvidia-smi --query-gpu=<ClockSampler.FIELDS>` csv lines: the
    median SM clock over the samples taken within a second of [t0, t1] (all
    samples if none is), the max clock, and every throttle reason seen active
    in that window."""
    mhz, mx, reasons, all_mhz = [], None, set(), []
    names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    for line in text.splitlines():
        parts = [x.strip() for x in line.split(",")]
        if len(parts) < 10:
            continue
        try:
            ts = time.mktime(time.strptime(parts[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
            sm, smx = float(parts[2]), float(parts[3])
        except ValueError:
            continue
        all_mhz.append(sm)
        mx = smx
        if t0 is not None and t1 is not None and t0 - 1 <= ts <= t1 + 1:
            mhz.append(sm)
            for n, v in zip(names, parts[6:10]):
                if v.lower() == "active":
                    reasons.add(n)
    src = mhz or all_mhz
    return {"sm_mhz": statistics.median(src) if src else None, "sm_max_mhz": mx,
            "reasons": sorted(reasons), "samples": len(mhz)}


def rank_seed(seed: int, rank: int) -> int:
    """Each rank draws its own instance of the workload (weak scaling)."""
    return seed + rank


def reduce_max(value: float, world: int, device=None) -> float:
    """Max of a per-rank scalar over all ranks (the job is as slow as its slowest rank)."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(flop_per_rank_step: float, world: int, max_ms_per_step: float) -> float:
    """Whole-job throughput: every rank's work over the slowest rank's time."""
    return world * flop_per_rank_step / (max_ms_per_step * 1e-3) / 1e12


def host_inputs(wl, seed):
    B, H, N, d, causal, dtype, sigma, passes = WORKLOADS[wl]
    arrs = synth.attention_inputs(B, H, N, d, seed=seed, sigma=sigma, dtype=dtype,
                                  with_dout=(passes == "fwdbwd"))
    return arrs


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from io_aware_exact_30_b200 import attn

    B, H, N, d, causal, dtype, sigma, passes = WORKLOADS[args.workload]
    if args.passes:
        passes = args.passes
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float16
    scale = 1.0 / math.sqrt(d)

    arrs = host_inputs(args.workload, seed=rank_seed(args.seed, rank))
    pinned = []
    for a in arrs:
        t = torch.from_numpy(a.view(np.int16)).view(tdt) if dtype == "bf16" else torch.from_numpy(a)
        pinned.append(t.pin_memory())
    dev_in = [t.to(dev) for t in pinned]
    q, k, v = dev_in[:3]
    do = dev_in[3] if passes == "fwdbwd" else None
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    if passes == "fwdbwd":
        dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
        ws = torch.empty(attn.attn_bwd_workspace_bytes(B, H, N, d), dtype=torch.uint8, device=dev)
    working_set = sum(t.numel() * t.element_size() for t in dev_in) + o.numel() * 2
    flush = None
    if working_set < 2 * L2_BYTES:
        flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)

    stream = torch.cuda.current_stream(dev)
    n_launch = {"fwd": 1, "fwdbwd": 1 + attn.bwd_launches(d)}[passes]

    def step(evs=None):
        if flush is not None:
            flush.zero_()
        if evs:
            evs[0].record(stream)
        attn.attn_fwd(q, k, v, o, lse, causal, scale)
        if evs:
            evs[1].record(stream)
        if passes == "fwdbwd":
            attn.attn_bwd_prep(o, do, lse, ws)
            if evs:
                evs[2].record(stream)
            attn.attn_bwd_main(q, k, v, do, dq, dk, dv, ws, causal, scale)
            if evs:
                evs[3].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if attn.attn_last_device_status() != 0:
        raise RuntimeError("device status not OK after warm-up")

    clocks = ClockSampler(local_rank)
    if rank == 0:
        clocks.start()
    per_step = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.mark(True)
    t_start.record(stream)
    for i in range(args.steps):
        step(per_step[i])
    t_end.record(stream)
    torch.cuda.synchronize()
    clocks.mark(False)
    if world > 1:
        dist.barrier()
    status = attn.attn_last_device_status()
    total_ms = t_start.elapsed_time(t_end)
    fwd_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in per_step)
    prep_ms = main_ms = 0.0
    if passes == "fwdbwd":
        prep_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in per_step)
        main_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in per_step)

    # whole-job time = slowest rank
    max_ms = reduce_max(total_ms, world, dev)
    clk = clocks.stop() if rank == 0 else None

    # ---- end to end through the public API with host buffers -------------
    e2e_steps = max(3, min(args.steps, 20))
    host_out = [torch.empty_like(pinned[0]).pin_memory() for _ in range(3 if passes == "fwdbwd" else 1)]
    host_lse = torch.empty((B, H, N), dtype=torch.float32).pin_memory()

    def e2e_step():
        for src, dst in zip(pinned, dev_in):
            dst.copy_(src, non_blocking=True)
        attn.attn_fwd(q, k, v, o, lse, causal, scale)
        if passes == "fwdbwd":
            attn.attn_bwd(q, k, v, o, lse, do, dq, dk, dv, ws, causal, scale)
            for src, dst in zip((dq, dk, dv), host_out):
                dst.copy_(src, non_blocking=True)
        else:
            host_out[0].copy_(o, non_blocking=True)
            host_lse.copy_(lse, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = reduce_max(e0.elapsed_time(e1) / e2e_steps, world, dev)
    h2d = sum(t.numel() * t.element_size() for t in pinned)
    d2h = sum(t.numel() * t.element_size() for t in host_out) + (
        0 if passes == "fwdbwd" else host_lse.numel() * 4)
    if attn.attn_last_device_status() != 0 or status != 0:
        raise RuntimeError("device status not OK after timing")

    if rank != 0:
        return None
    f_fwd, f_bwd = flops(B, H, N, d, causal)
    f_step = f_fwd + (f_bwd if passes == "fwdbwd" else 0.0)
    ms_step = max_ms / args.steps
    value = job_tflops(f_step, world, ms_step)
    burst, sustained, hbm, src = peaks()
    # The backward-main call launches, for d = 128, the main kernel and then the dQ
    # conversion; they are timed together and their traffic is summed.
    if passes == "fwdbwd":
        dom = (["attn_bwd_main128_kernel", "attn_bwd_dq_convert_kernel"] if d == 128
               else ["attn_bwd_main_kernel"], f_bwd, main_ms)
    else:
        dom = (["attn_fwd_kernel"], f_fwd, fwd_ms)
    traffic = kernel_traffic(dom[0]) if args.workload == "large_head" else None
    achieved = dom[1] / (dom[2] * 1e-3) / 1e12
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": dtype,
        "data": "synthetic (seeded splitmix64/Box-Muller, N(0, sigma^2), rounded to %s)" % dtype,
        "config": {
            "workload": DESCRIPTION[args.workload] + ("" if passes == WORKLOADS[args.workload][7] else f" ({passes} only)"),
            "B": B, "H": H, "N": N, "d": d, "causal": causal, "passes": passes,
            "flop_per_step": f_step,
            "flop_convention": "fwd 4BHN^2d, bwd 10BHN^2d, halved when causal",
            "l2": "inputs larger than L2 (working set %.0f MB)" % (working_set / 1e6)
            if flush is None else "L2 flushed between steps (256 MB write)",
            "parallelism": f"dp{world} (independent heads per rank, no collective)",
        },
        "fwd_tflops": round(f_fwd / (fwd_ms * 1e-3) / 1e12, 2),
        "fwd_ms": round(fwd_ms, 4),
        "pct_of_2250_spec": round(100 * value / world / 2250.0, 2),
        "pct_of_measured_burst": round(100 * value / world / burst, 2),
        "pct_of_measured_sustained": round(100 * value / world / sustained, 2),
        "roofline": {
            "kernel": " + ".join(dom[0]),
            "bound": "tensor",
            "achieved": round(achieved, 2),
            "peak": sustained,
            "peak_kind": f"bf16_tflops_sustained ({src})",
            "unit": "TFLOP/s",
            "frac": round(achieved / sustained, 4),
            "traffic": traffic,
            "traffic_unit": "bytes per launch (ncu dram read+write; profiles/traffic.json)",
        },
        "e2e": {"value": round(job_tflops(f_step, world, e2e_ms), 2), "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(e2e_ms, 4)},
        "gpu_launches": n_launch * args.steps,
        "clocks": clk,
    }
    if passes == "fwdbwd":
        line["bwd_prep_ms"] = round(prep_ms, 4)
        line["bwd_main_ms"] = round(main_ms, 4)
        line["bwd_tflops"] = round(f_bwd / ((prep_ms + main_ms) * 1e-3) / 1e12, 2)
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.workload, passes, args.cpu_seconds)
    return line


def cpu_baseline(workload, passes, budget_s):
    """The fp64 oracle as it stands, on the host cores, on a bounded sample."""
    import oracle
    B, H, N, d, causal, dtype, sigma, _ = WORKLOADS[workload]
    scale = 1.0 / math.sqrt(d)
    arrs = synth.attention_inputs(1, 1, N, d, seed=0, sigma=sigma, dtype=dtype, with_dout=True)
    f64 = [synth.to_f64(a, dtype) for a in arrs]
    cores = oracle.num_threads()
    if passes == "fwdbwd":
        # one head, a prefix of rows sized to the budget; rows i < R of a causal head
        # cost sum_{i<R} (i+1) key visits; algorithmic flops counted the same way
        t0 = time.time()
        R = min(N, 256)
        rows = np.arange(R)
        oracle.fwd_rows(*f64[:3], causal, scale, rows)
        probe = time.time() - t0
        # full head fwd+bwd via the oracle's backward (it recomputes the forward)
        visits_head = N * (N + 1) / 2 if causal else N * N
        visits_probe = R * (R + 1) / 2 if causal else R * N
        est = probe * visits_head / visits_probe * 3.5
        if est < budget_s * 1.5:
            t0 = time.time()
            oracle.bwd_heads(*f64, causal, scale, heads=[0])
            dt = time.time() - t0
            fl = 14.0 * visits_head * d
            sample = f"one head (N={N}, d={d}, {'causal' if causal else 'full'}) fwd+bwd in fp64"
        else:
            # rows prefix of the backward is not separable; time the forward on a row sample
            nrows = max(1, int(R * budget_s / max(probe, 1e-6) / 3.5))
            rows = np.linspace(0, N - 1, min(N, nrows)).astype(np.int64)
            t0 = time.time()
            oracle.fwd_rows(*f64[:3], causal, scale, rows)
            dt = time.time() - t0
            fl = 4.0 * d * float(np.sum(rows + 1 if causal else np.full(rows.size, N)))
            sample = f"{rows.size} forward rows of one head (fwd only; bwd too slow)"
    else:
        rows_all = N
        t0 = time.time()
        rows = np.arange(min(N, 64))
        oracle.fwd_rows(*f64[:3], causal, scale, rows)
        probe = max(time.time() - t0, 1e-6)
        per_row = probe / rows.size
        nrows = int(min(rows_all, max(64, budget_s / per_row)))
        rows = np.linspace(0, N - 1, nrows).astype(np.int64)
        t0 = time.time()
        oracle.fwd_rows(*f64[:3], causal, scale, rows)
        dt = time.time() - t0
        fl = 4.0 * d * float(np.sum(rows + 1 if causal else np.full(rows.size, N)))
        sample = f"{rows.size} query rows of one head, fp64 two-pass forward"
    return {"value": round(fl / dt / 1e12, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": sample, "seconds": round(dt, 2)}


def run_reference(args, rank, world):
    """--impl reference: the fp64 oracle on host cores (rank 0 only)."""
    if rank != 0:
        return None
    B, H, N, d, causal, dtype, sigma, passes = WORKLOADS[args.workload]
    if args.passes:
        passes = args.passes
    per_step = max(2.0, 60.0 / max(1, args.steps + args.warmup))
    vals = []
    for i in range(args.warmup + args.steps):
        cb = cpu_baseline(args.workload, passes, per_step)
        if i >= args.warmup:
            vals.append(cb)
    value = statistics.mean(v["value"] for v in vals)
    cb = dict(vals[-1])
    cb["value"] = round(value, 6)
    f_fwd, f_bwd = flops(B, H, N, d, causal)
    f_step = f_fwd + (f_bwd if passes == "fwdbwd" else 0.0)
    ms = f_step / (value * 1e12) * 1e3
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": DESCRIPTION[args.workload], "B": B, "H": H, "N": N, "d": d,
                   "causal": causal, "passes": passes},
        "cpu_baseline": cb,
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="large_head", choices=sorted(WORKLOADS))
    ap.add_argument("--passes", choices=["fwd", "fwdbwd"], default=None)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    import datetime

    import torch.distributed as dist
    if world > 1:
        import torch
        torch.cuda.set_device(local_rank)
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=None)
    try:
        line = run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            dist.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
