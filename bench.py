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
    "large_head_blocksparse": (4, 16, 4096, 128, False, "bf16", 1.0, "fwdbwd"),
    "large_head_fp8_fwd": (4, 16, 4096, 128, True, "bf16", 1.0, "fwd"),
    "large_head_linear": (4, 16, 4096, 128, True, "bf16", 1.0, "fwd"),
}
# Block-sparse workloads: density of the seeded 128 x 128 block mask (the
# diagonal is always marked, so no row is empty).
BLOCK_MASKS = {"large_head_blocksparse": 0.5}
# FP8-score workloads: each step quantises Q and K (rotated) and runs the
# forward with e4m3 scores.
FP8_WORKLOADS = {"large_head_fp8_fwd"}
# Causal linear attention workloads (chunked, three kernels per step).
LINEAR_WORKLOADS = {"large_head_linear"}
DESCRIPTION = {
    "tiny": "tiny exact attention fwd B=1 H=2 N=256 d=64 non-causal bf16",
    "bert_large": "BERT-large-shaped fwd B=8 H=16 N=512 d=64 non-causal bf16",
    "gpt2_causal": "GPT-2-shaped causal fwd+bwd B=8 H=12 N=1024 d=64 bf16",
    "long_day": "long single-sequence causal fwd B=1 H=12 N=23400 d=64 fp16 sigma=0.5",
    "large_head": "large-head causal fwd+bwd B=4 H=16 N=4096 d=128 bf16",
    "large_head_blocksparse": "block-sparse fwd+bwd B=4 H=16 N=4096 d=128 bf16, "
                              "half of the 128x128 blocks marked (seeded, diagonal kept)",
    "large_head_fp8_fwd": "FP8-score causal fwd B=4 H=16 N=4096 d=128 (Q, K rotated and quantised "
                          "to e4m3 in the step, P V in bf16)",
    "large_head_linear": "causal linear attention B=4 H=16 N=4096 d=128 bf16, chunks of 128 "
                         "(fused: per head and half of the value features, the chunks in order "
                         "with the state on chip; masked in-chunk product + Q S)",
}
METRIC = "attention fwd and fwd+bwd TFLOP/s on 1 B200; % of dense BF16 tensor peak"
L2_BYTES = 126 * 1024 * 1024


def flops(B, H, N, d, causal):
    f = 4.0 * B * H * N * N * d
    if causal:
        f /= 2
    return f, 2.5 * f  # forward, backward


def block_mask(N, density, seed=1):
    """Seeded (nb, nb) uint8 block mask with the diagonal marked."""
    nb = (N + 127) // 128
    m = (np.random.default_rng(seed).random((nb, nb)) < density).astype(np.uint8)
    np.fill_diagonal(m, 1)
    return m


def blocksparse_flops(B, H, N, d, mask):
    """Forward and backward FLOPs of the marked blocks (the same convention as
    flops(): 4 d per visible query-key pair forward, 10 d backward)."""
    sizes = np.minimum(128, N - 128 * np.arange(mask.shape[0]))
    pairs = float(sizes @ mask.astype(np.float64) @ sizes)
    f = 4.0 * B * H * d * pairs
    return f, 2.5 * f


def linear_flops(B, H, N, d, C=128):
    """Contractions of the chunked linear attention as computed: per chunk of
    C rows, Q K^T and P V (2 C^2 d each, the masked half included) and Q S and
    K^T V (2 C d^2 each)."""
    nc = (N + C - 1) // C
    return float(B * H * nc) * 4.0 * C * d * (C + d)


def workload_flops(wl):
    B, H, N, d, causal, _, _, _ = WORKLOADS[wl]
    if wl in LINEAR_WORKLOADS:
        return linear_flops(B, H, N, d), 0.0
    if wl in BLOCK_MASKS:
        return blocksparse_flops(B, H, N, d, block_mask(N, BLOCK_MASKS[wl]))
    return flops(B, H, N, d, causal)


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


def l2_text(working_set):
    """How a workload keeps L2 from serving its inputs between timed steps."""
    if working_set >= 2 * L2_BYTES:
        return "inputs larger than L2 (working set %.0f MB)" % (working_set / 1e6)
    return "L2 flushed between steps (256 MB write, outside the per-step events)"


def run_config(workload, passes, world):
    """The `config` object of a line, the same for both arms: the workload, its
    FLOPs per step and how it is measured on the GPU."""
    B, H, N, d, causal, _, _, default_passes = WORKLOADS[workload]
    f_fwd, f_bwd = workload_flops(workload)
    # device inputs (q, k, v, and dO for the backward) plus O, 16-bit each
    working_set = ((4 if passes == "fwdbwd" else 3) + 1) * B * H * N * d * 2
    return {
        "workload": DESCRIPTION[workload] + ("" if passes == default_passes else f" ({passes} only)"),
        "B": B, "H": H, "N": N, "d": d, "causal": causal, "passes": passes,
        "flop_per_step": f_fwd + (f_bwd if passes == "fwdbwd" else 0.0),
        "flop_convention": "fwd 4BHN^2d, bwd 10BHN^2d, halved when causal",
        "l2": l2_text(working_set),
        "timing": "ms_per_step = median over the timed steps of per-step CUDA events "
                  "(max over ranks); ms_bracket_mean = barrier-to-barrier events / steps",
        "parallelism": f"dp{world} (independent heads per rank, no collective)",
    }


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
        """Ends sampling; returns the csv text (None if nvidia-smi never ran)."""
        if self.proc is None:
            self.file.close()
            os.unlink(self.file.name)
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
        return text


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


def _device_tensors(wl, seed, dev, passes):
    """Seeded host inputs (pinned) and their device copies for workload `wl`."""
    import torch
    B, H, N, d, causal, dtype, sigma, _ = WORKLOADS[wl]
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float16
    arrs = synth.attention_inputs(B, H, N, d, seed=seed, sigma=sigma, dtype=dtype,
                                  with_dout=(passes == "fwdbwd"))
    pinned = []
    for a in arrs:
        t = torch.from_numpy(a.view(np.int16)).view(tdt) if dtype == "bf16" else torch.from_numpy(a)
        pinned.append(t.pin_memory())
    return pinned, [t.to(dev) for t in pinned]


class DeviceRun:
    """Buffers and one step (forward, then the backward's two phases) of a
    workload on one device, with CUDA events on the launching stream."""

    def __init__(self, wl, passes, seed, dev):
        import torch
        from io_aware_exact_30_b200 import attn
        self.attn = attn
        B, H, N, d, causal, dtype, sigma, _ = WORKLOADS[wl]
        self.wl, self.passes, self.causal, self.scale = wl, passes, causal, 1.0 / math.sqrt(d)
        self.shape = (B, H, N, d)
        self.pinned, self.dev_in = _device_tensors(wl, seed, dev, passes)
        self.q, self.k, self.v = self.dev_in[:3]
        self.do = self.dev_in[3] if passes == "fwdbwd" else None
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
        if passes == "fwdbwd":
            self.dq, self.dk, self.dv = (torch.empty_like(self.q) for _ in range(3))
            self.ws = torch.empty(attn.attn_bwd_workspace_bytes(B, H, N, d), dtype=torch.uint8,
                                  device=dev)
        self.working_set = sum(t.numel() * t.element_size() for t in self.dev_in) + \
            self.o.numel() * self.o.element_size()
        self.flush = None
        if self.working_set < 2 * L2_BYTES:
            self.flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
        self.fp8 = None
        if wl in FP8_WORKLOADS:
            nb = (N + 127) // 128
            self.fp8 = dict(
                q8=torch.empty((B, H, N, d), dtype=torch.uint8, device=dev),
                k8=torch.empty((B, H, N, d), dtype=torch.uint8, device=dev),
                qs=torch.empty((B, H, nb), dtype=torch.float32, device=dev),
                ks=torch.empty((B, H, nb), dtype=torch.float32, device=dev),
                signs=torch.from_numpy(synth.random_signs(d, seed)).to(dev))
        self.lin_ws = None
        if wl in LINEAR_WORKLOADS:
            self.lin_ws = torch.empty(attn.attn_linear_workspace_bytes(B, H, N, d),
                                      dtype=torch.uint8, device=dev)
        self.mask = None
        if wl in BLOCK_MASKS:
            self.mask = torch.from_numpy(block_mask(N, BLOCK_MASKS[wl])).to(dev)
        self.stream = torch.cuda.current_stream(dev)
        self.n_launch = 1 + (attn.bwd_launches(d) if passes == "fwdbwd" else 0)
        self.n_events = 4 if passes == "fwdbwd" else 2

    def l2_note(self):
        return l2_text(self.working_set)

    def step(self, evs=None):
        a, st = self.attn, self.stream
        if self.flush is not None:
            self.flush.zero_()
        if evs:
            evs[0].record(st)
        if self.lin_ws is not None:
            a.attn_linear_fwd(self.q, self.k, self.v, self.o, self.lin_ws, self.scale)
        elif self.fp8 is not None:
            f = self.fp8
            a.attn_fp8_quantize(self.q, f["q8"], f["qs"], f["signs"], True)
            a.attn_fp8_quantize(self.k, f["k8"], f["ks"], f["signs"], True)
            a.attn_fwd_fp8(f["q8"], f["k8"], f["qs"], f["ks"], self.v, self.o, self.lse,
                           self.causal, self.scale, True)
        elif self.mask is None:
            a.attn_fwd(self.q, self.k, self.v, self.o, self.lse, self.causal, self.scale)
        else:
            a.attn_fwd_blocksparse(self.q, self.k, self.v, self.o, self.lse, self.mask,
                                   self.causal, self.scale)
        if evs:
            evs[1].record(st)
        if self.passes == "fwdbwd":
            if self.mask is None:
                a.attn_bwd_prep(self.o, self.do, self.lse, self.ws)
                if evs:
                    evs[2].record(st)
                a.attn_bwd_main(self.q, self.k, self.v, self.do, self.dq, self.dk, self.dv,
                                self.ws, self.causal, self.scale)
            else:  # one call (prep + main): the prep share is timed with the main phase
                if evs:
                    evs[2].record(st)
                a.attn_bwd_blocksparse(self.q, self.k, self.v, self.o, self.lse, self.do, self.dq,
                                       self.dk, self.dv, self.ws, self.mask, self.causal,
                                       self.scale)
            if evs:
                evs[3].record(st)

    def events(self, steps):
        import torch
        return [[torch.cuda.Event(enable_timing=True) for _ in range(self.n_events)]
                for _ in range(steps)]

    @staticmethod
    def medians(per_step):
        """Median per-step times (ms): whole step, forward, backward prep, backward main."""
        med = lambda xs: statistics.median(xs) if xs else 0.0
        step = med([e[0].elapsed_time(e[-1]) for e in per_step])
        fwd = med([e[0].elapsed_time(e[1]) for e in per_step])
        prep = med([e[1].elapsed_time(e[2]) for e in per_step]) if len(per_step[0]) > 2 else 0.0
        main = med([e[2].elapsed_time(e[3]) for e in per_step]) if len(per_step[0]) > 2 else 0.0
        return step, fwd, prep, main


def roofline_entry(d, passes, f_fwd, f_bwd, fwd_ms, main_ms, traffic):
    """Roofline of the dominant kernel call: the backward main call (main kernel,
    plus the dQ conversion it launches at d = 128) when the backward runs, else
    the forward.  The peak is the measured burst bf16 rate: the kernels are timed
    over a timed region of milliseconds at full clock, not a seconds-long loop
    under the power cap (fp16 contractions run at the same tensor rate)."""
    burst, _, _, src = peaks()
    if passes == "fwdbwd":
        kern = (["attn_bwd_main128_kernel", "attn_bwd_dq_convert_kernel"] if d == 128
                else ["attn_bwd_main_kernel"])
        flop, ms = f_bwd, main_ms
    else:
        kern, flop, ms = ["attn_fwd_kernel"], f_fwd, fwd_ms
    achieved = flop / (ms * 1e-3) / 1e12
    return {
        "kernel": " + ".join(kern),
        "bound": "tensor",
        "achieved": round(achieved, 2),
        "peak": burst,
        "peak_kind": f"bf16_tflops burst ({src}); fp16 runs at the same tensor rate",
        "unit": "TFLOP/s",
        "frac": round(achieved / burst, 4),
        "traffic": traffic,
        "traffic_unit": "bytes per launch (ncu dram read+write; profiles/traffic.json)",
    }, kern


def side_workloads(args, dev, clocks):
    """Every other configuration, timed the same way (median of per-step CUDA
    events after warm-up, L2 flushed between steps when the inputs fit in L2);
    parity cases for the tests, reported here so each has a measured number."""
    import torch
    out = {}
    burst, _, _, _ = peaks()
    for wl in WORKLOADS:
        if wl == args.workload:
            continue
        B, H, N, d, causal, dtype, sigma, passes = WORKLOADS[wl]
        run = DeviceRun(wl, passes, args.seed, dev)
        for _ in range(max(3, args.warmup)):
            run.step()
        torch.cuda.synchronize()
        steps = max(20, min(args.steps, 50))
        per = run.events(steps)
        t0 = time.time()
        for i in range(steps):
            run.step(per[i])
        torch.cuda.synchronize()
        t1 = time.time()
        if run.attn.attn_last_device_status() != 0:
            raise RuntimeError(f"device status not OK after {wl}")
        step_ms, fwd_ms, prep_ms, main_ms = DeviceRun.medians(per)
        f_fwd, f_bwd = workload_flops(wl)
        f_step = f_fwd + (f_bwd if passes == "fwdbwd" else 0.0)
        roof, _ = roofline_entry(d, passes, f_fwd, f_bwd, fwd_ms, main_ms, None)
        roof.pop("traffic")
        roof.pop("traffic_unit")
        if wl in LINEAR_WORKLOADS:
            # memory-bound: Q, K, V read and O written once (algorithmic), against
            # the measured copy bandwidth (64 heads: the fused kernel, whose state
            # stays on chip)
            _, _, hbm, src = peaks()
            alg = 4.0 * B * H * N * d * 2
            roof = {"kernel": "linear_fused_kernel",
                    "bound": "hbm", "achieved": round(alg / (fwd_ms * 1e-3) / 1e9, 1),
                    "peak": hbm, "peak_kind": f"hbm_gbs ({src})", "unit": "GB/s",
                    "frac": round(alg / (fwd_ms * 1e-3) / 1e9 / hbm, 4),
                    "algorithmic_bytes": alg}
        if wl in FP8_WORKLOADS:
            # S = Q K^T (half the FLOPs) at the FP8 rate, twice the bf16 rate; P V at
            # bf16: the attainable peak for the mix is 4/3 of the bf16 peak
            roof["peak"] = round(burst * 4.0 / 3.0, 1)
            roof["peak_kind"] = ("bf16_tflops burst (measured) x 4/3: S at the nominal fp8/bf16 "
                                 "ratio of 2, P V at bf16; step includes the quantisation")
            roof["frac"] = round(roof["achieved"] / roof["peak"], 4)
        e = {
            "workload": DESCRIPTION[wl], "passes": passes, "steps": steps,
            "ms_per_step": round(step_ms, 4),
            "tflops": round(f_step / (step_ms * 1e-3) / 1e12, 2),
            "fwd_ms": round(fwd_ms, 4), "fwd_tflops": round(f_fwd / (fwd_ms * 1e-3) / 1e12, 2),
            "pct_of_2250_spec": round(100 * f_step / (step_ms * 1e-3) / 1e12 / 2250.0, 2),
            "frac_of_measured_burst": round(f_step / (step_ms * 1e-3) / 1e12 / burst, 4),
            "roofline": roof, "l2": run.l2_note(),
        }
        if passes == "fwdbwd":
            e["bwd_prep_ms"] = round(prep_ms, 4)
            e["bwd_main_ms"] = round(main_ms, 4)
            e["bwd_tflops"] = round(f_bwd / ((prep_ms + main_ms) * 1e-3) / 1e12, 2)
        e["clocks_window"] = [t0, t1]
        out[wl] = e
        del run
        torch.cuda.empty_cache()
    return out


def profile_workload(args):
    """One workload's steps alone, on cuda:0: W warm-up and K timed steps."""
    import torch
    wl = args.profile_workload
    passes = WORKLOADS[wl][7]
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    run = DeviceRun(wl, passes, args.seed, dev)
    for _ in range(args.warmup):
        run.step()
    per = run.events(args.steps)
    for i in range(args.steps):
        run.step(per[i])
    torch.cuda.synchronize()
    if run.attn.attn_last_device_status() != 0:
        raise RuntimeError("device status not OK")
    step_ms = DeviceRun.medians(per)[0]
    return {"workload": DESCRIPTION[wl], "steps": args.steps, "ms_per_step": round(step_ms, 4)}


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    B, H, N, d, causal, dtype, sigma, passes = WORKLOADS[args.workload]
    if args.passes:
        passes = args.passes
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    run = DeviceRun(args.workload, passes, rank_seed(args.seed, rank), dev)
    attn = run.attn

    for _ in range(args.warmup):
        run.step()
    torch.cuda.synchronize()
    if attn.attn_last_device_status() != 0:
        raise RuntimeError("device status not OK after warm-up")

    clocks = ClockSampler(local_rank)
    if rank == 0:
        clocks.start()
    per_step = run.events(args.steps)
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.mark(True)
    t_start.record(run.stream)
    for i in range(args.steps):
        run.step(per_step[i])
    t_end.record(run.stream)
    torch.cuda.synchronize()
    clocks.mark(False)
    if world > 1:
        dist.barrier()
    status = attn.attn_last_device_status()
    bracket_ms = t_start.elapsed_time(t_end)
    step_ms, fwd_ms, prep_ms, main_ms = DeviceRun.medians(per_step)

    # whole-job time per step = slowest rank's median step
    max_step_ms = reduce_max(step_ms, world, dev)
    max_bracket_ms = reduce_max(bracket_ms, world, dev)

    # ---- end to end through the public API with host buffers -------------
    # attn_sdpa_host: the inputs come from pinned host memory and the results
    # go back there inside the call, chunk by chunk over heads with copies in,
    # kernels and copies out overlapped on the library's internal streams.
    e2e_steps = max(3, min(args.steps, 20))
    pinned = run.pinned
    host_out = [torch.empty_like(pinned[0]).pin_memory() for _ in range(3 if passes == "fwdbwd" else 1)]
    host_lse = torch.empty((B, H, N), dtype=torch.float32).pin_memory()
    with_bwd = passes == "fwdbwd"
    scratch = torch.empty(attn.attn_sdpa_host_scratch_bytes(B, H, N, d, with_bwd),
                          dtype=torch.uint8, device=dev)

    def e2e_step():
        if with_bwd:
            attn.attn_sdpa_host(pinned[0], pinned[1], pinned[2], pinned[3], None, None,
                                host_out[0], host_out[1], host_out[2], scratch, causal, run.scale)
        else:
            attn.attn_sdpa_host(pinned[0], pinned[1], pinned[2], None, host_out[0], host_lse,
                                None, None, None, scratch, causal, run.scale)

    e2e_step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(run.stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(run.stream)
    torch.cuda.synchronize()
    e2e_ms = reduce_max(e0.elapsed_time(e1) / e2e_steps, world, dev)
    h2d = sum(t.numel() * t.element_size() for t in pinned)
    d2h = sum(t.numel() * t.element_size() for t in host_out) + (
        0 if with_bwd else host_lse.numel() * 4)
    del scratch
    if attn.attn_last_device_status() != 0 or status != 0:
        raise RuntimeError("device status not OK after timing")
    l2_note = run.l2_note()
    del run
    torch.cuda.empty_cache()

    if rank != 0:
        clocks.stop()
        return None
    others = side_workloads(args, dev, clocks) if (world == 1 and not args.headline_only) else None
    clocks_text = clocks.stop()
    clk = parse_clock_samples(clocks_text, clocks.t0, clocks.t1) if clocks_text is not None else None
    if others:
        for e in others.values():
            t0, t1 = e.pop("clocks_window")
            if clocks_text is not None:
                e["clocks"] = parse_clock_samples(clocks_text, t0, t1)

    f_fwd, f_bwd = workload_flops(args.workload)
    f_step = f_fwd + (f_bwd if passes == "fwdbwd" else 0.0)
    config = run_config(args.workload, passes, world)
    config["l2"] = l2_note  # the run's own buffers (the same sizes run_config counts)
    value = job_tflops(f_step, world, max_step_ms)
    burst, sustained, hbm, src = peaks()
    roof, kern = roofline_entry(d, passes, f_fwd, f_bwd, fwd_ms, main_ms, None)
    roof["traffic"] = kernel_traffic(kern) if args.workload == "large_head" else None
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(max_step_ms, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": dtype,
        "data": "synthetic (seeded splitmix64/Box-Muller, N(0, sigma^2), rounded to %s)" % dtype,
        "config": config,
        "ms_bracket_mean": round(max_bracket_ms / args.steps, 4),
        "fwd_tflops": round(f_fwd / (fwd_ms * 1e-3) / 1e12, 2),
        "fwd_ms": round(fwd_ms, 4),
        "pct_of_2250_spec": round(100 * value / world / 2250.0, 2),
        "pct_of_measured_burst": round(100 * value / world / burst, 2),
        "roofline": roof,
        "e2e": {"value": round(job_tflops(f_step, world, e2e_ms), 2), "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(e2e_ms, 4),
                "api": "attn_sdpa_host (pinned host buffers in and out, copies inside the call)"},
        "gpu_launches": (1 + (attn.bwd_launches(d) if passes == "fwdbwd" else 0)) * args.steps,
        "clocks": clk,
    }
    if passes == "fwdbwd":
        line["bwd_prep_ms"] = round(prep_ms, 4)
        line["bwd_main_ms"] = round(main_ms, 4)
        line["bwd_tflops"] = round(f_bwd / ((prep_ms + main_ms) * 1e-3) / 1e12, 2)
    if others is not None:
        line["workloads"] = others
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.workload, passes, args.cpu_seconds)
        if others is not None:
            for wl in ("tiny", "bert_large"):
                if wl in others:
                    others[wl]["cpu_baseline_1thread"] = cpu_baseline(wl, "fwd", 3.0, threads=1)
    return line


def cpu_baseline(workload, passes, budget_s, threads=None):
    """The fp64 oracle as it stands, on the host cores (or `threads` of them), on
    a bounded sample."""
    import oracle
    if threads is not None:
        prev = oracle.num_threads()
        oracle.set_num_threads(threads)
        try:
            return cpu_baseline(workload, passes, budget_s)
        finally:
            oracle.set_num_threads(prev)
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
        reps, t0 = 0, time.time()
        while True:  # repeat small samples until at least a second has passed
            oracle.fwd_rows(*f64[:3], causal, scale, rows)
            reps += 1
            dt = time.time() - t0
            if dt >= min(1.0, budget_s):
                break
        fl = reps * 4.0 * d * float(np.sum(rows + 1 if causal else np.full(rows.size, N)))
        sample = (f"{rows.size} query rows of one head, fp64 two-pass forward"
                  + (f", repeated {reps} times" if reps > 1 else ""))
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
        "ms_per_step": round(ms, 3),
        # ms_per_step is the whole workload at the sampled rate; each timed step
        # ran one bounded sample of it, which took this long
        "sample_ms_per_step": round(1e3 * statistics.mean(v["seconds"] for v in vals), 1),
        "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": run_config(args.workload, passes, world),
        "cpu_baseline": cb,
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="large_head",
                    choices=sorted(w for w in WORKLOADS if w not in BLOCK_MASKS
                                   and w not in FP8_WORKLOADS and w not in LINEAR_WORKLOADS))
    ap.add_argument("--passes", choices=["fwd", "fwdbwd"], default=None)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--headline-only", action="store_true",
                    help="skip the other workloads (timed after the headline at N=1)")
    ap.add_argument("--profile-workload", default=None, choices=sorted(WORKLOADS),
                    help="run only this workload's steps (for a profiler) and print their "
                         "median time; no end-to-end leg, no CPU baseline")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    if args.profile_workload:
        print(json.dumps(profile_workload(args)), flush=True)
        return
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
