"""Host-side logic of bench.py, on the CPU: the FLOP convention against FLOP
counts worked out by hand for the five workloads, the traffic lookup and its
invalidation when a kernel source changes, clock-sample parsing, and the
weak-scaling helpers."""

import json
import os
import shutil
import sys
import time

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402

# (B, H, N, d, causal, forward GFLOP, fwd+bwd GFLOP or None), worked out by hand
# to three significant digits (4 B H N^2 d forward, x 3.5 with the backward,
# halved when causal)
TABLE = [
    (1, 2, 256, 64, False, 0.0336, None),
    (8, 16, 512, 64, False, 8.59, None),
    (8, 12, 1024, 64, True, 12.9, 45.1),
    (1, 12, 23400, 64, True, 841.0, None),
    (4, 16, 4096, 128, True, 275.0, 962.0),
]


@pytest.mark.parametrize("B,H,N,d,causal,gf,gfb", TABLE)
def test_flops_match_the_table(B, H, N, d, causal, gf, gfb):
    f, fb = bench.flops(B, H, N, d, causal)
    assert f / 1e9 == pytest.approx(gf, rel=2e-3)
    if gfb is not None:
        assert (f + fb) / 1e9 == pytest.approx(gfb, rel=2e-3)


def test_blocksparse_flops():
    # all blocks marked: the dense non-causal count; a ragged tail counts its
    # real rows and keys only; one 128 x 60 block by hand
    import numpy as np
    f, fb = bench.blocksparse_flops(2, 3, 700, 64, np.ones((6, 6), np.uint8))
    assert (f, fb) == bench.flops(2, 3, 700, 64, False)
    m = np.zeros((6, 6), np.uint8)
    m[1, 5] = 1
    assert bench.blocksparse_flops(1, 1, 700, 64, m)[0] == 4.0 * 64 * 128 * 60
    assert bench.block_mask(4096, 0.5).diagonal().all()


def test_workloads_cover_the_five_configs():
    shapes = {(w[0], w[1], w[2], w[3], w[4]) for w in bench.WORKLOADS.values()}
    for B, H, N, d, causal, _, _ in TABLE:
        assert (B, H, N, d, causal) in shapes


def _copy_tree(dst):
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        table = json.load(f)
    os.makedirs(os.path.join(dst, "profiles"))
    shutil.copy(os.path.join(ROOT, "profiles", "traffic.json"), os.path.join(dst, "profiles"))
    for entry in table.values():
        if isinstance(entry, dict):
            for src in entry["sources"]:
                os.makedirs(os.path.dirname(os.path.join(dst, src)), exist_ok=True)
                shutil.copy(os.path.join(ROOT, src), os.path.join(dst, src))
    return table


def test_traffic_is_summed_and_dropped_when_a_source_changes(tmp_path, monkeypatch):
    import hashlib
    table = _copy_tree(str(tmp_path))
    # stamp the copy with the hashes of the copied sources, as a capture does
    for entry in table.values():
        if isinstance(entry, dict):
            m = hashlib.sha1()
            for src in entry["sources"]:
                with open(os.path.join(str(tmp_path), src), "rb") as f:
                    m.update(f.read())
            entry["source_sha1"] = m.hexdigest()
    with open(os.path.join(str(tmp_path), "profiles", "traffic.json"), "w") as f:
        json.dump(table, f)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    names = [k for k in table if not k.startswith("_")]
    want = sum(table[k]["dram_bytes_read"] + table[k]["dram_bytes_write"] for k in names)
    assert bench.kernel_traffic(names) == want
    assert bench.kernel_traffic(names + ["no_such_kernel"]) is None
    src = os.path.join(str(tmp_path), table[names[0]]["sources"][-1])
    with open(src, "a") as f:
        f.write("\n// changed\n")
    assert bench.kernel_traffic(names[:1]) is None


def test_clock_samples_window_median_and_reasons():
    t0 = time.mktime(time.strptime("2026/01/01 10:00:10", "%Y/%m/%d %H:%M:%S"))
    t1 = t0 + 5

    def line(sec, mhz, cap="Not Active", therm="Not Active"):
        return (f"2026/01/01 10:00:{sec:02d}.123, 0, {mhz}, 1965, 900.0, 0x4, "
                f"Not Active, Not Active, {therm}, {cap}")
    text = "\n".join([
        line(2, 500, therm="Active"),         # before the window: ignored
        line(10, 1965), line(12, 1900, cap="Active"), line(14, 1950),
        line(30, 300, therm="Active"),        # after the window: ignored
        "garbage line",
    ])
    got = bench.parse_clock_samples(text, t0, t1)
    assert got["sm_mhz"] == 1950 and got["sm_max_mhz"] == 1965
    assert got["reasons"] == ["sw_power_cap"] and got["samples"] == 3
    assert bench.parse_clock_samples("", t0, t1)["sm_mhz"] is None


def test_weak_scaling_helpers():
    # whole-job TFLOP/s: every rank's FLOPs over the slowest rank's time
    assert bench.job_tflops(1e12, 4, 2.0) == pytest.approx(2000.0)
    assert len({bench.rank_seed(7, r) for r in range(8)}) == 8


def test_reference_arm_line():
    """--impl reference: the oracle times a bounded sample on the host (rank 0
    only) and the line carries the contract's keys."""
    import argparse
    args = argparse.Namespace(workload="tiny", passes=None, steps=1, warmup=3)
    assert bench.run_reference(args, 1, 2) is None
    line = bench.run_reference(args, 0, 1)
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC
    assert line["value"] > 0 and line["unit"] == "TFLOP/s" and line["higher_is_better"]
    assert line["ms_per_step"] > 0 and line["sample_ms_per_step"] > 0
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"]
    assert cb["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": "TFLOP/s",
                           "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    # the same config object as the GPU arm's line for this workload
    assert line["config"] == bench.run_config("tiny", bench.WORKLOADS["tiny"][7], 1)


def test_config_of_the_headline():
    c = bench.run_config("large_head", "fwdbwd", 1)
    assert (c["B"], c["H"], c["N"], c["d"], c["causal"]) == (4, 16, 4096, 128, True)
    assert c["flop_per_step"] == sum(bench.flops(4, 16, 4096, 128, True))
    assert c["l2"] == "inputs larger than L2 (working set 336 MB)"
    assert bench.run_config("tiny", "fwd", 1)["l2"].startswith("L2 flushed")
