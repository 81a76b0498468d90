"""Forward parity: the CUDA path against the fp64 oracle (needs a B200).

Small shapes are compared element by element over every output; the full
workloads are compared on sampled rows (the oracle computes each row on its
own) with the same launch configuration the benchmark times.
"""

import numpy as np
import pytest

import oracle
from helpers import CONFIGS, check_fwd, default_scale, inputs, sample_rows, to_device

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from io_aware_exact_30_b200 import attn  # noqa: E402


def run_fwd(arrs, dtype, causal, scale):
    q, k, v = (to_device(a, dtype) for a in arrs[:3])
    o, lse = attn.forward(q, k, v, causal, scale)
    torch.cuda.synchronize()
    assert attn.attn_last_device_status() == 0
    return o.double().cpu().numpy(), lse.double().cpu().numpy()


SMALL = [
    # B, H, N, d, causal, dtype
    (1, 1, 1, 64, False, "bf16"),
    (1, 1, 1, 128, True, "bf16"),
    (1, 2, 17, 64, True, "bf16"),
    (2, 1, 128, 64, False, "bf16"),
    (1, 2, 129, 128, False, "bf16"),
    (1, 2, 129, 64, True, "fp16"),
    (1, 1, 255, 128, True, "fp16"),
    (2, 3, 300, 64, False, "fp16"),
    (1, 2, 640, 128, True, "bf16"),
    (1, 1, 1000, 128, False, "bf16"),
]


@pytest.mark.parametrize("B,H,N,d,causal,dtype", SMALL)
def test_fwd_small_full_compare(B, H, N, d, causal, dtype):
    arrs, f64 = inputs(B, H, N, d, dtype=dtype, seed=N + d)
    scale = default_scale(d)
    o, lse = run_fwd(arrs, dtype, causal, scale)
    o_ref, lse_ref = oracle.fwd(*f64, causal, scale)
    check_fwd(o, lse, o_ref, lse_ref, f"{(B, H, N, d, causal, dtype)}")


def test_fwd_tiny_config_full():
    B, H, N, d, causal, dtype, sigma, _ = CONFIGS["tiny"]
    arrs, f64 = inputs(B, H, N, d, dtype=dtype, sigma=sigma)
    o, lse = run_fwd(arrs, dtype, causal, default_scale(d))
    check_fwd(o, lse, *oracle.fwd(*f64, causal, default_scale(d)), "tiny")


def test_fwd_bert_large_config_full():
    B, H, N, d, causal, dtype, sigma, _ = CONFIGS["bert_large"]
    arrs, f64 = inputs(B, H, N, d, dtype=dtype, sigma=sigma)
    o, lse = run_fwd(arrs, dtype, causal, default_scale(d))
    check_fwd(o, lse, *oracle.fwd(*f64, causal, default_scale(d)), "bert_large")


@pytest.mark.parametrize("name", ["gpt2_causal", "long_day", "large_head"])
def test_fwd_full_size_sampled_rows(name):
    B, H, N, d, causal, dtype, sigma, _ = CONFIGS[name]
    arrs, f64 = inputs(B, H, N, d, dtype=dtype, sigma=sigma)
    scale = default_scale(d)
    o, lse = run_fwd(arrs, dtype, causal, scale)
    rows = sample_rows(B * H, N, per_head=16)
    o_ref, lse_ref = oracle.fwd_rows(*f64, causal, scale, rows)
    check_fwd(o.reshape(-1, d)[rows], lse.reshape(-1)[rows], o_ref, lse_ref, name)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))


def test_fwd_is_deterministic():
    arrs, _ = inputs(2, 4, 700, 128, seed=9)
    q, k, v = (to_device(a, "bf16") for a in arrs)
    o1, l1 = attn.forward(q, k, v, True)
    o2, l2 = attn.forward(q, k, v, True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_fwd_allocates_nothing_on_long_sequence():
    # The 23,400-step, 12-head fp16 score matrix would take about 13 GB; the
    # call must not allocate device memory at all (caller owns every buffer).
    B, H, N, d, causal, dtype, sigma, _ = CONFIGS["long_day"]
    arrs, _ = inputs(B, H, N, d, dtype=dtype, sigma=sigma)
    q, k, v = (to_device(a, dtype) for a in arrs)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    attn.attn_fwd(q, k, v, o, lse, causal)  # warm: lazy module load happens once
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    alloc0 = torch.cuda.memory_allocated()
    attn.attn_fwd(q, k, v, o, lse, causal)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert torch.cuda.memory_allocated() == alloc0
    assert free0 - free1 < 64 << 20
