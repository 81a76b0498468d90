"""Backward parity: dQ, dK, dV of the CUDA path against the fp64 oracle's
exact gradients of sum(O * dO) (needs a B200).

The GPU backward consumes the GPU forward's O and LSE, as a user would; the
oracle differentiates the definition directly.  Small shapes compare every
head; the full workloads compare whole heads picked across the batch.
"""

import numpy as np
import pytest

import oracle
from helpers import CONFIGS, check_fwd, check_grads, default_scale, inputs, to_device

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from io_aware_exact_30_b200 import attn  # noqa: E402


def gpu_fwd_bwd(arrs, dtype, causal, scale, split=False):
    q, k, v, do = (to_device(a, dtype) for a in arrs)
    o, lse = attn.forward(q, k, v, causal, scale)
    if split:
        B, H, N, d = q.shape
        dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
        ws = torch.empty(attn.attn_bwd_workspace_bytes(B, H, N, d), dtype=torch.uint8, device="cuda")
        attn.attn_bwd_prep(o, do, lse, ws)
        attn.attn_bwd_main(q, k, v, do, dq, dk, dv, ws, causal, scale)
    else:
        dq, dk, dv = attn.backward(q, k, v, o, lse, do, causal, scale)
    torch.cuda.synchronize()
    assert attn.attn_last_device_status() == 0
    return [t.double().cpu().numpy() for t in (dq, dk, dv)]


SMALL = [
    # B, H, N, d, causal, dtype
    (1, 1, 1, 64, False, "bf16"),
    (1, 1, 1, 128, True, "fp16"),
    (1, 2, 17, 64, True, "bf16"),
    (1, 1, 128, 128, False, "bf16"),
    (1, 2, 129, 64, False, "bf16"),
    (2, 1, 200, 128, True, "fp16"),
    (1, 1, 300, 64, True, "bf16"),
    (1, 2, 640, 128, True, "bf16"),
    (1, 1, 513, 128, False, "fp16"),
]


@pytest.mark.parametrize("B,H,N,d,causal,dtype", SMALL)
def test_bwd_small_full_compare(B, H, N, d, causal, dtype):
    arrs, f64 = inputs(B, H, N, d, dtype=dtype, seed=3 * N + d, with_dout=True)
    scale = default_scale(d)
    g = gpu_fwd_bwd(arrs, dtype, causal, scale)
    ref = oracle.bwd(*f64, causal, scale)
    check_grads(g, ref, f"{(B, H, N, d, causal, dtype)}")


@pytest.mark.parametrize("name,heads", [("gpt2_causal", [0, 47, 50, 95]), ("large_head", [0, 31, 63])])
def test_bwd_full_size_selected_heads(name, heads):
    B, H, N, d, causal, dtype, sigma, with_bwd = CONFIGS[name]
    assert with_bwd
    arrs, f64 = inputs(B, H, N, d, dtype=dtype, sigma=sigma, with_dout=True)
    scale = default_scale(d)
    g = gpu_fwd_bwd(arrs, dtype, causal, scale)
    ref = oracle.bwd_heads(*f64, causal, scale, heads=heads)
    g_sel = [x.reshape(B * H, N, d)[heads] for x in g]
    check_grads(g_sel, ref, name)
    for x in g:
        assert np.all(np.isfinite(x))


def test_bwd_split_phases_equal_single_call():
    arrs, _ = inputs(2, 3, 333, 128, seed=4, with_dout=True)
    a = gpu_fwd_bwd(arrs, "bf16", True, 0.1)
    b = gpu_fwd_bwd(arrs, "bf16", True, 0.1, split=True)
    np.testing.assert_array_equal(a[1], b[1])  # dK, dV are deterministic
    np.testing.assert_array_equal(a[2], b[2])
    np.testing.assert_allclose(a[0], b[0], rtol=0, atol=2e-2)  # dQ: atomic order


def test_bwd_workspace_contents_do_not_matter():
    B, H, N, d = 1, 2, 260, 64
    arrs, f64 = inputs(B, H, N, d, seed=8, with_dout=True)
    q, k, v, do = (to_device(a, "bf16") for a in arrs)
    o, lse = attn.forward(q, k, v, True)
    ws = torch.full((attn.attn_bwd_workspace_bytes(B, H, N, d),), 0x7F, dtype=torch.uint8, device="cuda")
    dq, dk, dv = attn.backward(q, k, v, o, lse, do, True, workspace=ws)
    torch.cuda.synchronize()
    ref = oracle.bwd(*f64, True, default_scale(d))
    check_grads([t.double().cpu().numpy() for t in (dq, dk, dv)], ref, "garbage workspace")


# Shapes whose work items outnumber the multiprocessors (several items per
# persistent CTA, taken dynamically under the causal mask and in static snake
# order without it), with ragged key and query tails, and one with long items.
MANY_ITEMS = [
    (2, 40, 1000, 128, True),
    (3, 20, 777, 128, False),
    (1, 2, 5000, 128, True),
]


@pytest.mark.parametrize("B,H,N,d,causal", MANY_ITEMS)
def test_fwd_bwd_many_items_per_cta(B, H, N, d, causal):
    arrs, f64 = inputs(B, H, N, d, seed=2, with_dout=True)
    scale = default_scale(d)
    q, k, v, do = (to_device(a, "bf16") for a in arrs)
    o, lse = attn.forward(q, k, v, causal, scale)
    dq, dk, dv = attn.backward(q, k, v, o, lse, do, causal, scale)
    torch.cuda.synchronize()
    assert attn.attn_last_device_status() == 0
    got = [t.double().cpu().numpy() for t in (o, lse, dq, dk, dv)]
    for bh in (0, B * H - 1):
        b, h = divmod(bh, H)
        sel = [x[b:b + 1, h:h + 1] for x in f64]
        o_ref, lse_ref = oracle.fwd(*sel[:3], causal, scale)
        check_fwd(got[0][b:b + 1, h:h + 1], got[1][b:b + 1, h:h + 1], o_ref, lse_ref,
                  f"{(B, H, N, d, causal)} head {bh}")
        ref = oracle.bwd(*sel, causal, scale)
        check_grads([x[b:b + 1, h:h + 1] for x in got[2:]], ref, f"{(B, H, N, d, causal)} head {bh}")
