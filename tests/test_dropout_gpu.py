"""Dropout on the attention probabilities on a B200, against the oracle.

The mask comes from Philox4x32-10 keyed by the seed (counter (j / 16, i,
head)), generated in the forward by the thread that owns query row i and in
the backward by the warps that own key rows (each lane generating its own
query's bytes, the warp transposing them).  Both must give the oracle's mask
exactly, so O, LSE and dQ, dK, dV are compared element by element with the
oracle's dropout forward and backward at the tolerances of the dense path.
"""

import numpy as np
import pytest

import oracle
from helpers import check_fwd, check_grads, default_scale, inputs, to_device

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from io_aware_exact_30_b200 import attn  # noqa: E402

CASES = [
    # B, H, N, d, causal, dtype, p
    (1, 2, 300, 64, True, "bf16", 0.1),
    (1, 2, 300, 128, False, "bf16", 0.1),
    (2, 1, 700, 128, True, "bf16", 0.3),
    (1, 3, 513, 64, False, "fp16", 0.5),
    (1, 2, 129, 128, True, "fp16", 0.75),
    (2, 40, 1000, 128, True, "bf16", 0.2),  # more work items than multiprocessors
]


@pytest.mark.parametrize("B,H,N,d,causal,dtype,p", CASES)
def test_dropout_fwd_bwd_parity(B, H, N, d, causal, dtype, p):
    seed = 0x5EED0000 + N * 7 + d
    # sigma 0.5 (the long-day workload's): kept values are scaled by 1 / (1 - p),
    # and with sigma 1 an early causal row (few keys) reaches |O| > 4, where
    # half a bf16 ulp (2^-6) alone exceeds the 1e-2 max-abs bar
    arrs, f64 = inputs(B, H, N, d, dtype=dtype, sigma=0.5, seed=N, with_dout=True)
    scale = default_scale(d)
    q, k, v, do = (to_device(a, dtype) for a in arrs)
    o, lse = attn.forward_dropout(q, k, v, p, seed, causal, scale)
    dq, dk, dv = attn.backward_dropout(q, k, v, o, lse, do, p, seed, causal, scale)
    torch.cuda.synchronize()
    assert attn.attn_last_device_status() == 0
    got = [t.double().cpu().numpy() for t in (o, lse, dq, dk, dv)]
    label = f"{(B, H, N, d, causal, dtype, p)}"
    # the mask depends on the head index: the oracle sees every head
    o_ref, lse_ref = oracle.fwd_dropout(*f64[:3], causal, scale, p, seed)
    heads = range(B * H) if B * H <= 6 else (0, B * H // 2, B * H - 1)
    for bh in heads:
        b, h = divmod(bh, H)
        check_fwd(got[0][b, h], got[1][b, h], o_ref[b, h], lse_ref[b, h], f"{label} head {bh}")
        ref = oracle.bwd_dropout_heads(*f64, causal, scale, p, seed, heads=[bh])
        check_grads([g[b, h][None] for g in got[2:]], ref, f"{label} head {bh}")


def test_dropout_zero_equals_plain_path():
    B, H, N, d = 1, 3, 400, 128
    arrs, _ = inputs(B, H, N, d, seed=4, with_dout=True)
    q, k, v, do = (to_device(a, "bf16") for a in arrs)
    o1, l1 = attn.forward(q, k, v, True)
    o2, l2 = attn.forward_dropout(q, k, v, 0.0, 123, True)
    g1 = attn.backward(q, k, v, o1, l1, do, True)
    g2 = attn.backward_dropout(q, k, v, o2, l2, do, 0.0, 123, True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    assert torch.equal(g1[1], g2[1]) and torch.equal(g1[2], g2[2])


def test_dropout_rejects_bad_probability():
    q = torch.zeros(1, 1, 16, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(attn.AttnError):
        attn.forward_dropout(q, q, q, 1.0, 1)
    with pytest.raises(attn.AttnError):
        attn.forward_dropout(q, q, q, -0.1, 1)
