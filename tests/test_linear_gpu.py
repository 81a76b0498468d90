"""Causal linear attention (chunked, tcgen05) on a B200 against the oracle.

O_i = scale sum_{j <= i} (q_i . k_j) v_j, computed in chunks of 128 rows
(the intra-/inter-block split of "Lightning Attention-2" (chatpaper.ai
summary) and the chunk-wise form of "Gated Linear Attention Transformers with
Hardware-Efficient Training" (nubint.ai review)).  The output is not
normalised (|O| grows with the row index), so the bars are relative: relative
L2 <= 5e-3 (the forward's bar) and max-abs <= 1e-2 times max |O|.
"""

import numpy as np
import pytest

import oracle
from helpers import default_scale, inputs, rel_l2, to_device

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from io_aware_exact_30_b200 import attn  # noqa: E402

LIN_REL_L2 = 5e-3
LIN_MAX_REL = 1e-2


def check(got, want, label):
    assert np.all(np.isfinite(got)), label
    rl = rel_l2(got, want)
    ma = float(np.abs(got - want).max()) / max(float(np.abs(want).max()), 1e-30)
    assert rl <= LIN_REL_L2, f"{label} rel-L2 {rl}"
    assert ma <= LIN_MAX_REL, f"{label} max-abs / max|O| {ma}"


# B H < 32 runs the three chunk-parallel kernels, B H >= 32 the fused one
# (one CTA per head and half of the value features, walking the chunks)
@pytest.mark.parametrize("B,H,N,dtype", [(1, 2, 700, "bf16"), (1, 3, 513, "fp16"),
                                         (2, 1, 1, "bf16"), (1, 2, 129, "bf16"),
                                         (1, 1, 128, "fp16"), (2, 40, 1000, "bf16"),
                                         (1, 31, 300, "bf16"), (1, 32, 300, "fp16"),
                                         (4, 8, 1, "bf16"), (8, 4, 129, "fp16"),
                                         (2, 16, 128, "bf16"), (1, 33, 1535, "bf16")])
def test_linear_attention_parity(B, H, N, dtype):
    d = 128
    arrs, f64 = inputs(B, H, N, d, dtype=dtype, seed=N)
    scale = default_scale(d)
    o = attn.linear_forward(*(to_device(a, dtype) for a in arrs), scale)
    torch.cuda.synchronize()
    assert attn.attn_last_device_status() == 0
    got = o.double().cpu().numpy()
    if B * H <= 6:
        check(got, oracle.linear_attn(*f64, scale), f"{(B, H, N, dtype)}")
    else:
        for bh in (0, B * H // 2, B * H - 1):
            b, h = divmod(bh, H)
            sel = [x[b:b + 1, h:h + 1] for x in f64]
            check(got[b:b + 1, h:h + 1], oracle.linear_attn(*sel, scale), f"head {bh}")


def test_linear_attention_large_head_shape_sampled_heads():
    B, H, N, d = 4, 16, 4096, 128
    arrs, f64 = inputs(B, H, N, d, seed=0)
    o = attn.linear_forward(*(to_device(a, "bf16") for a in arrs))
    torch.cuda.synchronize()
    got = o.double().cpu().numpy()
    for bh in (0, 31, 63):
        b, h = divmod(bh, H)
        sel = [x[b:b + 1, h:h + 1] for x in f64]
        check(got[b:b + 1, h:h + 1], oracle.linear_attn(*sel, default_scale(d)), f"head {bh}")


def test_linear_attention_rejects_d64():
    q = torch.zeros(1, 1, 64, 64, dtype=torch.bfloat16, device="cuda")
    assert attn.attn_linear_workspace_bytes(1, 1, 64, 64) == 0
    with pytest.raises(ValueError):
        attn.linear_forward(q, q, q)
