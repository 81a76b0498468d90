"""Block-sparse attention on a B200 against the fp64 block-sparse oracle.

The kernels take a 128 x 128 block mask (one for every head) and skip the
blocks it leaves out ("FlashAttention の概要", zenn.dev, the paragraph on
Block-Sparse FlashAttention).  Seeded random masks include query tiles with
no marked block (their rows give O = 0 and LSE = -inf) and key tiles no query
tile attends to (their dK, dV are 0); shapes have ragged tails and more work
items than multiprocessors, causal and not, d = 64 and 128, bf16 and fp16.
"""

import numpy as np
import pytest

import oracle
from helpers import check_fwd, check_grads, default_scale, inputs, to_device

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from io_aware_exact_30_b200 import attn  # noqa: E402


def seeded_mask(nb, density, seed, empty_row=None, empty_col=None):
    rng = np.random.default_rng(seed)
    m = (rng.random((nb, nb)) < density).astype(np.uint8)
    if empty_row is not None:
        m[empty_row, :] = 0
    if empty_col is not None:
        m[:, empty_col] = 0
    return m


def run(arrs, dtype, mask, causal, scale, with_bwd=True):
    q, k, v = (to_device(a, dtype) for a in arrs[:3])
    mdev = torch.from_numpy(mask).cuda()
    o, lse = attn.forward_blocksparse(q, k, v, mdev, causal, scale)
    out = [o, lse]
    if with_bwd:
        do = to_device(arrs[3], dtype)
        out += list(attn.backward_blocksparse(q, k, v, o, lse, do, mdev, causal, scale))
    torch.cuda.synchronize()
    assert attn.attn_last_device_status() == 0
    return [t.double().cpu().numpy() for t in out]


def check_against_oracle(got, f64, mask, causal, scale, label, with_bwd=True):
    o, lse = got[:2]
    o_ref, lse_ref = oracle.fwd_blocksparse(*f64[:3], mask, causal, scale)
    empty = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse), empty), label
    assert np.all(o[empty] == 0.0), label
    live = ~empty
    check_fwd(o[live], lse[live], o_ref[live], lse_ref[live], label)
    if with_bwd:
        ref = oracle.bwd_blocksparse(*f64, mask, causal, scale)
        check_grads(got[2:], ref, label)


CASES = [
    # B, H, N, d, causal, dtype, density, empty query tile, empty key tile
    (1, 2, 700, 64, False, "bf16", 0.5, 2, 4),
    (1, 2, 700, 128, False, "bf16", 0.5, 1, 3),
    (2, 1, 1000, 128, True, "bf16", 0.6, 5, 0),
    (1, 3, 777, 64, True, "fp16", 0.6, 0, 6),
    (1, 2, 513, 128, False, "fp16", 0.3, None, None),
    (2, 40, 1000, 128, True, "bf16", 0.5, 3, 2),  # many items per persistent CTA
    (2, 40, 1000, 64, False, "bf16", 0.5, 3, 2),
    # mostly empty: runs of key tiles no query tile attends to (items whose
    # per-item handshakes must still stay in step)
    (1, 16, 2048, 128, False, "bf16", 0.08, None, None),
    (1, 16, 2048, 128, True, "bf16", 0.08, None, None),
]


@pytest.mark.parametrize("B,H,N,d,causal,dtype,density,er,ec", CASES)
def test_blocksparse_fwd_bwd_parity(B, H, N, d, causal, dtype, density, er, ec):
    nb = (N + 127) // 128
    mask = seeded_mask(nb, density, seed=N + d, empty_row=er, empty_col=ec)
    arrs, f64 = inputs(B, H, N, d, dtype=dtype, seed=N, with_dout=True)
    scale = default_scale(d)
    got = run(arrs, dtype, mask, causal, scale)
    label = f"{(B, H, N, d, causal, dtype, density)}"
    if B * H <= 6:
        check_against_oracle(got, f64, mask, causal, scale, label)
    else:  # many heads: compare the first, a middle and the last head
        for bh in (0, (B * H) // 2, B * H - 1):
            b, h = divmod(bh, H)
            sel = [x[b:b + 1, h:h + 1] for x in f64]
            check_against_oracle([g[b:b + 1, h:h + 1] for g in got], sel, mask, causal, scale,
                                 f"{label} head {bh}")


@pytest.mark.parametrize("d,causal", [(64, False), (128, True), (128, False)])
def test_all_ones_mask_equals_dense_path(d, causal):
    B, H, N = 2, 3, 600
    arrs, _ = inputs(B, H, N, d, seed=11, with_dout=True)
    mask = np.ones(((N + 127) // 128,) * 2, np.uint8)
    got = run(arrs, "bf16", mask, causal, default_scale(d))
    q, k, v, do = (to_device(a, "bf16") for a in arrs)
    o, lse = attn.forward(q, k, v, causal)
    dq, dk, dv = attn.backward(q, k, v, o, lse, do, causal)
    torch.cuda.synchronize()
    dense = [t.double().cpu().numpy() for t in (o, lse, dq, dk, dv)]
    for name, a, b in zip(("O", "LSE", "dK", "dV"), got[:2] + got[3:], dense[:2] + dense[3:]):
        np.testing.assert_array_equal(a, b, err_msg=name)  # same per-item arithmetic
    np.testing.assert_allclose(got[2], dense[2], rtol=0, atol=2e-2)  # dQ: fp32 add order


def test_empty_mask_gives_zero_outputs():
    B, H, N, d = 1, 2, 300, 128
    arrs, _ = inputs(B, H, N, d, seed=5, with_dout=True)
    got = run(arrs, "bf16", np.zeros((3, 3), np.uint8), False, default_scale(d))
    assert np.all(got[0] == 0.0) and np.all(np.isneginf(got[1]))
    for g in got[2:]:
        assert np.all(g == 0.0)


def test_blocksparse_full_size_sampled():
    # the large-head shape with half of the blocks marked (and the diagonal,
    # so that no row is empty): forward on sampled rows, backward on 3 heads
    B, H, N, d = 4, 16, 4096, 128
    mask = seeded_mask(32, 0.5, seed=1)
    np.fill_diagonal(mask, 1)
    arrs, f64 = inputs(B, H, N, d, seed=0, with_dout=True)
    scale = default_scale(d)
    got = run(arrs, "bf16", mask, False, scale)
    for bh in (0, 31, 63):
        b, h = divmod(bh, H)
        sel = [x[b:b + 1, h:h + 1] for x in f64]
        o_ref, lse_ref = oracle.fwd_blocksparse(*sel[:3], mask, False, scale)
        check_fwd(got[0][b:b + 1, h:h + 1], got[1][b:b + 1, h:h + 1], o_ref, lse_ref, f"head {bh}")
        ref = oracle.bwd_blocksparse(*sel, mask, False, scale)
        check_grads([g[b:b + 1, h:h + 1] for g in got[2:]], ref, f"head {bh}")
