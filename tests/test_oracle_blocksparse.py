"""Pins of the block-sparse oracle (CPU only).

Block-sparse attention ("FlashAttention の概要", zenn.dev, the paragraph on
Block-Sparse FlashAttention) computes attention only over the (query block,
key block) pairs a block mask marks.  The oracle's functions are pinned to:
brute force on the full N x N matrix with the mask expanded by np.kron and
scipy's softmax/logsumexp; an all-ones mask reducing to the exact attention
(itself pinned in test_oracle_pins.py); a block-diagonal mask reducing to
independent attention over each block; fully masked rows giving O = 0 and
LSE = -inf; fp64 autograd of the brute-force definition and central
differences for the gradients.  Planted mistakes in a compiled copy of the
source (mask transposed, the causal rule dropped inside marked blocks, block
index off by one row) each fail the brute-force pin.
"""

import ctypes
import math
import os
import subprocess
import tempfile

import numpy as np
import pytest
import scipy.special as sps
import torch

import oracle

RNG = np.random.default_rng(777)
SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle",
                   "attn_oracle.c")


def rand(*shape):
    return RNG.standard_normal(shape)


def visibility(mask, N, blk, causal):
    """Full (N, N) boolean visibility: the block mask expanded, cut to N."""
    full = np.kron(np.asarray(mask, bool), np.ones((blk, blk), bool))[:N, :N]
    if causal:
        full &= np.tril(np.ones((N, N), bool))
    return full


def brute(q, k, v, mask, blk, causal, scale):
    N = q.shape[-2]
    vis = visibility(mask, N, blk, causal)
    s = np.where(vis, scale * np.einsum("...id,...jd->...ij", q, k), -np.inf)
    lse = sps.logsumexp(s, axis=-1)
    empty = ~vis.any(-1)
    p = np.exp(s - np.where(np.isfinite(lse), lse, 0.0)[..., None])
    p[..., empty, :] = 0.0
    return p @ v, lse


def random_mask(nb, density, rng, keep_diag=False):
    m = (rng.random((nb, nb)) < density).astype(np.uint8)
    if keep_diag:
        np.fill_diagonal(m, 1)
    return m


CASES = [(1, 2, 40, 4, 8, 0.5), (2, 1, 37, 8, 10, 0.4), (1, 1, 64, 16, 16, 0.6),
         (1, 3, 19, 5, 4, 0.3)]


@pytest.mark.parametrize("B,H,N,d,blk,density", CASES)
@pytest.mark.parametrize("causal", [False, True])
def test_blocksparse_fwd_equals_bruteforce(B, H, N, d, blk, density, causal):
    q, k, v = rand(B, H, N, d), rand(B, H, N, d), rand(B, H, N, d)
    nb = (N + blk - 1) // blk
    mask = random_mask(nb, density, RNG)
    o, lse = oracle.fwd_blocksparse(q, k, v, mask, causal, 0.4, block=blk)
    ob, lb = brute(q, k, v, mask, blk, causal, 0.4)
    np.testing.assert_allclose(o, ob, rtol=0, atol=1e-13)
    fin = np.isfinite(lb)
    assert np.array_equal(fin, np.isfinite(lse))
    np.testing.assert_allclose(lse[fin], lb[fin], rtol=0, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_all_ones_mask_is_exact_attention(causal):
    q, k, v = rand(1, 2, 50, 8), rand(1, 2, 50, 8), rand(1, 2, 50, 8)
    o, lse = oracle.fwd_blocksparse(q, k, v, np.ones((4, 4), np.uint8), causal, 0.3, block=16)
    o2, lse2 = oracle.fwd(q, k, v, causal, 0.3)
    np.testing.assert_allclose(o, o2, rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse, lse2, rtol=0, atol=1e-14)


def test_block_diagonal_mask_is_independent_blocks():
    blk, nb = 8, 5
    N = blk * nb - 3
    q, k, v = rand(1, 1, N, 4), rand(1, 1, N, 4), rand(1, 1, N, 4)
    o, lse = oracle.fwd_blocksparse(q, k, v, np.eye(nb, dtype=np.uint8), False, 0.5, block=blk)
    for b in range(nb):
        sl = slice(b * blk, min(N, (b + 1) * blk))
        ob, lb = oracle.fwd(q[..., sl, :], k[..., sl, :], v[..., sl, :], False, 0.5)
        np.testing.assert_allclose(o[..., sl, :], ob, rtol=0, atol=1e-14)
        np.testing.assert_allclose(lse[..., sl], lb, rtol=0, atol=1e-14)


def test_fully_masked_rows_are_zero_with_minus_inf_lse():
    blk, N = 4, 12
    mask = np.ones((3, 3), np.uint8)
    mask[1, :] = 0  # query block 1 sees nothing
    q, k, v, do = (rand(1, 1, N, 3) for _ in range(4))
    o, lse = oracle.fwd_blocksparse(q, k, v, mask, False, 1.0, block=blk)
    assert np.all(o[0, 0, 4:8] == 0.0) and np.all(np.isneginf(lse[0, 0, 4:8]))
    assert np.all(np.isfinite(lse[0, 0, :4])) and np.all(np.isfinite(lse[0, 0, 8:]))
    dq, dk, dv = oracle.bwd_blocksparse(q, k, v, do, mask, False, 1.0, block=blk)
    assert np.all(dq[0, 0, 4:8] == 0.0)


def _torch_loss(q, k, v, do, mask, blk, causal, scale):
    N = q.shape[-2]
    vis = torch.tensor(visibility(mask, N, blk, causal))
    s = (scale * q @ k.transpose(-1, -2)).masked_fill(~vis, float("-inf"))
    p = torch.softmax(s, -1).nan_to_num(0.0)  # rows with no visible key: P = 0
    return (p @ v * do).sum()


@pytest.mark.parametrize("causal", [False, True])
def test_blocksparse_bwd_equals_fp64_autograd(causal):
    B, H, N, d, blk = 1, 2, 30, 5, 6
    mask = random_mask(5, 0.5, RNG, keep_diag=True)
    mask[2, :] = 0  # and one empty query block
    q, k, v, do = (rand(B, H, N, d) for _ in range(4))
    got = oracle.bwd_blocksparse(q, k, v, do, mask, causal, 0.45, block=blk)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    _torch_loss(tq, tk, tv, torch.tensor(do), mask, blk, causal, 0.45).backward()
    for mine, ref in zip(got, (tq.grad, tk.grad, tv.grad)):
        np.testing.assert_allclose(mine, ref.numpy(), rtol=0, atol=1e-12)


def test_blocksparse_bwd_central_differences():
    N, d, blk = 10, 3, 4
    mask = np.array([[1, 0, 1], [0, 1, 0], [1, 1, 1]], np.uint8)
    q, k, v, do = (rand(1, 1, N, d) for _ in range(4))
    dq, dk, dv = oracle.bwd_blocksparse(q, k, v, do, mask, True, 0.7, block=blk)

    def loss(q, k, v):
        o, _ = oracle.fwd_blocksparse(q, k, v, mask, True, 0.7, block=blk)
        return float((o * do).sum())
    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args = {"q": q, "k": k, "v": v}
            num[idx] = (loss(**{**args, name: xp}) - loss(**{**args, name: xm})) / (2 * h)
        np.testing.assert_allclose(g, num, rtol=0, atol=1e-6 * max(1.0, np.abs(num).max()))


MUTANTS = {
    "mask transposed": ("if (mask[(i / blk) * nb + j / blk] && (!causal || j <= i)) idx[n++] = j;",
                        "if (mask[(j / blk) * nb + i / blk] && (!causal || j <= i)) idx[n++] = j;"),
    "causal rule dropped in marked blocks":
        ("if (mask[(i / blk) * nb + j / blk] && (!causal || j <= i)) idx[n++] = j;",
         "if (mask[(i / blk) * nb + j / blk]) idx[n++] = j;"),
    "query block off by one row": ("if (mask[(i / blk) * nb + j / blk]",
                                   "if (mask[((i + 1) / blk < nb ? (i + 1) / blk : nb - 1) * nb + j / blk]"),
    "dS uses the row max list index wrongly": ("double dsij = p[r] * (dpij - Di);",
                                               "double dsij = p[j] * (dpij - Di);"),
}


def _build(text):
    dd = tempfile.mkdtemp(prefix="oracle_bs_mutant_")
    c, so = os.path.join(dd, "m.c"), os.path.join(dd, "m.so")
    with open(c, "w") as f:
        f.write(text)
    subprocess.run(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-o", so, c, "-lm"], check=True)
    L = ctypes.CDLL(so)
    dp, lp = ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int64)
    u8 = ctypes.POINTER(ctypes.c_uint8)
    i64, ci, cd = ctypes.c_int64, ctypes.c_int, ctypes.c_double
    L.oracle_fwd_blocksparse.argtypes = [dp, dp, dp, dp, dp, i64, i64, i64, ci, cd, u8, i64]
    L.oracle_bwd_blocksparse_heads.argtypes = [dp, dp, dp, dp, i64, i64, i64, ci, cd, u8, i64,
                                               lp, i64, dp, dp, dp]
    return L


def _pins_pass(L):
    rng = np.random.default_rng(9)
    P = lambda a: a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))
    for causal in (0, 1):
        BH, N, d, blk, scale = 2, 23, 3, 5, 0.6
        nb = (N + blk - 1) // blk
        mask = random_mask(nb, 0.5, rng, keep_diag=True)
        mask[0, 1] = 1 - mask[1, 0]  # not symmetric
        q, k, v, do = (rng.standard_normal((BH, N, d)) for _ in range(4))
        o, lse = np.empty_like(q), np.empty((BH, N))
        L.oracle_fwd_blocksparse(P(q), P(k), P(v), P(o), P(lse), BH, N, d, causal, scale,
                                 mask.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)), blk)
        ob, lb = brute(q, k, v, mask, blk, causal, scale)
        if not (np.allclose(o, ob, atol=1e-12) and np.allclose(lse, lb, atol=1e-12)):
            return False
        heads = np.arange(BH, dtype=np.int64)
        dq, dk, dv = (np.empty_like(q) for _ in range(3))
        L.oracle_bwd_blocksparse_heads(P(q), P(k), P(v), P(do), BH, N, d, causal, scale,
                                       mask.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)), blk,
                                       heads.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), BH,
                                       P(dq), P(dk), P(dv))
        tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
        _torch_loss(tq, tk, tv, torch.tensor(do), mask, blk, causal, scale).backward()
        for mine, ref in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
            if not np.allclose(mine, ref.numpy(), atol=1e-11):
                return False
    return True


def test_unmutated_blocksparse_copy_passes():
    with open(SRC) as f:
        assert _pins_pass(_build(f.read()))


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_blocksparse_mutant_is_caught(name):
    old, new = MUTANTS[name]
    with open(SRC) as f:
        text = f.read()
    assert text.count(old) == 1, f"mutation site missing or ambiguous: {old}"
    assert not _pins_pass(_build(text.replace(old, new, 1)))
