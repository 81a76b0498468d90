"""Pins of the dropout part of the oracle (CPU only).

Dropout on the attention probabilities (the dropout_p argument of the
attention call in "Is a full day of context better than ten minutes?"
(marketmaker.cc), section "integration is eight lines"), with the keep mask
drawn from Philox4x32-10 (Salmon et al., SC 2011).  Pinned:
 - the generator against the known-answer vectors published with the
   authors' reference release (tests/golden/philox4x32_10_kat.txt);
 - the mask: keep fraction t / 256 within four standard deviations, p = 0
   keeping everything;
 - the forward: p = 0 equal to the exact forward; brute force (scipy
   softmax, explicit mask) for p > 0; the average over many seeds tending to
   the dropout-free output (the 256 / t scaling makes it unbiased);
 - the backward against fp64 torch autograd of the brute force with the same
   explicit mask;
 - planted mistakes in a compiled copy of the source are caught.
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

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(os.path.dirname(HERE), "oracle", "attn_oracle.c")
RNG = np.random.default_rng(2024)


def kat_vectors():
    out = []
    for line in open(os.path.join(HERE, "golden", "philox4x32_10_kat.txt")):
        if line.startswith("#") or not line.strip():
            continue
        ctr, key, res = (part.split() for part in line.split("|"))
        out.append(([int(x, 16) for x in ctr], [int(x, 16) for x in key],
                    [int(x, 16) for x in res]))
    return out


def test_philox_known_answers():
    vecs = kat_vectors()
    assert len(vecs) == 3
    for ctr, key, want in vecs:
        assert oracle.philox4x32_10(ctr, key) == want


@pytest.mark.parametrize("p", [0.1, 0.5, 0.9])
def test_mask_keep_fraction(p):
    t = oracle.dropout_threshold(p)
    z = oracle.dropout_mask(3, 400, seed=123, p=p)
    n, keep = z.size, t / 256.0
    assert abs(z.mean() - keep) < 4 * math.sqrt(keep * (1 - keep) / n)
    assert np.all(oracle.dropout_mask(1, 50, seed=1, p=0.0) == 1)


def test_mask_follows_the_stated_counter_layout():
    # Z_ij = [byte (j % 16) of Philox(counter (j / 16, i, bh, 0), key (seed lo, hi)) < t]
    seed, p = 0x1234_5678_9ABC_DEF0, 0.3
    t = oracle.dropout_threshold(p)
    z = oracle.dropout_mask(3, 70, seed, p)
    for bh, i, j in [(0, 0, 0), (2, 69, 69), (1, 5, 17), (2, 33, 47), (0, 64, 3)]:
        w = oracle.philox4x32_10([j >> 4, i, bh, 0], [seed & 0xFFFFFFFF, seed >> 32])
        byte = (w[(j % 16) // 4] >> (8 * (j % 4))) & 0xFF
        assert z[bh, i, j] == (byte < t)


def brute(q, k, v, causal, scale, z, t):
    s = scale * np.einsum("...id,...jd->...ij", q, k)
    if causal:
        N = q.shape[-2]
        s = np.where(np.tril(np.ones((N, N), bool)), s, -np.inf)
    P = sps.softmax(s, axis=-1)
    return (P * z * (256.0 / t)) @ v, sps.logsumexp(s, axis=-1)


@pytest.mark.parametrize("causal", [False, True])
def test_p_zero_is_exact_attention(causal):
    q, k, v = (RNG.standard_normal((2, 37, 8)) for _ in range(3))
    o, lse = oracle.fwd_dropout(q, k, v, causal, 0.35, p=0.0, seed=5)
    o2, lse2 = oracle.fwd(q, k, v, causal, 0.35)
    np.testing.assert_allclose(o, o2, rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse, lse2, rtol=0, atol=1e-14)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("p", [0.2, 0.6])
def test_forward_equals_bruteforce(causal, p):
    BH, N, d = 3, 45, 6
    q, k, v = (RNG.standard_normal((BH, N, d)) for _ in range(3))
    z = oracle.dropout_mask(BH, N, seed=77, p=p)
    o, lse = oracle.fwd_dropout(q, k, v, causal, 0.5, p=p, seed=77)
    ob, lb = brute(q, k, v, causal, 0.5, z, oracle.dropout_threshold(p))
    np.testing.assert_allclose(o, ob, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lb, rtol=0, atol=1e-13)


def test_average_over_seeds_is_unbiased():
    q, k, v = (RNG.standard_normal((1, 16, 4)) for _ in range(3))
    exact, _ = oracle.fwd(q, k, v, False, 0.5)
    mean = np.mean([oracle.fwd_dropout(q, k, v, False, 0.5, p=0.5, seed=s)[0]
                    for s in range(600)], axis=0)
    assert np.abs(mean - exact).max() < 0.15


@pytest.mark.parametrize("causal", [False, True])
def test_backward_equals_fp64_autograd(causal):
    BH, N, d, p, seed = 2, 30, 5, 0.3, 9
    q, k, v, do = (RNG.standard_normal((BH, N, d)) for _ in range(4))
    got = oracle.bwd_dropout(q, k, v, do, causal, 0.45, p, seed)
    z = torch.tensor(oracle.dropout_mask(BH, N, seed, p), dtype=torch.float64)
    t = oracle.dropout_threshold(p)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    s = 0.45 * tq @ tk.transpose(-1, -2)
    if causal:
        s = s.masked_fill(~torch.ones(N, N, dtype=torch.bool).tril(), float("-inf"))
    ((torch.softmax(s, -1) * z * (256.0 / t)) @ tv * torch.tensor(do)).sum().backward()
    for mine, ref in zip(got, (tq.grad, tk.grad, tv.grad)):
        np.testing.assert_allclose(mine, ref.numpy(), rtol=0, atol=1e-12)


MUTANTS = {
    "kept values not rescaled": ("oi[t] += s[j] * inv_keep * vj[t];", "oi[t] += s[j] * vj[t];"),
    "byte index from the low bits only": ("uint32_t byte = (w[(j & 15) >> 2] >> (8 * (j & 3))) & 0xFFu;",
                                          "uint32_t byte = (w[0] >> (8 * (j & 3))) & 0xFFu;"),
    "counter words swapped": ("uint32_t ctr[4] = {(uint32_t)(j >> 4), (uint32_t)i, (uint32_t)bh, 0u};",
                              "uint32_t ctr[4] = {(uint32_t)i, (uint32_t)(j >> 4), (uint32_t)bh, 0u};"),
    "Philox multiplier": ("uint32_t lo0 = mulhilo32(0xD2511F53u, c0, &hi0);",
                          "uint32_t lo0 = mulhilo32(0xD2511F55u, c0, &hi0);"),
    "dP not masked": ("double dpij = zj * dot(doi, vj, d);", "double dpij = inv_keep * dot(doi, vj, d);"),
    "dV not masked": ("dvj[t] += p[j] * zj * doi[t];", "dvj[t] += p[j] * doi[t];"),
}


def _build(text):
    dd = tempfile.mkdtemp(prefix="oracle_dropout_mutant_")
    c, so = os.path.join(dd, "m.c"), os.path.join(dd, "m.so")
    with open(c, "w") as f:
        f.write(text)
    subprocess.run(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-o", so, c, "-lm"], check=True)
    L = ctypes.CDLL(so)
    dp, lp = ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int64)
    u32p = ctypes.POINTER(ctypes.c_uint32)
    i64, ci, cd, u64 = ctypes.c_int64, ctypes.c_int, ctypes.c_double, ctypes.c_uint64
    L.oracle_philox4x32_10.argtypes = [u32p, u32p, u32p]
    L.oracle_dropout_mask.argtypes = [i64, i64, u64, ci, ctypes.POINTER(ctypes.c_uint8)]
    L.oracle_fwd_dropout.argtypes = [dp, dp, dp, dp, dp, i64, i64, i64, ci, cd, u64, ci]
    L.oracle_bwd_dropout_heads.argtypes = [dp, dp, dp, dp, i64, i64, i64, ci, cd, u64, ci, lp,
                                           i64, dp, dp, dp]
    return L


def _pins_pass(L):
    P = lambda a, t=ctypes.c_double: a.ctypes.data_as(ctypes.POINTER(t))
    for ctr, key, want in kat_vectors():
        c = (ctypes.c_uint32 * 4)(*ctr)
        k = (ctypes.c_uint32 * 2)(*key)
        out = (ctypes.c_uint32 * 4)()
        L.oracle_philox4x32_10(c, k, out)
        if list(out) != want:
            return False
    rng = np.random.default_rng(3)
    BH, N, d, p, seed, scale = 2, 40, 4, 0.4, 11, 0.6
    t = oracle.dropout_threshold(p)
    q, k, v, do = (rng.standard_normal((BH, N, d)) for _ in range(4))
    for causal in (0, 1):
        z = np.empty((BH, N, N), np.uint8)
        L.oracle_dropout_mask(BH, N, seed, t, P(z, ctypes.c_uint8))
        if not np.array_equal(z, oracle.dropout_mask(BH, N, seed, p)):  # the committed mask
            return False
        o, lse = np.empty_like(q), np.empty((BH, N))
        L.oracle_fwd_dropout(P(q), P(k), P(v), P(o), P(lse), BH, N, d, causal, scale, seed, t)
        ob, lb = brute(q, k, v, causal, scale, z, t)
        if not (np.allclose(o, ob, atol=1e-12) and np.allclose(lse, lb, atol=1e-12)):
            return False
        heads = np.arange(BH, dtype=np.int64)
        dq, dk, dv = (np.empty_like(q) for _ in range(3))
        L.oracle_bwd_dropout_heads(P(q), P(k), P(v), P(do), BH, N, d, causal, scale, seed, t,
                                   heads.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), BH,
                                   P(dq), P(dk), P(dv))
        tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
        s = scale * tq @ tk.transpose(-1, -2)
        if causal:
            s = s.masked_fill(~torch.ones(N, N, dtype=torch.bool).tril(), float("-inf"))
        zt = torch.tensor(z, dtype=torch.float64)
        ((torch.softmax(s, -1) * zt * (256.0 / t)) @ tv * torch.tensor(do)).sum().backward()
        for mine, ref in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
            if not np.allclose(mine, ref.numpy(), atol=1e-11):
                return False
    return True


def test_unmutated_dropout_copy_passes():
    with open(SRC) as f:
        assert _pins_pass(_build(f.read()))


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_dropout_mutant_is_caught(name):
    old, new = MUTANTS[name]
    with open(SRC) as f:
        text = f.read()
    assert text.count(old) == 1, f"mutation site missing or ambiguous: {old}"
    assert not _pins_pass(_build(text.replace(old, new, 1)))
