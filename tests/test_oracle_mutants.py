"""Planted mistakes in a copy of the oracle source must fail the pins.

Each mutant is a plausible slip (a dropped term, a wrong sign or index, a
transposed operand); the copy is compiled to a temporary library on the
CPU and checked with the same independent references the pins use
(brute-force softmax and fp64 autograd), and separately with the hand-worked
exact examples of tests/golden/worked_examples.txt alone.  The committed
oracle is untouched.
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

from helpers import load_worked_examples

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "attn_oracle.c")

MUTANTS = {
    "scale dropped in scores": ("s[j] = scale * dot(qi, K + j * d, d);", "s[j] = dot(qi, K + j * d, d);"),
    "max not subtracted": ("s[j] = exp(s[j] - M);", "s[j] = exp(s[j]);"),
    "LSE without log": ("return M + log(Z);", "return M + Z;"),
    "causal excludes diagonal": ("return causal ? i + 1 : N;", "return causal ? (i > 0 ? i : 1) : N;"),
    "dS sign flipped": ("double dsij = p[j] * (dpij - Di);", "double dsij = p[j] * (Di - dpij);"),
    "D term dropped": ("double dsij = p[j] * (dpij - Di);", "double dsij = p[j] * dpij;"),
    "dK uses k instead of q": ("dkj[t] += scale * dsij * qi[t];", "dkj[t] += scale * dsij * kj[t];"),
    "dV transposed operand": ("dvj[t] += p[j] * doi[t];", "dvj[t] += p[j] * vj[t];"),
    "dQ scale dropped": ("dqi[t] += scale * dsij * kj[t];", "dqi[t] += dsij * kj[t];"),
}


def _build(text):
    d = tempfile.mkdtemp(prefix="oracle_mutant_")
    c, so = os.path.join(d, "m.c"), os.path.join(d, "m.so")
    with open(c, "w") as f:
        f.write(text)
    subprocess.run(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-o", so, c, "-lm"], check=True)
    L = ctypes.CDLL(so)
    dp, lp = ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int64)
    i64, ci, cd = ctypes.c_int64, ctypes.c_int, ctypes.c_double
    L.oracle_fwd.argtypes = [dp, dp, dp, dp, dp, i64, i64, i64, ci, cd]
    L.oracle_bwd_heads.argtypes = [dp, dp, dp, dp, i64, i64, i64, ci, cd, lp, i64, dp, dp, dp]
    return L


def _pins_pass(L):
    rng = np.random.default_rng(5)
    P = lambda a: a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))
    for causal in (0, 1):
        BH, N, dd, scale = 2, 11, 4, 0.7
        q, k, v, do = (rng.standard_normal((BH, N, dd)) for _ in range(4))
        o, lse = np.empty_like(q), np.empty((BH, N))
        L.oracle_fwd(P(q), P(k), P(v), P(o), P(lse), BH, N, dd, causal, scale)
        s = scale * q @ k.transpose(0, 2, 1)
        if causal:
            s = np.where(np.tril(np.ones((N, N), bool)), s, -np.inf)
        if not (np.allclose(o, sps.softmax(s, -1) @ v, atol=1e-12) and
                np.allclose(lse, sps.logsumexp(s, -1), atol=1e-12)):
            return False
        heads = np.arange(BH, dtype=np.int64)
        dq, dk, dv = (np.empty_like(q) for _ in range(3))
        L.oracle_bwd_heads(P(q), P(k), P(v), P(do), BH, N, dd, causal, scale,
                           heads.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), BH, P(dq), P(dk), P(dv))
        tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
        ts = scale * tq @ tk.transpose(-1, -2)
        if causal:
            ts = ts.masked_fill(~torch.ones(N, N, dtype=torch.bool).tril(), float("-inf"))
        (torch.softmax(ts, -1) @ tv * torch.tensor(do)).sum().backward()
        for mine, ref in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
            if not np.allclose(mine, ref.numpy(), atol=1e-11):
                return False
    return True


def test_unmutated_copy_passes():
    with open(SRC) as f:
        assert _pins_pass(_build(f.read()))


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    old, new = MUTANTS[name]
    with open(SRC) as f:
        text = f.read()
    assert text.count(old) >= 1, f"mutation site missing: {old}"
    assert not _pins_pass(_build(text.replace(old, new, 1)))


def _worked_pass(L):
    """The hand-worked examples, through the library's own entry points."""
    P = lambda a: a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))
    for ex in load_worked_examples():
        N = ex["q"].size
        q, k, v = (np.ascontiguousarray(ex[n], dtype=np.float64) for n in ("q", "k", "v"))
        causal, scale = int(ex["causal"][0]), float(ex["scale"][0])
        o, lse = np.empty(N), np.empty(N)
        L.oracle_fwd(P(q), P(k), P(v), P(o), P(lse), 1, N, 1, causal, scale)
        if not (np.allclose(o, ex["o"], rtol=0, atol=1e-13) and
                np.allclose(lse, ex["lse"], rtol=0, atol=1e-13)):
            return False
        if "dout" in ex:
            do = np.ascontiguousarray(ex["dout"], dtype=np.float64)
            dq, dk, dv = np.empty(N), np.empty(N), np.empty(N)
            heads = np.zeros(1, dtype=np.int64)
            L.oracle_bwd_heads(P(q), P(k), P(v), P(do), 1, N, 1, causal, scale,
                               heads.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), 1, P(dq),
                               P(dk), P(dv))
            for mine, want in ((dq, ex["dq"]), (dk, ex["dk"]), (dv, ex["dv"])):
                if not np.allclose(mine, want, rtol=0, atol=1e-13):
                    return False
    return True


def test_unmutated_copy_passes_worked_examples():
    with open(SRC) as f:
        assert _worked_pass(_build(f.read()))


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught_by_worked_examples(name):
    old, new = MUTANTS[name]
    with open(SRC) as f:
        text = f.read()
    assert not _worked_pass(_build(text.replace(old, new, 1)))
