"""Pins of the causal linear attention oracle (CPU only).

O_i = scale sum_{j <= i} (q_i . k_j) v_j (the plainest reading of the linear
attention of "Lightning Attention-2" (chatpaper.ai summary) and "Gated Linear
Attention Transformers with Hardware-Efficient Training" (nubint.ai
review)), pinned to: the lower-triangular matrix product written with
numpy, the chunked form (in-chunk products plus a running d x d state,
the pages' intra-/inter-block split) for several chunk sizes, closed forms
(one token; zero queries; constant values), linearity in V, and planted
mistakes in a compiled copy of the source.
"""

import ctypes
import os
import subprocess
import tempfile

import numpy as np
import pytest

import oracle

RNG = np.random.default_rng(99)
SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle",
                   "attn_oracle.c")


def brute(q, k, v, scale):
    N = q.shape[-2]
    a = scale * np.einsum("...id,...jd->...ij", q, k) * np.tril(np.ones((N, N)))
    return a @ v


@pytest.mark.parametrize("shape", [(1, 1, 1, 3), (2, 3, 17, 5), (1, 2, 64, 16)])
def test_equals_masked_matrix_product(shape):
    q, k, v = (RNG.standard_normal(shape) for _ in range(3))
    np.testing.assert_allclose(oracle.linear_attn(q, k, v, 0.3), brute(q, k, v, 0.3),
                               rtol=0, atol=1e-12)


@pytest.mark.parametrize("chunk", [1, 7, 16, 128])
def test_chunked_form_equals_definition(chunk):
    q, k, v = (RNG.standard_normal((2, 50, 6)) for _ in range(3))
    np.testing.assert_allclose(oracle.linear_attn_chunked(q, k, v, 0.5, chunk),
                               oracle.linear_attn(q, k, v, 0.5), rtol=0, atol=1e-12)


def test_closed_forms_and_linearity():
    q, k, v = (RNG.standard_normal((1, 1, 20, 4)) for _ in range(3))
    o = oracle.linear_attn(q, k, v, 0.7)
    np.testing.assert_allclose(o[0, 0, 0], 0.7 * (q[0, 0, 0] @ k[0, 0, 0]) * v[0, 0, 0], atol=1e-14)
    assert np.all(oracle.linear_attn(np.zeros_like(q), k, v, 0.7) == 0.0)
    c = np.full_like(v, 2.5)
    want = 0.7 * np.cumsum(q[0, 0] @ k[0, 0].T * np.tril(np.ones((20, 20))), axis=1)[:, -1]
    np.testing.assert_allclose(oracle.linear_attn(q, k, c, 0.7)[0, 0, :, 1], 2.5 * want, atol=1e-12)
    np.testing.assert_allclose(oracle.linear_attn(q, k, 3 * v, 0.7), 3 * o, rtol=1e-13, atol=1e-13)


MUTANTS = {
    "future keys included": ("for (int64_t j = 0; j <= i; ++j) {\n                double a = scale",
                             "for (int64_t j = 0; j < N; ++j) {\n                double a = scale"),
    "diagonal excluded": ("for (int64_t j = 0; j <= i; ++j) {\n                double a = scale",
                          "for (int64_t j = 0; j < i; ++j) {\n                double a = scale"),
    "scale dropped": ("double a = scale * dot(qi, k + (bh * N + j) * d, d);",
                      "double a = dot(qi, k + (bh * N + j) * d, d);"),
    "value row of the query": ("const double* vj = v + (bh * N + j) * d;\n                for (int64_t t = 0; t < d; ++t) oi[t] += a * vj[t];",
                               "const double* vj = v + (bh * N + i) * d;\n                for (int64_t t = 0; t < d; ++t) oi[t] += a * vj[t];"),
}


def _build(text):
    dd = tempfile.mkdtemp(prefix="oracle_lin_mutant_")
    c, so = os.path.join(dd, "m.c"), os.path.join(dd, "m.so")
    with open(c, "w") as f:
        f.write(text)
    subprocess.run(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-o", so, c, "-lm"], check=True)
    L = ctypes.CDLL(so)
    dp, i64 = ctypes.POINTER(ctypes.c_double), ctypes.c_int64
    L.oracle_linear_attn.argtypes = [dp, dp, dp, dp, i64, i64, i64, ctypes.c_double]
    return L


def _pins_pass(L):
    P = lambda a: a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))
    rng = np.random.default_rng(4)
    q, k, v = (rng.standard_normal((2, 23, 5)) for _ in range(3))
    o = np.empty_like(q)
    L.oracle_linear_attn(P(q), P(k), P(v), P(o), 2, 23, 5, 0.4)
    return np.allclose(o, brute(q, k, v, 0.4), atol=1e-12)


def test_unmutated_linear_copy_passes():
    with open(SRC) as f:
        assert _pins_pass(_build(f.read()))


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_linear_mutant_is_caught(name):
    old, new = MUTANTS[name]
    with open(SRC) as f:
        text = f.read()
    assert text.count(old) == 1, f"mutation site missing or ambiguous: {old}"
    assert not _pins_pass(_build(text.replace(old, new, 1)))
