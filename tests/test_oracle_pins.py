"""Pins of the fp64 oracle to facts outside itself (CPU only).

Each test ties the oracle to something the pages or mathematics fix:
brute force on the full N x N matrix with library softmax/logsumexp,
rows of P summing to one, the online recurrence equalling two passes,
key permutation invariance, constant V, closed forms, hand-worked
examples with exact values (tests/golden/worked_examples.txt), central
finite differences and fp64 autograd of the brute-force definition for the
gradients.
"""

import math

import numpy as np
import pytest
import scipy.special as sps
import torch

import oracle
from helpers import load_worked_examples

RNG = np.random.default_rng(12345)


def rand(*shape, scale=1.0):
    return RNG.standard_normal(shape) * scale


def brute(q, k, v, causal, scale):
    """Materialise S for every head and use scipy's softmax/logsumexp."""
    s = scale * np.einsum("bhid,bhjd->bhij", q, k)
    if causal:
        N = q.shape[-2]
        s = np.where(np.tril(np.ones((N, N), bool)), s, -np.inf)
    return np.einsum("bhij,bhjd->bhid", sps.softmax(s, axis=-1), v), sps.logsumexp(s, axis=-1)


SHAPES = [(1, 1, 1, 1), (1, 2, 5, 3), (2, 1, 17, 8), (1, 3, 33, 16), (1, 1, 64, 64)]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("causal", [False, True])
def test_fwd_equals_bruteforce(shape, causal):
    q, k, v = rand(*shape), rand(*shape), rand(*shape)
    scale = 1.0 / math.sqrt(shape[-1])
    o, lse = oracle.fwd(q, k, v, causal, scale)
    ob, lb = brute(q, k, v, causal, scale)
    np.testing.assert_allclose(o, ob, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse, lb, rtol=0, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_rows_of_p_sum_to_one(causal):
    # With d = N and V = identity, O is exactly the probability matrix P.
    N = 24
    q, k = rand(1, 1, N, N), rand(1, 1, N, N)
    v = np.eye(N)[None, None]
    p, _ = oracle.fwd(q, k, v, causal, 0.3)
    np.testing.assert_allclose(p.sum(-1), 1.0, rtol=0, atol=1e-12)
    assert (p >= 0).all()
    if causal:
        assert np.all(np.triu(p[0, 0], 1) == 0.0)      # no weight on future keys
        assert p[0, 0, 0, 0] == pytest.approx(1.0, abs=1e-15)


@pytest.mark.parametrize("block", [1, 7, 16])
@pytest.mark.parametrize("causal", [False, True])
def test_online_recurrence_equals_two_pass(block, causal):
    shape = (2, 2, 45, 8)
    q, k, v = rand(*shape, scale=2.0), rand(*shape, scale=2.0), rand(*shape)
    o2, l2 = oracle.fwd(q, k, v, causal, 0.5)
    o1, l1 = oracle.fwd_online(q, k, v, causal, 0.5, block)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-12)


def test_key_permutation_invariance():
    shape = (1, 2, 40, 16)
    q, k, v = rand(*shape), rand(*shape), rand(*shape)
    perm = RNG.permutation(shape[2])
    o, lse = oracle.fwd(q, k, v, False, 0.25)
    op, lp = oracle.fwd(q, k[:, :, perm], v[:, :, perm], False, 0.25)
    np.testing.assert_allclose(op, o, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lp, lse, rtol=0, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_constant_v_gives_constant_output(causal):
    shape = (1, 1, 30, 6)
    q, k = rand(*shape, scale=3.0), rand(*shape, scale=3.0)
    c = rand(6)
    v = np.broadcast_to(c, shape).copy()
    o, _ = oracle.fwd(q, k, v, causal, 1.0)
    np.testing.assert_allclose(o, np.broadcast_to(c, shape), rtol=0, atol=1e-13)


def test_single_key_closed_form():
    q, k, v = rand(2, 3, 1, 8), rand(2, 3, 1, 8), rand(2, 3, 1, 8)
    for causal in (False, True):
        o, lse = oracle.fwd(q, k, v, causal, 0.7)
        np.testing.assert_array_equal(o, v)
        np.testing.assert_allclose(lse, 0.7 * (q * k).sum(-1), rtol=0, atol=1e-14)


def test_causal_row_zero_closed_form():
    shape = (1, 2, 19, 4)
    q, k, v = rand(*shape), rand(*shape), rand(*shape)
    o, lse = oracle.fwd(q, k, v, True, 0.9)
    np.testing.assert_array_equal(o[:, :, 0], v[:, :, 0])
    np.testing.assert_allclose(lse[:, :, 0], 0.9 * (q[:, :, 0] * k[:, :, 0]).sum(-1), atol=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_zero_query_gives_mean_of_visible_values(causal):
    N, d = 21, 5
    q = np.zeros((1, 1, N, d))
    k, v = rand(1, 1, N, d), rand(1, 1, N, d)
    o, lse = oracle.fwd(q, k, v, causal, 1.0)
    if causal:
        mean = np.cumsum(v[0, 0], axis=0) / np.arange(1, N + 1)[:, None]
        cnt = np.arange(1, N + 1)
    else:
        mean = np.broadcast_to(v[0, 0].mean(0), (N, d))
        cnt = np.full(N, N)
    np.testing.assert_allclose(o[0, 0], mean, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse[0, 0], np.log(cnt), rtol=0, atol=1e-14)


WORKED = load_worked_examples()


def test_worked_examples_fixture_is_complete():
    names = [e["name"] for e in WORKED]
    assert names == ["two keys, non-causal", "two keys, causal", "two keys, scale 1/2",
                     "three keys, non-causal", "three keys, causal"]
    for e in WORKED:
        assert {"causal", "scale", "q", "k", "v", "o", "lse"} <= set(e)


@pytest.mark.parametrize("ex", WORKED, ids=lambda e: e["name"])
def test_worked_example(ex):
    """Exact values worked by hand from the definition (no numeric example is
    printed on the pages); the derivations are in the fixture's header."""
    N = ex["q"].size
    t = {k: ex[k].reshape(1, 1, N, 1) for k in ("q", "k", "v")}
    causal, scale = bool(ex["causal"][0]), float(ex["scale"][0])
    o, lse = oracle.fwd(t["q"], t["k"], t["v"], causal, scale)
    np.testing.assert_allclose(o.ravel(), ex["o"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse.ravel(), ex["lse"], rtol=0, atol=1e-14)
    if "dout" in ex:
        dq, dk, dv = oracle.bwd(t["q"], t["k"], t["v"], ex["dout"].reshape(1, 1, N, 1), causal,
                                scale)
        np.testing.assert_allclose(dq.ravel(), ex["dq"], rtol=0, atol=1e-14)
        np.testing.assert_allclose(dk.ravel(), ex["dk"], rtol=0, atol=1e-14)
        np.testing.assert_allclose(dv.ravel(), ex["dv"], rtol=0, atol=1e-14)


def test_rows_subset_matches_full():
    shape = (2, 2, 37, 8)
    q, k, v = rand(*shape), rand(*shape), rand(*shape)
    for causal in (False, True):
        o, lse = oracle.fwd(q, k, v, causal, 0.3)
        rows = np.array([0, 5, 36, 37, 80, 147])
        orr, lr = oracle.fwd_rows(q, k, v, causal, 0.3, rows)
        np.testing.assert_array_equal(orr, o.reshape(-1, 8)[rows])
        np.testing.assert_array_equal(lr, lse.reshape(-1)[rows])


def _loss(q, k, v, dout, causal, scale):
    o, _ = oracle.fwd(q, k, v, causal, scale)
    return float((o * dout).sum())


@pytest.mark.parametrize("causal", [False, True])
def test_backward_central_differences(causal):
    shape = (1, 1, 9, 4)
    q, k, v, dout = (rand(*shape) for _ in range(4))
    scale = 0.6
    dq, dk, dv = oracle.bwd(q, k, v, dout, causal, scale)
    h = 1e-5
    for x, g in ((q, dq), (k, dk), (v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            old = x[idx]
            x[idx] = old + h
            fp = _loss(q, k, v, dout, causal, scale)
            x[idx] = old - h
            fm = _loss(q, k, v, dout, causal, scale)
            x[idx] = old
            num[idx] = (fp - fm) / (2 * h)
        err = np.linalg.norm(num - g) / np.linalg.norm(g)
        assert err <= 1e-6, err


@pytest.mark.parametrize("shape", [(1, 2, 16, 8), (2, 1, 33, 16)])
@pytest.mark.parametrize("causal", [False, True])
def test_backward_equals_fp64_autograd(shape, causal):
    q, k, v, dout = (rand(*shape) for _ in range(4))
    scale = 1.0 / math.sqrt(shape[-1])
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    s = scale * tq @ tk.transpose(-1, -2)
    if causal:
        N = shape[2]
        s = s.masked_fill(~torch.ones(N, N, dtype=torch.bool).tril(), float("-inf"))
    o = torch.softmax(s, dim=-1) @ tv
    (o * torch.tensor(dout)).sum().backward()
    dq, dk, dv = oracle.bwd(q, k, v, dout, causal, scale)
    for mine, ref in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad)):
        np.testing.assert_allclose(mine, ref.numpy(), rtol=0, atol=1e-12)


def test_backward_causal_last_key_sees_only_last_row():
    # Under the causal mask, key N-1 is visible to query N-1 only, so its
    # gradients cannot depend on dO of earlier rows.
    shape = (1, 1, 12, 4)
    q, k, v, dout = (rand(*shape) for _ in range(4))
    _, dk, dv = oracle.bwd(q, k, v, dout, True, 0.5)
    dout2 = dout.copy()
    dout2[:, :, :-1] = rand(1, 1, 11, 4, scale=100.0)
    _, dk2, dv2 = oracle.bwd(q, k, v, dout2, True, 0.5)
    np.testing.assert_allclose(dk2[:, :, -1], dk[:, :, -1], atol=1e-13)
    np.testing.assert_allclose(dv2[:, :, -1], dv[:, :, -1], atol=1e-13)
    # and dV_{N-1} = P_{N-1,N-1} dO_{N-1}
    p_last = np.exp(0.5 * (q[0, 0, -1] @ k[0, 0, -1]) - oracle.fwd(q, k, v, True, 0.5)[1][0, 0, -1])
    np.testing.assert_allclose(dv[0, 0, -1], p_last * dout[0, 0, -1], atol=1e-13)


def test_backward_head_subset_matches_full():
    shape = (2, 2, 20, 8)
    q, k, v, dout = (rand(*shape) for _ in range(4))
    full = oracle.bwd(q, k, v, dout, True, 0.4)
    sub = oracle.bwd_heads(q, k, v, dout, True, 0.4, heads=[3, 1])
    for f, s in zip(full, sub):
        fr = f.reshape(4, 20, 8)
        np.testing.assert_allclose(s[0], fr[3], atol=1e-14)
        np.testing.assert_allclose(s[1], fr[1], atol=1e-14)
