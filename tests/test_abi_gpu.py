"""C-ABI behaviour on a B200: argument errors, the bounded-wait timeout
path, and that calls leave the context usable (needs a GPU)."""

import ctypes

import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from io_aware_exact_30_b200 import attn  # noqa: E402


def _t(*shape, dtype=torch.bfloat16):
    return torch.zeros(*shape, dtype=dtype, device="cuda")


def test_argument_errors_return_codes():
    L = attn.lib()
    q = _t(1, 1, 16, 64)
    lse = torch.zeros(1, 1, 16, dtype=torch.float32, device="cuda")
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    args = lambda **kw: dict(dict(B=1, H=1, N=16, d=64, causal=0, scale=0.125, dtype=0), **kw)

    def call(**kw):
        a = args(**kw)
        return L.attn_fwd(P(q), P(q), P(q), P(q), P(lse), a["B"], a["H"], a["N"], a["d"],
                          a["causal"], a["scale"], a["dtype"], None)

    assert call(d=96) == -3
    assert call(N=0) == -2
    assert call(B=0) == -2
    assert call(dtype=7) == -5
    assert call(scale=float("nan")) == -9
    assert call(scale=-1.0) == -9
    # misaligned pointer
    rc = L.attn_fwd(ctypes.c_void_p(q.data_ptr() + 2), P(q), P(q), P(q), P(lse), 1, 1, 16, 64, 0,
                    0.125, 0, None)
    assert rc == -4
    # host pointer
    h = torch.zeros(1, 1, 16, 64, dtype=torch.bfloat16).pin_memory()
    rc = L.attn_fwd(P(h), P(q), P(q), P(q), P(lse), 1, 1, 16, 64, 0, 0.125, 0, None)
    assert rc == -6
    assert attn.attn_last_device_status() == 0


def test_bounded_wait_times_out_and_context_survives():
    attn.attn_selftest_wait_timeout(20_000)  # 20 ms wait on a barrier nothing completes
    assert attn.attn_last_device_status() == -8
    assert attn.attn_last_device_status() == 0  # the word is cleared on read
    q = torch.randn(1, 2, 200, 64, device="cuda", dtype=torch.bfloat16)
    o, lse = attn.forward(q, q, q, True)
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all() and attn.attn_last_device_status() == 0
