"""attn_bwd_noalloc — the backward for callers that cannot allocate.

Some callers hold their input and output tensors but have no way to get a
scratch workspace: a plugin living inside a framework that owns every device
allocation, or a latency-critical loop that must not call cudaMalloc once it
runs.  For them the library keeps a fixed scratch array of its own on each
device.  These tests call that entry point through the C ABI and check that
it gives the same gradients as attn_bwd with a caller-supplied workspace,
twice in a row (the second call starts from whatever the first left in the
shared array), that those gradients also match the fp64 oracle, and that a
problem too big for the array is refused.

This file is collected last on purpose, and passes alone or after the rest.
"""

import ctypes

import numpy as np
import pytest

import oracle
from helpers import GRAD_REL_L2, check_grads, default_scale, inputs, rel_l2, to_device

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from io_aware_exact_30_b200 import attn  # noqa: E402


@pytest.mark.parametrize("B,H,N,d,causal,dtype", [(2, 3, 700, 128, False, "bf16"),
                                                  (1, 4, 1029, 64, True, "fp16")])
def test_noalloc_matches_workspace_backward_twice(B, H, N, d, causal, dtype):
    assert attn.attn_bwd_workspace_bytes(B, H, N, d) <= attn.NOALLOC_SCRATCH_BYTES
    arrs, f64 = inputs(B, H, N, d, dtype=dtype, seed=N, with_dout=True)
    q, k, v, do = (to_device(a, dtype) for a in arrs)
    o, lse = attn.forward(q, k, v, causal)
    ref = attn.backward(q, k, v, o, lse, do, causal)  # existing entry point, own workspace
    torch.cuda.synchronize()
    ref = [t.double().cpu().numpy() for t in ref]
    for call in range(2):
        dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
        attn.attn_bwd_noalloc(q, k, v, o, lse, do, dq, dk, dv, causal)
        torch.cuda.synchronize()
        assert attn.attn_last_device_status() == 0
        for name, got, want in zip(("dQ", "dK", "dV"), (dq, dk, dv), ref):
            got = got.double().cpu().numpy()
            assert np.all(np.isfinite(got)), (call, name)
            err = rel_l2(got, want)
            assert err <= GRAD_REL_L2, f"call {call} {name} rel-L2 {err}"
        if call == 1:  # and against the oracle, on the last head
            exact = oracle.bwd_heads(*f64, causal, default_scale(d), heads=[B * H - 1])
            got = [t.double().cpu().numpy().reshape(B * H, N, d)[-1:] for t in (dq, dk, dv)]
            check_grads(got, exact, f"noalloc {(B, H, N, d, causal, dtype)}")


def test_noalloc_refuses_problems_larger_than_its_scratch():
    L = attn.lib()
    t = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    p = ctypes.c_void_p(t.data_ptr())
    B, H, N, d = 4, 16, 4096, 128  # needs about 135 MB of scratch
    assert attn.attn_bwd_workspace_bytes(B, H, N, d) > attn.NOALLOC_SCRATCH_BYTES
    rc = L.attn_bwd_noalloc(p, p, p, p, p, p, p, p, p, B, H, N, d, 1, 0.088, 0, None)
    assert rc == -10 and "scratch" in attn.strerror(rc)
    assert attn.attn_last_device_status() == 0
