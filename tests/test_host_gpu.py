"""End-to-end calls from host buffers (attn_sdpa_host): results equal the
device-buffer calls on the same inputs and the oracle (needs a B200)."""

import math

import numpy as np
import pytest

import oracle
from helpers import GRAD_REL_L2, inputs, rel_l2

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from io_aware_exact_30_b200 import attn  # noqa: E402


def _host(arrs):
    return [torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).pin_memory() for a in arrs]


@pytest.mark.parametrize("B,H,N,d,causal,hc", [
    (1, 3, 300, 128, True, 1), (2, 5, 777, 64, False, 2), (1, 7, 1000, 128, True, 0),
    (1, 1, 129, 64, True, 0), (2, 4, 256, 128, False, 3)])
def test_host_call_equals_device_call_and_oracle(B, H, N, d, causal, hc):
    arrs, f64 = inputs(B, H, N, d, seed=B * 100 + N, with_dout=True)
    host = _host(arrs)
    ho = torch.empty_like(host[0]).pin_memory()
    hl = torch.empty(B, H, N, dtype=torch.float32).pin_memory()
    hdq, hdk, hdv = (torch.empty_like(host[0]).pin_memory() for _ in range(3))
    scratch = torch.empty(attn.attn_sdpa_host_scratch_bytes(B, H, N, d, True, hc),
                          dtype=torch.uint8, device="cuda")
    attn.attn_sdpa_host(*host, ho, hl, hdq, hdk, hdv, scratch, causal, heads_per_chunk=hc)
    torch.cuda.synchronize()
    assert attn.attn_last_device_status() == 0
    dev = [t.cuda() for t in host]
    o, lse = attn.forward(*dev[:3], causal)
    dq, dk, dv = attn.backward(*dev[:3], o, lse, dev[3], causal)
    torch.cuda.synchronize()
    assert torch.equal(ho, o.cpu()) and torch.equal(hl, lse.cpu())
    assert torch.equal(hdk, dk.cpu()) and torch.equal(hdv, dv.cpu())
    assert rel_l2(hdq.double().numpy(), dq.double().cpu().numpy()) < 1e-3
    b, h = B - 1, H - 1
    sel = [x[b:b + 1, h:h + 1] for x in f64]
    ref = oracle.bwd(*sel, causal, 1 / math.sqrt(d))
    for t, r in zip((hdq, hdk, hdv), ref):
        assert rel_l2(t[b:b + 1, h:h + 1].double().numpy(), r) <= GRAD_REL_L2


def test_host_forward_only():
    B, H, N, d, causal = 2, 3, 400, 128, True
    arrs, _ = inputs(B, H, N, d, seed=9)
    host = _host(arrs)
    ho = torch.empty_like(host[0]).pin_memory()
    hl = torch.empty(B, H, N, dtype=torch.float32).pin_memory()
    scratch = torch.empty(attn.attn_sdpa_host_scratch_bytes(B, H, N, d, False, 2),
                          dtype=torch.uint8, device="cuda")
    attn.attn_sdpa_host(*host, None, ho, hl, None, None, None, scratch, causal,
                        heads_per_chunk=2)
    torch.cuda.synchronize()
    o, lse = attn.forward(*[t.cuda() for t in host], causal)
    assert torch.equal(ho, o.cpu()) and torch.equal(hl, lse.cpu())


def test_host_call_rejects_small_scratch():
    B, H, N, d = 1, 2, 128, 64
    arrs, _ = inputs(B, H, N, d, seed=3, with_dout=True)
    host = _host(arrs)
    outs = [torch.empty_like(host[0]).pin_memory() for _ in range(3)]
    need = attn.attn_sdpa_host_scratch_bytes(B, H, N, d, True, 0)
    scratch = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(attn.AttnError):
        attn.attn_sdpa_host(*host, None, None, *outs, scratch, True)
