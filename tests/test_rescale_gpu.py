"""Forward and backward parity on inputs whose row maxima keep growing along
the keys (needs a B200).

The forward keeps its running max until a key tile's row max exceeds it by
more than 2^8, then moves it and rescales the output accumulator held in
tensor memory (the online-softmax recurrence: "Is a full day of context
better than ten minutes?" (marketmaker.cc), sections "Flash Attention
algorithm" and "online softmax recurrence").  Gaussian inputs at the
workloads' sigma never trigger that; the ``steps`` and ``shared`` patterns of
``helpers.rescale_inputs`` do, in most rows, several times per row, and with
warps whose rows disagree on whether to move.  tests/test_rescale_inputs.py
checks on the CPU that they do.  O and LSE are compared element by element
with the fp64 oracle at the forward tolerances.

The backward is compared too (relative L2 of dQ, dK, dV) on the ``steps``
inputs only.  On ``shared`` the causal softmax is saturated (each row's own
key carries almost all the weight), so the exact dS = P (dP - D) nearly
vanishes and the method's D = rowsum(dO O), taken from the stored
half-precision O, is off by more than the gradient itself: computing D from
the oracle's own O rounded to bf16 already moves dQ by 79 % (relative L2) at
d = 128.  That is the conditioning of the recompute-from-stored-O backward,
not of this implementation; the forward on those inputs is still checked.
"""

import numpy as np
import pytest

import oracle
from helpers import (check_fwd, check_grads, default_scale, mixed_warps, rescale_inputs,
                     rescale_moves, to_device)

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from io_aware_exact_30_b200 import attn  # noqa: E402

CASES = [(p, d, dt, c) for p in ("steps", "shared") for d in (64, 128) for dt in ("bf16", "fp16")
         for c in (True, False) if not (p == "shared" and not c)]


@pytest.mark.parametrize("pattern,d,dtype,causal", CASES)
def test_rescale_branch_fwd_bwd_parity(pattern, d, dtype, causal):
    B, H, N = 1, 2, 700  # five full 128-key tiles and a ragged tail of 60
    stored, f64 = rescale_inputs(pattern, B, H, N, d, dtype=dtype, seed=3)
    scale = default_scale(d)
    # the branch is reached on these inputs (at 64- and 128-key tiles alike)
    moved, kept = rescale_moves(f64[0][0, 0], f64[1][0, 0], causal, scale, 128)
    assert moved.sum(1).astype(bool).sum() >= 250
    if pattern == "steps":
        assert (moved.sum(1) >= 2).sum() >= 150 and mixed_warps(moved, kept) >= 20

    q, k, v, do = (to_device(a, dtype) for a in stored)
    o, lse = attn.forward(q, k, v, causal, scale)
    dq, dk, dv = attn.backward(q, k, v, o, lse, do, causal, scale)
    torch.cuda.synchronize()
    assert attn.attn_last_device_status() == 0
    o_ref, lse_ref = oracle.fwd(*f64[:3], causal, scale)
    label = f"{pattern} d={d} {dtype} causal={causal}"
    check_fwd(o.double().cpu().numpy(), lse.double().cpu().numpy(), o_ref, lse_ref, label)
    if pattern == "steps":
        ref = oracle.bwd(*f64, causal, scale)
        check_grads([t.double().cpu().numpy() for t in (dq, dk, dv)], ref, label)
