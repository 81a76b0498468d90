"""The stream and event protocol of attn_sdpa_host, checked on the CPU.

tests/host_pipe_model.py replays the call's enqueue sequence (three chunk
slots; copies in, kernels and copies out on three streams; events ordering
them after the caller's earlier work and the caller's stream after the last
copy back) under random schedules, several calls back to back.  Every read
must see the version of the buffer it needs.  The protocol holds for several
head counts and chunk sizes, and leaving out any one of its waits is caught.
"""

import pytest

from host_pipe_model import run


@pytest.mark.parametrize("BH,hc", [(7, 2), (8, 3), (1, 1), (12, 1), (5, 5)])
def test_protocol_holds(BH, hc):
    for seed in range(400):
        run(seed, calls=3, BH=BH, hc=hc)


@pytest.mark.parametrize("wait", ["start", "drained", "loaded", "computed", "done"])
def test_each_wait_is_needed(wait):
    caught = 0
    for seed in range(400):
        try:
            run(seed, calls=3, BH=7, hc=2, drop=(wait,))
        except AssertionError:
            caught += 1
    assert caught > 0, f"dropping the {wait} wait went unnoticed"
