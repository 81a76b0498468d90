"""The d = 64 backward kernel's mbarrier protocol on the CPU under random
schedules (tests/protocol_model_bwd64.py mirrors the kernel's roles), and the
checker rejecting two mistakes in it."""

import pytest

import protocol_model_bwd64 as pm


@pytest.mark.parametrize("n_it", [1, 2, 3, 5, 8])
def test_d64_protocol_holds_under_random_schedules(n_it):
    for seed in range(150):
        pm.run_schedule(n_it, seed)


@pytest.mark.parametrize("mistake", ["no_srd", "no_dsf_wait"])
def test_checker_rejects_d64_mistakes(mistake):
    caught = 0
    for seed in range(300):
        try:
            pm.run_schedule(5, seed, pm.Variant(**{mistake: True}))
        except pm.ProtocolError:
            caught += 1
    assert caught > 0
