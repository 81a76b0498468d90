"""The d = 64 backward kernel's mbarrier protocol on the CPU under random
schedules (tests/protocol_model_bwd64.py mirrors the kernel's roles), and the
checker rejecting mistakes."""

import pytest

import protocol_model_bwd64 as pm


@pytest.mark.parametrize("n_it", [0, 1, 2, 3, 5, 8])
def test_d64_protocol_holds_under_random_schedules(n_it):
    for seed in range(150):
        pm.run_schedule(n_it, seed)


@pytest.mark.parametrize("mistake", ["no_srd", "no_dsf_wait", "flag_without_endb"])
def test_checker_rejects_d64_mistakes(mistake):
    caught = 0
    for seed in range(300):
        try:
            pm.run_schedule(5, seed, pm.Variant(**{mistake: True}))
        except pm.ProtocolError:
            caught += 1
    assert caught > 0, f"{mistake} was never caught"


@pytest.mark.parametrize("skipped", ["ds_without_dqf_wait", "dq_without_dqe_wait"])
def test_two_waits_are_implied_by_the_issue_order(skipped):
    """The kernel keeps two waits of the deferred dQ drain that the order makes
    redundant (see Variant); skipping either alone is never caught.  They stay
    as guards against a reordering."""
    for seed in range(150):
        pm.run_schedule(5, seed, pm.Variant(**{skipped: True}))


def test_next_s_needs_the_dv_wait_although_issued_later():
    """S^T(g+1) overwrites the columns dV(g) reads P^T from, on another
    accumulator: completed in issue order the missing wait goes unseen; with
    the completion order the hardware allows, it is caught."""
    v = pm.Variant(s_without_dvd_wait=True)
    for seed in range(100):
        pm.run_schedule(4, seed, v, in_order=True)
    caught = 0
    for seed in range(300):
        try:
            pm.run_schedule(4, seed, v)
        except pm.ProtocolError:
            caught += 1
    assert caught > 0
