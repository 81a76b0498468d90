"""The d = 64 backward kernel's mbarrier protocol on the CPU under random
schedules (tests/protocol_model_bwd64.py mirrors the kernel's roles): the
kernel as it is (one work item per CTA), the persistent design for it, and the
checker rejecting mistakes."""

import pytest

import protocol_model_bwd64 as pm


@pytest.mark.parametrize("n_it", [1, 2, 3, 5, 8])
def test_d64_protocol_holds_under_random_schedules(n_it):
    for seed in range(150):
        pm.run_schedule(n_it, seed)


@pytest.mark.parametrize("plan", [[3, 1, 4], [1, 1, 1, 1], [2, 5, 2], [8, 1]],
                         ids=lambda p: "-".join(map(str, p)))
def test_persistent_d64_design_holds(plan):
    for seed in range(100):
        pm.run_schedule(plan, seed)


def test_persistent_d64_static_item_order_holds():
    # without the mask the items are dealt in a fixed order: no response slots
    for seed in range(100):
        pm.run_schedule([3, 1, 4, 2], seed, pm.Variant(static_items=True))


def test_accumulator_release_is_implied_by_the_role_order():
    for seed in range(150):
        pm.run_schedule([3, 2, 4, 1], seed, pm.Variant(no_acce=True))


@pytest.mark.parametrize("mistake", ["no_srd", "no_dsf_wait", "flag_without_endb"])
@pytest.mark.parametrize("plan", [5, [3, 2, 4, 1]], ids=["one-item", "persistent"])
def test_checker_rejects_d64_mistakes(mistake, plan):
    caught = 0
    for seed in range(300):
        try:
            pm.run_schedule(plan, seed, pm.Variant(**{mistake: True}))
        except pm.ProtocolError:
            caught += 1
    assert caught > 0


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
