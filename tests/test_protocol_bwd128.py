"""The d = 128 backward kernel's mbarrier protocol, checked on the CPU under
random schedules (tests/protocol_model.py mirrors the kernel's roles).

Every barrier test must find its barrier in the phase it is for or the next,
every arrival must land in its phase, every read must see the version it needs,
and no schedule may deadlock.  The same checker must reject the protocol
mistakes that were made while building the kernel, which shows it can see
them.  Plans include items without query tiles (block-sparse key tiles no
query tile attends to), whose handshakes still run once per item."""

import pytest

import protocol_model as pm

PLANS = [[1], [2], [5], [3, 1, 4], [1, 1, 1, 1], [2, 2, 2], [4, 3, 2, 1],
         [0], [2, 0, 3], [0, 0, 1, 0], [1, 0, 0, 2, 0]]


@pytest.mark.parametrize("single", [False, True], ids=["halves", "single"])
@pytest.mark.parametrize("plan", PLANS, ids=lambda p: "-".join(map(str, p)))
def test_protocol_holds_under_random_schedules(plan, single):
    # two dQ staging schemes: two 16 KB halves (dense) and one 32 KB tile
    # (the block-sparse instantiation)
    for seed in range(120):
        pm.run_schedule(plan, seed, single_staging=single)


def test_earlier_correct_design_also_holds():
    # dP^T(g) after dS^T(g-1) (before the early dP^T release) is slower, not wrong
    for seed in range(120):
        pm.run_schedule([3, 2, 4, 1], seed, pm.Variant(no_dpe=True))


def test_static_item_order_holds():
    # without the mask the items are dealt in a fixed order: no response slots
    for seed in range(100):
        pm.run_schedule([3, 2, 4, 1], seed, pm.Variant(static_items=True))


@pytest.mark.parametrize("mistake", ["single_srd", "single_dsf", "epilogue_tile_wait",
                                     "clc_no_empty_wait", "empty_item_no_epf_wait",
                                     "empty_item_no_b_wait", "stg_half_no_read_wait"])
def test_checker_rejects_known_mistakes(mistake):
    caught = 0
    plan = {"clc_no_empty_wait": [2, 1, 1, 3],
            "empty_item_no_epf_wait": [1, 0, 0, 2, 0],
            "empty_item_no_b_wait": [2, 0, 3, 0, 0, 1]}.get(mistake, [3, 2, 4, 1])
    for seed in range(400):
        try:
            pm.run_schedule(plan, seed, pm.Variant(**{mistake: True}))
        except pm.ProtocolError:
            caught += 1
    assert caught > 0, f"{mistake} was never caught"


def test_barrier_parity_rule():
    b = pm.Barrier("x", 2)
    assert b.test(-1)             # the phase before the first counts as complete
    assert not b.test(0)
    b.arrive(0)
    b.arrive(0)
    assert b.test(0) and not b.test(1)
    with pytest.raises(pm.ProtocolError):
        b.test(2)                 # a waiter ahead: the hardware would say "done"
    with pytest.raises(pm.ProtocolError):
        b.arrive(0)               # an arrival for a phase that has completed
