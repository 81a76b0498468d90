"""The forward kernel's mbarrier protocol, checked on the CPU under random
schedules (tests/protocol_model_fwd.py mirrors the kernel's roles): barrier
tests in the phase they are for or the next, arrivals in their phase, reads of
the versions they need, no deadlock; and protocol mistakes are rejected.
Dense (causal and not) and block-sparse plans, including items where a tile
starts attending in the middle, tiles with no marked key tile and items with
none at all."""

import pytest

import protocol_model_fwd as pf

PLANS = {
    "noncausal": [(3, 3), (3, 3), (1, 1)],
    "causal": [(1, 2), (3, 4), (5, 0)],
    "causal-repeat": [(2, 3), (2, 3), (2, 3), (4, 5)],
    "single-step": [(1, 0), (1, 2), (1, 1)],
    "sparse": [(4, 4, (1, 0, 1, 0), (0, 1, 1, 1)), (3, 3, (0, 0, 1), (1, 0, 0)),
               (4, 4, (1, 1, 1, 1), (0, 0, 0, 0)), (2, 2, (0, 0), (0, 0)),
               (3, 3, (0, 1, 0), (0, 1, 1))],
    "sparse-causal": [(3, 4, (0, 1, 1), (1, 0, 0, 1)), (1, 0, (1,), ()),
                      (5, 6, (1, 0, 0, 0, 1), (0, 0, 1, 0, 0, 1)), (1, 2, (0,), (0, 1))],
    "sparse-gaps": [(3, 3, (1, 0, 1), (0, 1, 0))] * 4,
}


@pytest.mark.parametrize("stages", [2, 3, 4])
@pytest.mark.parametrize("name", sorted(PLANS))
def test_forward_protocol_holds_under_random_schedules(name, stages):
    # 2 K/V stages at d = 128, 3 with e4m3 scores at d = 128, 4 at d = 64
    for seed in range(100):
        pf.run_schedule(PLANS[name], seed, stages=stages)


@pytest.mark.parametrize("plan", ["causal", "sparse"])
def test_next_s_needs_the_pv_wait_although_issued_later(plan):
    """S_t of the next key tile overwrites the columns P_t V reads.  Completed
    in issue order the mistake would go unseen; with MMAs on different
    accumulators free to complete out of order, as the hardware allows, it is
    caught."""
    v = pf.Variant(s_without_od_wait=True)
    for seed in range(100):
        pf.run_schedule(PLANS[plan], seed, v, in_order=True)
    caught = 0
    for seed in range(300):
        try:
            pf.run_schedule(PLANS[plan], seed, v)
        except pf.ProtocolError:
            caught += 1
    assert caught > 0


@pytest.mark.parametrize("stages", [2, 4])
@pytest.mark.parametrize("name", sorted(PLANS))
def test_forward_protocol_with_p_in_own_columns(name, stages):
    # the d = 64 layout: P_t in columns of its own, next S_t after P-ready only
    for seed in range(100):
        pf.run_schedule(PLANS[name], seed, stages=stages, p_own=True)


@pytest.mark.parametrize("plan", ["causal", "sparse"])
def test_p_write_needs_the_pv_wait(plan):
    """With P in columns of its own the next S_t goes out ahead of P_t V, so
    nothing but the softmax's own wait keeps its next P_t write off the
    columns that P V still reads; skipping that wait is caught."""
    caught = 0
    for seed in range(300):
        try:
            pf.run_schedule(PLANS[plan] + [(3, 3), (2, 4)], seed,
                            pf.Variant(p_write_no_od_wait=True), stages=4, p_own=True)
        except pf.ProtocolError:
            caught += 1
    assert caught > 0


def test_static_item_order_holds():
    # without a mask of either kind the items are dealt in a fixed order
    for seed in range(100):
        pf.run_schedule(PLANS["noncausal"], seed, pf.Variant(static_items=True))


@pytest.mark.parametrize("mistake,plan,stages", [("ke_before_pv", "causal", 2),
                                                 ("epilogue_no_od_wait", "causal", 2),
                                                 ("clc_no_empty_wait", "causal", 2),
                                                 ("s_wait_ignores_fresh_tile", "sparse-gaps", 4)])
def test_checker_rejects_forward_mistakes(mistake, plan, stages):
    caught = 0
    for seed in range(300):
        try:
            pf.run_schedule(PLANS[plan] + [(1, 2), (3, 4), (5, 0), (2, 2)], seed,
                            pf.Variant(**{mistake: True}), stages=stages)
        except pf.ProtocolError:
            caught += 1
    assert caught > 0, f"{mistake} was never caught"


def test_skipped_wait_is_implied_with_two_stages():
    # the same skipped wait is harmless with two K/V stages (see Variant)
    for seed in range(150):
        pf.run_schedule(PLANS["sparse-gaps"], seed, pf.Variant(s_wait_ignores_fresh_tile=True),
                        stages=2)
