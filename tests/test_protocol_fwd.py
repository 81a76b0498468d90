"""The forward kernel's mbarrier protocol, checked on the CPU under random
schedules (tests/protocol_model_fwd.py mirrors the kernel's roles): barrier
tests in the phase they are for or the next, arrivals in their phase, reads of
the versions they need, no deadlock; and protocol mistakes are rejected."""

import pytest

import protocol_model_fwd as pf

PLANS = {
    "noncausal": [(3, 3), (3, 3), (1, 1)],
    "causal": [(1, 2), (3, 4), (5, 0)],
    "causal-repeat": [(2, 3), (2, 3), (2, 3), (4, 5)],
    "single-step": [(1, 0), (1, 2), (1, 1)],
}


@pytest.mark.parametrize("name", sorted(PLANS))
def test_forward_protocol_holds_under_random_schedules(name):
    for seed in range(150):
        pf.run_schedule(PLANS[name], seed)


@pytest.mark.parametrize("name", sorted(PLANS))
def test_split_softmax_design_holds(name):
    # next-step design: each tile's softmax over two column halves, exchanging
    # the row max per key tile and the row sum per item
    for seed in range(100):
        pf.run_schedule(PLANS[name], seed, pf.Variant(split=True))


@pytest.mark.parametrize("name", sorted(PLANS))
@pytest.mark.parametrize("split", [False, True], ids=["one-group", "split"])
def test_order_c_design_holds(name, split):
    # next-step design: per key tile both P V first, then both next S
    for seed in range(100):
        pf.run_schedule(PLANS[name], seed, pf.Variant(order_c=True, split=split))


@pytest.mark.parametrize("order_c", [False, True], ids=["order-a", "order-c"])
def test_next_s_needs_the_pv_wait_although_issued_later(order_c):
    """S_t(j+1) overwrites the columns P_t(j) V reads.  Completed in issue
    order the mistake would go unseen; with MMAs on different accumulators
    free to complete out of order, as the hardware allows, it is caught."""
    plan = [(3, 4), (2, 2)]
    v = pf.Variant(order_c=order_c, s_without_od_wait=True)
    for seed in range(100):
        pf.run_schedule(plan, seed, v, in_order=True)
    caught = 0
    for seed in range(300):
        try:
            pf.run_schedule(plan, seed, v)
        except pf.ProtocolError:
            caught += 1
    assert caught > 0


SD_PLANS = {
    "noncausal": [(6, 6), (6, 6), (2, 2)],
    "causal": [(2, 4), (6, 8), (10, 0)],
    "causal-repeat": [(3, 5), (3, 5), (1, 1), (8, 10)],
}


@pytest.mark.parametrize("name", sorted(SD_PLANS))
def test_double_buffered_s_design_holds(name):
    # next-step design: 64-key tiles, two S buffers per query tile; P ready and
    # P V done are one barrier per S buffer
    for seed in range(120):
        pf.run_schedule(SD_PLANS[name], seed, pf.Variant(s_double=True))


def test_double_buffered_s_needs_the_pv_wait():
    caught = 0
    for seed in range(300):
        try:
            pf.run_schedule(SD_PLANS["causal"], seed,
                            pf.Variant(s_double=True, s_double_no_od_wait=True))
        except pf.ProtocolError:
            caught += 1
    assert caught > 0


def test_static_item_order_holds():
    # without the mask the items are dealt in a fixed order: no response slots
    for seed in range(100):
        pf.run_schedule(PLANS["noncausal"], seed, pf.Variant(static_items=True))


@pytest.mark.parametrize("mistake", ["ke_before_pv", "epilogue_no_od_wait",
                                     "split_no_exchange_wait", "clc_no_empty_wait"])
def test_checker_rejects_forward_mistakes(mistake):
    caught = 0
    for seed in range(300):
        try:
            kw = {mistake: True, "split": mistake.startswith("split")}
            pf.run_schedule([(1, 2), (3, 4), (5, 0), (2, 2)], seed, pf.Variant(**kw))
        except pf.ProtocolError:
            caught += 1
    assert caught > 0, f"{mistake} was never caught"
