"""The fused linear-attention kernel's mbarrier protocol, checked on the CPU
under random schedules (tests/protocol_model_linear.py mirrors the kernel's
roles): every barrier test in the phase it is for or the next, every arrival
in its phase, every read of the version it needs, no deadlock; and each
planted mistake is caught."""

import pytest

import protocol_model_linear as pl


@pytest.mark.parametrize("nc", [1, 2, 3, 4, 7])
def test_linear_protocol_holds_under_random_schedules(nc):
    for seed in range(150):
        pl.run_schedule(nc, seed)


@pytest.mark.parametrize("nc", [1, 2, 5])
def test_linear_protocol_holds_in_issue_order(nc):
    for seed in range(20):
        pl.run_schedule(nc, seed, in_order=True)


@pytest.mark.parametrize("mistake", ["no_oe_wait", "no_ssf_wait", "no_od_wait", "contiguous_p"])
def test_checker_rejects_linear_mistakes(mistake):
    """The output and state waits are needed, and so is the P layout: the
    upper key half packing P next to the lower half's would overwrite columns
    the lower half may not have read."""
    caught = 0
    for seed in range(300):
        try:
            pl.run_schedule(6, seed, pl.Variant(**{mistake: True}))
        except pl.ProtocolError:
            caught += 1
    assert caught > 0, f"{mistake} was never caught"


@pytest.mark.parametrize("skipped", ["no_se_wait", "no_kve_wait", "no_pvd_wait"])
def test_three_waits_are_implied_by_the_issue_order(skipped):
    """The kernel keeps three waits that the current order makes redundant:
    the state warps' wait before overwriting a state buffer (the KV-full
    commit they waited on follows the Q S that read it), the issuer's wait for
    a KV buffer to be read (the state stored after that read was waited for
    one chunk earlier) and its wait for the P V of two chunks back (the same
    commit released the Q/K/V stage whose new loads it waits for).  Skipping
    any of them alone is never caught; they stay as a guard against a
    reordering."""
    for seed in range(150):
        pl.run_schedule(6, seed, pl.Variant(**{skipped: True}))
