"""The inputs of the rescale parity tests really reach the forward's rescale
branch (CPU only): replaying the max-keeping rule in fp64 on them, rows move
their max after the first key tile, several times per row, and warps mix rows
that move with rows that do not.  Checked for 64- and 128-key tiles."""

import numpy as np
import pytest

from helpers import default_scale, mixed_warps, rescale_inputs, rescale_moves


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("key_tile", [64, 128])
@pytest.mark.parametrize("causal", [True, False])
def test_steps_pattern_moves_the_max(d, key_tile, causal):
    _, f64 = rescale_inputs("steps", 1, 1, 700, d, seed=3)
    moved, kept = rescale_moves(f64[0][0, 0], f64[1][0, 0], causal, default_scale(d), key_tile)
    per_row = moved.sum(1)
    assert (per_row >= 1).sum() >= 250
    assert (per_row >= 2).sum() >= 150
    assert mixed_warps(moved, kept) >= 20


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("key_tile", [64, 128])
def test_shared_pattern_moves_the_max_causal(d, key_tile):
    _, f64 = rescale_inputs("shared", 1, 1, 700, d, seed=3)
    moved, _ = rescale_moves(f64[0][0, 0], f64[1][0, 0], True, default_scale(d), key_tile)
    assert (moved.sum(1) >= 1).sum() >= 400


def test_gaussian_workload_inputs_do_not_reach_the_branch():
    # why the dedicated inputs exist: at sigma 1 no row moves its max
    from helpers import inputs
    _, f64 = inputs(1, 1, 700, 128, seed=3)
    moved, _ = rescale_moves(f64[0][0, 0], f64[1][0, 0], False, default_scale(128), 128)
    assert not moved.any()
