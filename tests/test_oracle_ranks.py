"""CPU pins of the FLRC rank-allocation oracle (FLRC "Fisher-based layer-wise
rank allocation" and "progressive low-rank decoding")."""
import numpy as np
import pytest

from oracle import ranks


def test_proportional_split_hand_values():
    # alpha 1:2:3:4 of a budget of 100 -> 10, 20, 30, 40
    assert ranks.flrc_ranks([1, 2, 3, 4], 100, [1000] * 4).tolist() == [10, 20, 30, 40]
    # alpha 1:3 of 10 -> 2.5 and 7.5 -> ties to even: 2 and 8
    assert ranks.flrc_ranks([1, 3], 10, [100, 100]).tolist() == [2, 8]
    # 1:1 of 3 -> 1.5 each -> 2, 2 (ties to even)
    assert ranks.flrc_ranks([1, 1], 3, [10, 10]).tolist() == [2, 2]


def test_clamping_to_one_and_to_the_stored_rank():
    assert ranks.flrc_ranks([1e-9, 1.0], 64, [64, 64]).tolist() == [1, 64]
    assert ranks.flrc_ranks([1, 1], 1000, [300, 512]).tolist() == [300, 500]


def test_budget_is_met_within_rounding():
    rng = np.random.default_rng(0)
    alpha = rng.lognormal(0.0, 0.35, 128)
    r = ranks.flrc_ranks(alpha, 157280, [10 ** 6] * 128)
    assert abs(int(r.sum()) - 157280) <= 64     # at most half a unit per entry


def test_non_increasing_budget_gives_non_increasing_ranks():
    rng = np.random.default_rng(1)
    alpha = rng.lognormal(0.0, 0.35, 32)
    caps = rng.integers(200, 1500, 32)
    budgets = np.linspace(30000, 5000, 17)
    R = ranks.progressive_ranks(alpha, budgets, caps)
    assert (np.diff(R, axis=0) <= 0).all()
    assert (R >= 1).all() and (R <= caps[None, :]).all()


def test_scale_invariance_of_importances():
    # only the ratios alpha_p / S matter (powers of two keep every quotient exact)
    alpha = [3.0, 5.0, 11.0, 1.0]
    assert ranks.flrc_ranks(alpha, 777, [999] * 4).tolist() == \
        ranks.flrc_ranks([a * 8 for a in alpha], 777, [999] * 4).tolist()
