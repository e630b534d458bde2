"""Pins of the SASA oracle (oracle/sasa_oracle.py): the budget formula by hand, and the
augmentation by the properties that define it -- every taken entry outranks every skipped
entry left out, rows stay prefixes of their routing order, totals match the budget, and
ties resolve as stated."""
import numpy as np
import pytest

import oracle as O
from oracle import sasa_oracle as S


def test_mode_thresholds():
    assert S.mode([1.0, 1.04]) == "none"
    assert S.mode([1.0, 1.05]) == "sasa"
    assert S.mode([1.0, 1.099]) == "sasa"
    assert S.mode([1.0, 1.10]) == "rlb+sasa"
    assert S.mode([0.0, 1.0]) == "rlb+sasa"


def test_budgets_by_hand():
    # critical 10 ms; slacks 0, 0.5 (5% < 7%: no), 3, 10; c = 0.25 ms per block
    b = S.budgets([10.0, 9.5, 7.0, 0.0], 0.25)
    np.testing.assert_array_equal(b, [0, 0, int(np.floor(0.8 * 3.0 / 0.25)), int(np.floor(0.8 * 10.0 / 0.25))])
    assert b[2] == 9 and b[3] == 32
    # the augmented load never reaches the critical path
    L = np.array([10.0, 9.5, 7.0, 0.0])
    assert (L + b * 0.25 < 10.0 + 1e-12)[1:].all()


def _case(seed, BH=4, nB=6, R=2):
    rng = np.random.default_rng(seed)
    logits = rng.normal(0, 2.0, (BH, nB, nB))
    L = rng.integers(1, nB + 1, BH * nB)
    rank_of = np.arange(BH) % R
    budget = rng.integers(0, 12, R)
    return logits, L, rank_of, budget


@pytest.mark.parametrize("seed", range(25))
def test_taken_entries_outrank_the_rest(seed):
    logits, L, rank_of, budget = _case(seed)
    BH, nB, _ = logits.shape
    new_len = S.augment(logits, L, rank_of, budget)
    assert (new_len >= L).all() and (new_len <= nB).all()
    for r in range(len(budget)):
        taken, left = [], []
        for h in np.nonzero(rank_of == r)[0]:
            for a in range(nB):
                s = logits[h, a]
                order = O.routing_order(s)
                P = O.importance(s)
                row = h * nB + a
                for pos in range(L[row], nB):
                    (taken if pos < new_len[row] else left).append(P[order[pos]])
        skipped = len(taken) + len(left)
        assert len(taken) == min(int(budget[r]), skipped)
        if taken and left:
            assert min(taken) >= max(left)


def test_prefix_and_mass_grow():
    logits, L, rank_of, budget = _case(3, BH=3, nB=8, R=3)
    new_len = S.augment(logits, L, rank_of, budget)
    m0 = S.kept_mass(logits, L)
    m1 = S.kept_mass(logits, new_len)
    assert (m1 >= m0 - 1e-15).all()
    assert (m1 > m0).sum() == (new_len > L).sum()


def test_ties_lower_head_then_row_then_position():
    # all logits equal: every skipped entry has the same importance 1/nB
    BH, nB = 2, 4
    logits = np.zeros((BH, nB, nB))
    L = np.full(BH * nB, 2)
    new_len = S.augment(logits, L, np.zeros(BH, dtype=np.int64), np.array([3]))
    # head 0: rows 0, 1, 2, 3 each have 2 skipped entries; the first 3 taken are row 0 pos
    # 2, 3 and row 1 pos 2
    np.testing.assert_array_equal(new_len, [4, 3, 2, 2, 2, 2, 2, 2])


def test_budget_larger_than_candidates_takes_all():
    logits, L, rank_of, _ = _case(9)
    BH, nB, _ = logits.shape
    new_len = S.augment(logits, L, rank_of, np.array([10 ** 6, 10 ** 6]))
    np.testing.assert_array_equal(new_len, np.full(BH * nB, nB))
