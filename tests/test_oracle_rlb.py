"""Pins of the RLB planner oracle (oracle/rlb_oracle.py) against hand arithmetic,
invariants and exhaustive search on tiny cases -- never against itself."""
import itertools

import numpy as np
import pytest

from oracle import rlb_oracle as R


def test_contiguous_split_by_hand():
    np.testing.assert_array_equal(R.contiguous_split(40, 8), np.repeat(np.arange(8), 5))
    np.testing.assert_array_equal(R.contiguous_split(5, 2), [0, 0, 1, 1, 1])


def test_balanced_input_moves_nothing():
    rank_of, moves = R.rlb_plan(np.ones(40), 8, 0.0, 0.0)
    assert moves == []


def test_hand_example_heaviest_would_overshoot():
    # ranks {0: heads 0,1}, {1: heads 2,3}; loads 9,1 | 1,1 -> L = 10, 2 (factor 5).
    # Moving head 0 (9) gives L = 1, 11: the maximum grows, no gain. Moving head 1 (1)
    # gives L = 9, 3: K = 10 - 9 = 1 ms, G = 1 - 0.25 - 0.25 = 0.5 > 0. Rank 0 has then
    # used its one export, so the plan ends there.
    rank_of, moves = R.rlb_plan(np.array([9.0, 1.0, 1.0, 1.0]), 2, 0.25, 0.25)
    assert [(h, a, b) for h, a, b, _ in moves] == [(1, 0, 1)]
    assert moves[0][3] == pytest.approx(0.5)
    np.testing.assert_array_equal(rank_of, [0, 1, 1, 1])


def test_costs_above_any_gain_move_nothing():
    loads = np.array([5.0, 4.0, 1.0, 1.0])
    # the best possible K is 10 - max(5, 6)... = at most 4 ms; P + C = 5 ms exceeds it
    _, moves = R.rlb_plan(loads, 2, 3.0, 2.0)
    assert moves == []


def test_stops_below_threshold():
    # 4 ranks, one heavy head: L = 4, 1, 1, 1 -> after moving head 0 (3) to rank 1:
    # L = 1, 4, 1, 1 -- no gain; head 1 (1): L = 3, 2, 1, 1 gains 1 ms.
    loads = np.array([3.0, 1.0, 1.0, 0.0, 1.0, 0.0, 1.0, 0.0])
    rank_of, moves = R.rlb_plan(loads, 4, 0.0, 0.0, threshold=1.10)
    Lr = R.rank_loads(loads, rank_of, 4)
    assert Lr.max() <= 3.0
    for h, a, b, g in moves:
        assert g > 0


@pytest.mark.parametrize("seed", range(20))
def test_invariants_random(seed):
    rng = np.random.default_rng(seed)
    Rk = int(rng.integers(2, 9))
    H = Rk * int(rng.integers(1, 6))
    loads = rng.lognormal(0.0, 0.8, H) * 10.0
    comm, sched = float(rng.uniform(0, 1)), float(rng.uniform(0, 0.5))
    rank_of, moves = R.rlb_plan(loads, Rk, comm, sched)
    home = R.contiguous_split(H, Rk)
    L0 = R.rank_loads(loads, home, Rk)
    L1 = R.rank_loads(loads, rank_of, Rk)
    assert L1.max() <= L0.max() + 1e-12                       # the critical path never grows
    assert abs(L1.sum() - L0.sum()) < 1e-9                    # work is conserved
    exports = np.bincount([a for _, a, _, _ in moves], minlength=Rk)
    assert exports.max(initial=0) <= 1                        # at most one head per rank
    moved = [h for h, _, _, _ in moves]
    assert len(moved) == len(set(moved))                      # a received head never moves again
    for h, a, b, g in moves:
        assert home[h] == a and g > 0
    # the plan ends only below the threshold, on a used-up budget, or with no paying move
    mxmn = L1.max() / L1.min() if L1.min() > 0 else np.inf
    if mxmn >= R.K2:
        r_max = int(np.argmax(L1))
        if exports[r_max] == 0:
            r_min = int(np.argmin(L1))
            for h in range(H):
                if rank_of[h] == r_max and home[h] == r_max:
                    t = rank_of.copy()
                    t[h] = r_min
                    assert (L1.max() - R.rank_loads(loads, t, Rk).max()) - comm - sched <= 0


def test_exhaustive_single_move_choice():
    """On tiny cases, the first move is the heaviest own head of the most loaded rank among
    those whose move pays, found here by trying every head of every rank."""
    rng = np.random.default_rng(7)
    for _ in range(200):
        Rk, hpr = 3, 2
        loads = np.round(rng.uniform(0, 10, Rk * hpr), 3)
        home = R.contiguous_split(Rk * hpr, Rk)
        L = R.rank_loads(loads, home, Rk)
        if L.max() / L.min() < R.K2:
            continue
        rmax, rmin = int(np.argmax(L)), int(np.argmin(L))
        paying = []
        for h, r in itertools.product(range(Rk * hpr), range(Rk)):
            if home[h] != rmax or r != rmin:
                continue
            t = home.copy()
            t[h] = r
            g = L.max() - R.rank_loads(loads, t, Rk).max()
            if g > 0:
                paying.append((-loads[h], h))
        _, moves = R.rlb_plan(loads, Rk, 0.0, 0.0)
        if not paying:
            assert moves == []
        else:
            assert moves[0][0] == min(paying)[1]
