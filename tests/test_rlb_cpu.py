"""The library's RLB planner (fva_rlb_plan, host code behind the C ABI) against the
float64 oracle: identical moves, gains and final placement; argument checks."""
import ctypes

import numpy as np
import pytest

from adaptive_block_sparse_hilbert_b200 import fva
from oracle import rlb_oracle as R


def _same(loads, ranks, comm, sched, thr=1.10, per_rank=1):
    got_rank, got_moves = fva.fva_rlb_plan(loads, ranks, comm, sched, thr, per_rank)
    want_rank, want_moves = R.rlb_plan(np.asarray(loads, dtype=np.float64), ranks, comm, sched, thr, per_rank)
    np.testing.assert_array_equal(got_rank, want_rank)
    assert [m[:3] for m in got_moves] == [m[:3] for m in want_moves]
    for g, w in zip(got_moves, want_moves):
        assert g[3] == w[3]  # same float64 operations in the same order


def test_hand_example():
    _same([9.0, 1.0, 1.0, 1.0], 2, 0.25, 0.25)
    _, moves = fva.fva_rlb_plan([9.0, 1.0, 1.0, 1.0], 2, 0.25, 0.25)
    assert [m[:3] for m in moves] == [(1, 0, 1)]


@pytest.mark.parametrize("seed", range(40))
def test_matches_oracle_random(seed):
    rng = np.random.default_rng(100 + seed)
    ranks = int(rng.integers(1, 9))
    H = ranks * int(rng.integers(1, 7)) + int(rng.integers(0, 3))
    # lognormal head loads (heavy tails like the routed densities), some exact ties
    loads = np.round(rng.lognormal(0.0, 1.0, H) * 20.0, int(rng.integers(0, 3)))
    if seed % 5 == 0:
        loads[: H // 3] = 0.0
    _same(loads, ranks, float(rng.uniform(0, 2)), float(rng.uniform(0, 1)),
          float(rng.choice([1.0, 1.05, 1.10, 1.5])), int(rng.integers(0, 3)))


def test_eight_ranks_forty_heads():
    rng = np.random.default_rng(5)
    loads = rng.lognormal(0.0, 0.7, 40) * 1.7
    _same(loads, 8, 0.1, 0.1)


def test_argument_checks():
    L = fva.lib()
    loads = (ctypes.c_double * 4)(1.0, 2.0, 3.0, 4.0)
    rank = (ctypes.c_int32 * 4)()
    moves = (fva.fva_rlb_move * 4)()
    n = ctypes.c_int(0)
    args = dict(comm=0.0, sched=0.0, thr=1.1, per=1)

    def call(loads_=loads, H=4, R_=2, thr=1.1, per=1, cap=4, comm=0.0):
        return L.fva_rlb_plan(loads_, H, R_, comm, 0.0, thr, per, rank, moves, cap, ctypes.byref(n))

    assert call() == fva.FVA_OK
    assert call(R_=0) == fva.FVA_ERR_INVALID_ARG
    assert call(H=0) == fva.FVA_ERR_INVALID_ARG
    assert call(thr=0.9) == fva.FVA_ERR_INVALID_ARG
    assert call(comm=-1.0) == fva.FVA_ERR_INVALID_ARG
    assert call(cap=1) == fva.FVA_ERR_CAPACITY  # min(4 heads, 2 ranks x 1) = 2 needed
    bad = (ctypes.c_double * 4)(1.0, float("nan"), 3.0, 4.0)
    assert call(loads_=bad) == fva.FVA_ERR_INVALID_ARG
    bad = (ctypes.c_double * 4)(1.0, -2.0, 3.0, 4.0)
    assert call(loads_=bad) == fva.FVA_ERR_INVALID_ARG
