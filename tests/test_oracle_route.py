"""Pins for the oracle's pooling, block importance and Top-p / Top-k routing (CPU only).

Pinned by: hand-worked rows with exact dyadic importances (tests/golden), closed forms
(equal logits, one dominant block, p = 1, floor >= nB), brute-force enumeration of all
subsets on small rows, and the CSR invariants.
"""
import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "route_worked_examples.json")


# ------------------------------------------------------------------------------ pooling

def test_pool_constant_blocks_and_tail():
    N, d = 64 * 3 + 5, 3
    x = np.empty((N, d))
    for a in range(4):
        x[a * 64:(a + 1) * 64] = a + 0.5
    pooled = O.block_mean_pool(x)
    assert pooled.shape == (4, d)
    np.testing.assert_array_equal(pooled[:, 0], [0.5, 1.5, 2.5, 3.5])


def test_pool_tail_closed_form():
    # tail block holds 5 rows with values 1..5: mean 3 (not 15/64)
    N = 64 + 5
    x = np.zeros((N, 1))
    x[64:, 0] = np.arange(1, 6)
    x[:64, 0] = np.arange(64)
    pooled = O.block_mean_pool(x)
    assert pooled[0, 0] == 31.5 and pooled[1, 0] == 3.0


def test_pool_equals_averaging_matrix():
    rng = np.random.default_rng(1)
    N, d = 64 * 5 + 17, 8
    x = rng.standard_normal((N, d))
    nB = O.n_blocks(N)
    A = np.zeros((nB, N))
    for i in range(N):
        A[i // 64, i] = 1.0
    A /= A.sum(axis=1, keepdims=True)
    np.testing.assert_allclose(O.block_mean_pool(x), A @ x, rtol=1e-13, atol=1e-13)


# ------------------------------------------------------------------------------ routing

def _golden_cases():
    with open(GOLDEN) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: f"p{c['p']}_k{c['k_floor']}_{c['logits_ln']}")
def test_worked_examples(case):
    s = np.log(np.array(case["logits_ln"], dtype=np.float64))
    info = O.route_row(s, case["p"], case["k_floor"])
    assert info["kept"].tolist() == case["kept"]
    assert info["L_p"] == case["L_p"]
    want_P = np.array([float(Fraction(v)) for v in case["importance"]])
    np.testing.assert_allclose(info["P"], want_P, rtol=1e-15, atol=0)


@pytest.mark.parametrize("nB,p,kf", [(16, 0.9, 2), (16, 0.5, 0), (10, 0.95, 3), (512, 0.9, 4), (1182, 0.8, 4), (7, 0.3, 6)])
def test_equal_logits_closed_form(nB, p, kf):
    s = np.full(nB, 0.25)
    info = O.route_row(s, p, kf)
    # c_j = (j+1)/nB exactly when nB is a power of two; ceil(p nB) in general
    L = max(math.ceil(p * nB - 1e-12), min(kf, nB))
    assert info["L"] == L
    assert info["kept"].tolist() == list(range(L))


def test_tiny_workload_equal_logits_value():
    # 16 blocks, p = 0.9, floor 2: 15 blocks {0..14}
    info = O.route_row(np.zeros(16), 0.9, 2)
    assert info["kept"].tolist() == list(range(15))


@pytest.mark.parametrize("kf", [0, 1, 3])
def test_dominant_block(kf):
    s = np.zeros(20)
    s[13] = 50.0  # P ~ 1 - 19 e^-50
    info = O.route_row(s, 0.9, kf)
    assert info["L"] == max(1, kf)
    assert 13 in info["kept"].tolist()
    # the rest of the floor goes to the lowest indices (all tied)
    assert info["kept"].tolist() == sorted([13] + [b for b in range(20) if b != 13][:max(1, kf) - 1])


def test_p_one_and_big_floor_keep_all():
    rng = np.random.default_rng(2)
    s = rng.standard_normal(33) * 4
    assert O.route_row(s, 1.0, 0)["kept"].tolist() == list(range(33))
    assert O.route_row(s, 0.2, 33)["kept"].tolist() == list(range(33))
    assert O.route_row(s, 0.2, 1000)["kept"].tolist() == list(range(33))


@pytest.mark.parametrize("seed", range(40))
def test_minimal_prefix_and_superset_of_floor(seed):
    rng = np.random.default_rng(100 + seed)
    nB = int(rng.integers(2, 300))
    s = rng.standard_normal(nB) * rng.uniform(0.1, 8)
    p = float(rng.uniform(0.05, 0.999))
    kf = int(rng.integers(0, 8))
    info = O.route_row(s, p, kf)
    P = np.exp(s - s.max())
    P /= P.sum()
    kept = set(info["kept"].tolist())
    L_p = info["L_p"]
    # the L_p most important blocks reach p; L_p - 1 of them do not (fp64, exact sort here)
    by_mass = np.sort(P)[::-1]
    assert by_mass[:L_p].sum() >= p - 1e-12
    assert by_mass[:L_p - 1].sum() < p + 1e-12
    # superset of the top-k floor blocks
    top = np.argsort(-s, kind="stable")[:min(kf, nB)]
    assert set(top.tolist()) <= kept
    assert len(kept) == max(L_p, min(kf, nB))


@pytest.mark.parametrize("seed", range(25))
def test_brute_force_subsets(seed):
    rng = np.random.default_rng(500 + seed)
    nB = int(rng.integers(1, 13))
    s = rng.standard_normal(nB) * rng.uniform(0.3, 5)
    p = float(rng.uniform(0.05, 0.99))
    P = np.exp(s - s.max())
    P /= P.sum()
    best_k, best_sets = None, None
    for k in range(1, nB + 1):
        sets = [c for c in itertools.combinations(range(nB), k) if P[list(c)].sum() >= p]
        if sets:
            best_k, best_sets = k, sets
            break
    info = O.route_row(s, p, 0)
    # the smallest subset reaching p has L_p blocks ...
    assert info["L_p"] == best_k
    # ... and the kept set is the heaviest subset of that size
    heaviest = max(best_sets, key=lambda c: P[list(c)].sum())
    assert sorted(heaviest) == info["kept"].tolist()


def test_csr_invariants_and_head_counts():
    rng = np.random.default_rng(3)
    B, H, nB, d = 1, 3, 9, 16
    pq = rng.standard_normal((B, H, nB, d)) * 2
    pk = rng.standard_normal((B, H, nB, d)) * 2
    R = O.route(pq, pk, d, 0.85, 2)
    rp, ci = R["row_ptr"], R["col_idx"]
    assert rp[0] == 0 and rp.size == B * H * nB + 1 and np.all(np.diff(rp) >= 1)
    for r in range(B * H * nB):
        lst = ci[rp[r]:rp[r + 1]]
        assert np.all(np.diff(lst) > 0) and lst.min() >= 0 and lst.max() < nB
        h = r // nB
        info = O.route_row(O.block_logits(pq[0, h], pk[0, h], d)[r % nB], 0.85, 2)
        assert lst.tolist() == info["kept"].tolist()
    for h in range(H):
        assert R["head_kept"][h] == rp[(h + 1) * nB] - rp[h * nB]


def test_logit_scale_and_orientation():
    # s[a, b] = q_a . k_b / sqrt(d): an asymmetric case catches a transposed product
    pq = np.array([[1.0, 0.0], [0.0, 2.0]])
    pk = np.array([[3.0, 0.0], [1.0, 1.0], [0.0, 0.0]])
    s = O.block_logits(pq, pk, 4)
    np.testing.assert_array_equal(s, [[1.5, 0.5, 0.0], [0.0, 1.0, 0.0]])


def test_lpt_order_and_union_costs():
    # 1 head, 5 query blocks -> 3 tiles (2, 2, 1 rows)
    lists = [[0, 1], [1, 2], [4], [0, 1, 2, 3], [2]]
    rp = np.concatenate([[0], np.cumsum([len(x) for x in lists])])
    ci = np.concatenate([np.array(x) for x in lists])
    cost = O.tile_costs(rp, ci, 1, 5)
    assert cost.tolist() == [3, 5, 1]
    assert O.lpt_order(cost).tolist() == [1, 0, 2]
    assert O.lpt_order(np.array([2, 5, 2, 5, 0])).tolist() == [1, 3, 0, 2, 4]


# ---- ambiguity flags (they decide which GPU/oracle mask differences may be excused) ----

def _logits_for(w):
    """Logits whose softmax is w / sum(w): s = log w."""
    return np.log(np.asarray(w, dtype=np.float64))


@pytest.mark.parametrize("w,k_floor,want", [
    ([0.5, 0.4 - 2e-7, 0.1 + 2e-7], 0, True),    # c_1 = p - 2e-7: the cut could move up
    ([0.5, 0.4 + 2e-7, 0.1 - 2e-7], 0, True),    # c_1 = p + 2e-7: the cut could move down
    ([0.5, 0.3, 0.2], 0, False),                 # c = 0.5, 0.8, 1.0: every mass 0.1 from p
    ([0.5, 0.4 + 2e-7, 0.1 - 2e-7], 3, False),   # the floor (3 blocks) decides, not the mass
])
def test_mass_flag_only_when_the_cut_sits_within_the_band(w, k_floor, want):
    s = _logits_for(w)
    info = O.route_row(s, 0.9, k_floor)
    amb = O.row_ambiguity(s, info, 0.9)
    assert bool(amb["ambiguous_mass"]) == want
    assert not amb["ambiguous_tie"]


@pytest.mark.parametrize("s,want", [
    ([1.0, 0.5, 0.5, -3.0], True),               # L = 2 and the 2nd/3rd logits tie: which one is kept is moot
    ([1.0, 0.5, 0.5 - 5e-10, -3.0], True),       # closer than 1e-9 relative
    ([1.0, 0.5, 0.5 - 5e-9, -3.0], False),       # 5e-9 apart: outside the band
    ([1.0, -2.0, -3.0, -3.0], False),            # a tie, but away from the boundary (L = 1)
])
def test_tie_flag_only_at_the_boundary(s, want):
    s = np.asarray(s, dtype=np.float64)
    info = O.route_row(s, 0.5, 0)
    amb = O.row_ambiguity(s, info, 0.5)
    assert bool(amb["ambiguous_tie"]) == want
    assert not amb["ambiguous_mass"]
