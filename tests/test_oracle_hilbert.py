"""Pins for the oracle's Hilbert order (CPU only).

The oracle builds the curve by recursive quadrant copies. These tests check it against
an independent construction (the Lindenmayer-system turtle walk of the Hilbert curve),
against the order-1 base case, and against invariants that a wrong reflection or a
swapped axis would break: a bijection, unit steps on 2^m squares, and better locality
than raster order on the workloads' rectangular frames.
"""
import numpy as np
import pytest

import oracle as O


def lsystem_hilbert(m):
    """Hilbert curve cells by the L-system A -> +BF-AFA-FB+, B -> -AF+BFB+FA- (turtle walk).

    Start at (0, 0) heading +x; '+' turns left (counter-clockwise), '-' turns right.
    With this start the order-1 walk is (0,0) -> (0,1) -> (1,1) -> (1,0).
    """
    s = "A"
    rules = {"A": "+BF-AFA-FB+", "B": "-AF+BFB+FA-"}
    for _ in range(m):
        s = "".join(rules.get(ch, ch) for ch in s)
    x, y, dx, dy = 0, 0, 1, 0
    cells = [(0, 0)]
    for ch in s:
        if ch == "F":
            x, y = x + dx, y + dy
            cells.append((x, y))
        elif ch == "+":
            dx, dy = -dy, dx
        elif ch == "-":
            dx, dy = dy, -dx
    return np.array(cells, dtype=np.int64).reshape(-1, 2)


def test_order1_base_case():
    assert O.hilbert_curve(1).tolist() == [[0, 0], [0, 1], [1, 1], [1, 0]]
    assert O.hilbert_curve(0).tolist() == [[0, 0]]


@pytest.mark.parametrize("m", range(0, 8))
def test_matches_lsystem_construction(m):
    np.testing.assert_array_equal(O.hilbert_curve(m), lsystem_hilbert(m))


@pytest.mark.parametrize("m", range(1, 8))
def test_unit_steps_and_bijection_on_square(m):
    c = O.hilbert_curve(m)
    n = 1 << m
    assert c.shape == (n * n, 2)
    assert len({(int(a), int(b)) for a, b in c}) == n * n
    assert c.min() == 0 and c.max() == n - 1
    steps = np.abs(np.diff(c, axis=0)).sum(axis=1)
    assert np.all(steps == 1)
    # starts at the origin and ends at the lower-right corner
    assert tuple(c[0]) == (0, 0) and tuple(c[-1]) == (n - 1, 0)


@pytest.mark.parametrize("T,Hg,Wg", [(4, 16, 16), (21, 30, 52), (21, 45, 80), (13, 30, 45), (2, 1, 1), (3, 5, 3)])
def test_perm_is_bijection_with_frames_concatenated(T, Hg, Wg):
    perm, inv = O.hilbert_perm(T, Hg, Wg)
    N = T * Hg * Wg
    assert perm.shape == (N,)
    np.testing.assert_array_equal(np.sort(perm), np.arange(N))
    np.testing.assert_array_equal(perm[inv], np.arange(N))
    np.testing.assert_array_equal(inv[perm], np.arange(N))
    hw = Hg * Wg
    # frame t occupies positions [t*hw, (t+1)*hw) and holds exactly frame t's tokens
    for t in range(T):
        seg = perm[t * hw:(t + 1) * hw]
        assert seg.min() == t * hw and seg.max() == (t + 1) * hw - 1
        np.testing.assert_array_equal(seg - t * hw, perm[:hw])


def test_square_frame_neighbours_adjacent():
    # 16x16 frame (tiny workload): consecutive positions are grid neighbours
    perm, _ = O.hilbert_perm(1, 16, 16)
    y, x = perm // 16, perm % 16
    assert np.all(np.abs(np.diff(y)) + np.abs(np.diff(x)) == 1)


def _block_spread(perm, Hg, Wg, block=64):
    y, x = perm // Wg, perm % Wg
    nb = perm.size // block
    areas = []
    for a in range(nb):
        ys, xs = y[a * block:(a + 1) * block], x[a * block:(a + 1) * block]
        areas.append((ys.max() - ys.min() + 1) + (xs.max() - xs.min() + 1))
    return float(np.mean(areas))


@pytest.mark.parametrize("Hg,Wg", [(30, 52), (45, 80), (30, 45), (16, 16)])
def test_rectangular_locality_beats_raster(Hg, Wg):
    perm, _ = O.hilbert_perm(1, Hg, Wg)
    y, x = perm // Wg, perm % Wg
    step = np.abs(np.diff(y)) + np.abs(np.diff(x))
    raster = np.arange(Hg * Wg)
    ry, rx = raster // Wg, raster % Wg
    rstep = np.abs(np.diff(ry)) + np.abs(np.diff(rx))
    assert step.mean() < rstep.mean()
    # most consecutive pairs are grid neighbours even off the 2^m square
    assert np.mean(step == 1) > 0.9
    # 64-token blocks are compact (half-perimeter of their bounding box) vs raster rows
    assert _block_spread(perm, Hg, Wg) < _block_spread(raster, Hg, Wg)


def test_reorder_inverse_roundtrip():
    rng = np.random.default_rng(0)
    T, Hg, Wg, H, d = 2, 5, 7, 3, 4
    N = T * Hg * Wg
    x = rng.standard_normal((1, N, H, d))
    perm, inv = O.hilbert_perm(T, Hg, Wg)
    xr = O.reorder(x, perm)
    assert xr.shape == (1, H, N, d)
    # position i of head h holds token perm[i] of head h
    for i in (0, 5, N - 1):
        np.testing.assert_array_equal(xr[0, 2, i], x[0, perm[i], 2])
    np.testing.assert_array_equal(O.inverse_reorder(xr, perm), x)


@pytest.mark.parametrize("m", [0, 1, 2, 3, 5, 7])
def test_index_construction_inverts_the_recursive_curve(m):
    # the digit-by-digit index of every cell of the recursive curve is its position on it
    curve = O.hilbert_curve(m)
    np.testing.assert_array_equal(O.hilbert_index(m, curve[:, 0], curve[:, 1]), np.arange(4 ** m))


@pytest.mark.parametrize("T,Hg,Wg", [(1, 1, 1), (2, 3, 5), (1, 45, 80), (3, 30, 52), (1, 1, 200), (2, 97, 3),
                                     (1, 64, 64)])
def test_perm_by_index_equals_enumerated_perm(T, Hg, Wg):
    a = O.hilbert_perm(T, Hg, Wg)
    b = O.hilbert_perm_by_index(T, Hg, Wg)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


def test_index_on_the_largest_square_walks_unit_steps():
    # m = 16: consecutive indices along a sampled stretch are grid neighbours
    m = 16
    rng = np.random.default_rng(5)
    side = 1 << m
    for _ in range(4):
        x0, y0 = (int(v) for v in rng.integers(0, side, 2))
        d0 = int(O.hilbert_index(m, x0, y0))
        xs, ys = np.meshgrid(np.arange(max(0, x0 - 40), min(side, x0 + 40)),
                             np.arange(max(0, y0 - 40), min(side, y0 + 40)))
        d = O.hilbert_index(m, xs.ravel(), ys.ravel())
        near = np.argsort(d)
        dd, xx, yy = d[near], xs.ravel()[near], ys.ravel()[near]
        run = np.nonzero(np.diff(dd) == 1)[0]
        assert run.size > 100 and d0 in dd
        assert np.all(np.abs(xx[run + 1] - xx[run]) + np.abs(yy[run + 1] - yy[run]) == 1)
