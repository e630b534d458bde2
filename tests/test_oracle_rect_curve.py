"""Pins of the generalized (rectangular) Hilbert curve in the oracle: a bijection onto the
rectangle whose steps are grid moves (diagonal ones only where a side is odd), equal to the
classic curve (itself pinned to an L-system) on 2^m squares, and a visibly better
neighbourhood than the enclosing-square curve on the workloads' frames."""
import numpy as np
import pytest

import oracle as O


@pytest.mark.parametrize("W,H", [(1, 1), (1, 7), (7, 1), (2, 3), (3, 2), (5, 5), (6, 4), (9, 14), (31, 17),
                                 (80, 45), (52, 30), (45, 30), (16, 16), (40, 40)])
def test_bijection_and_steps(W, H):
    c = O.rect_hilbert_curve(W, H)
    assert c.shape == (W * H, 2)
    assert (c[:, 0] >= 0).all() and (c[:, 0] < W).all() and (c[:, 1] >= 0).all() and (c[:, 1] < H).all()
    assert len({(int(x), int(y)) for x, y in c}) == W * H
    assert c[0].tolist() == [0, 0]
    if W * H > 1:
        d = np.abs(np.diff(c, axis=0))
        assert d.max() <= 1 and (d.sum(axis=1) >= 1).all()    # unit or diagonal moves only
        if W % 2 == 0 and H % 2 == 0:
            assert (d.sum(axis=1) == 1).all()                  # even sides: unit moves only


def test_every_small_rectangle():
    for W in range(1, 25):
        for H in range(1, 25):
            c = O.rect_hilbert_curve(W, H)
            assert len({(int(x), int(y)) for x, y in c}) == W * H
            if W * H > 1:
                assert np.abs(np.diff(c, axis=0)).max() <= 1


@pytest.mark.parametrize("m", range(0, 7))
def test_equals_classic_curve_on_power_of_two_squares(m):
    np.testing.assert_array_equal(O.rect_hilbert_curve(2 ** m, 2 ** m), O.hilbert_curve(m))


@pytest.mark.parametrize("T,Hg,Wg", [(21, 45, 80), (21, 30, 52), (13, 30, 45)])
def test_frames_are_contiguous_walks(T, Hg, Wg):
    perm, inv = O.rect_curve_perm(T, Hg, Wg)
    np.testing.assert_array_equal(perm[inv], np.arange(T * Hg * Wg))
    f = perm.reshape(T, Hg * Wg)
    assert (f // (Hg * Wg) == np.arange(T)[:, None]).all()
    y, x = (f[0] % (Hg * Wg)) // Wg, f[0] % Wg
    steps = np.abs(np.diff(y)) + np.abs(np.diff(x))
    # enclosing-square curve on the same frame: its skipped cells break adjacency
    p0, _ = O.hilbert_perm(1, Hg, Wg)
    y0, x0 = p0 // Wg, p0 % Wg
    steps0 = np.abs(np.diff(y0)) + np.abs(np.diff(x0))
    assert steps.max() <= 2 and steps0.max() > 2
    assert steps.mean() < steps0.mean()
