"""The library's SASA budget rule (fva_sasa_budgets, host code) against the oracle, and
the argument checks of both SASA entry points that need no device."""
import ctypes

import numpy as np
import pytest

from adaptive_block_sparse_hilbert_b200 import fva
from oracle import sasa_oracle as S


@pytest.mark.parametrize("seed", range(30))
def test_budgets_match_oracle(seed):
    rng = np.random.default_rng(seed)
    R = int(rng.integers(1, 9))
    load = rng.uniform(0.0, 10.0, R)
    if seed % 4 == 0:
        load[rng.integers(0, R)] = 0.0
    c = float(rng.uniform(0.001, 0.5))
    n1, n2 = float(rng.choice([0.8, 0.5, 1.0])), float(rng.choice([0.07, 0.0, 0.2]))
    np.testing.assert_array_equal(fva.fva_sasa_budgets(load, c, n1, n2), S.budgets(load, c, n1, n2))


def test_budget_argument_checks():
    L = fva.lib()
    load = (ctypes.c_double * 2)(1.0, 2.0)
    out = (ctypes.c_int64 * 2)()
    assert L.fva_sasa_budgets(load, 2, 0.1, 0.8, 0.07, out) == fva.FVA_OK
    assert L.fva_sasa_budgets(load, 0, 0.1, 0.8, 0.07, out) == fva.FVA_ERR_INVALID_ARG
    assert L.fva_sasa_budgets(load, 2, 0.0, 0.8, 0.07, out) == fva.FVA_ERR_INVALID_ARG
    assert L.fva_sasa_budgets(load, 2, 0.1, -0.1, 0.07, out) == fva.FVA_ERR_INVALID_ARG
    bad = (ctypes.c_double * 2)(1.0, float("inf"))
    assert L.fva_sasa_budgets(bad, 2, 0.1, 0.8, 0.07, out) == fva.FVA_ERR_INVALID_ARG


def test_augment_argument_checks():
    s = fva.make_shape(1, 2, 64, 2, 8, 8, "bf16")
    L = fva.lib()
    m = fva.fva_mask()
    ws = fva.fva_sasa_workspace_bytes(s)
    assert ws > fva.fva_route_workspace_bytes(s, False)
    p = 1024  # never dereferenced: every call below fails its host checks first
    assert L.fva_sasa_augment(ctypes.byref(s), None, p, p, 2, p, 2, ctypes.byref(m), p, ws, None, None, None) == \
        fva.FVA_ERR_INVALID_ARG
    assert L.fva_sasa_augment(ctypes.byref(s), p, p, p, 0, p, 2, ctypes.byref(m), p, ws, None, None, None) == \
        fva.FVA_ERR_INVALID_ARG
    assert L.fva_sasa_augment(ctypes.byref(s), p, p, p, 65, p, 2, ctypes.byref(m), p, ws, None, None, None) == \
        fva.FVA_ERR_INVALID_ARG
    assert L.fva_sasa_augment(ctypes.byref(s), p, p, p, 2, p, 9, ctypes.byref(m), p, ws, None, None, None) == \
        fva.FVA_ERR_INVALID_ARG
    # an empty mask struct: missing output arrays
    assert L.fva_sasa_augment(ctypes.byref(s), p, p, p, 2, p, 2, ctypes.byref(m), p, ws, None, None, None) == \
        fva.FVA_ERR_INVALID_ARG
