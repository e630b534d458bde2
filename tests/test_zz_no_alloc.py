"""fva_route_noalloc: routing for callers that cannot allocate device memory (a plugin whose
host owns every device allocation, a service that allocates nothing after start-up).

It must give exactly the mask, tiles and work list of fva_route with a caller
workspace, on every call: two workloads in a row (the second call finds the first call's
larger scratch contents still in the library's fixed array), and the same inputs again
into a mask that already holds the previous result. It must turn away shapes whose
scratch does not fit before doing any work.

The file name sorts after every other test file, so pytest collects it last: a GPU run
that stops at its first failure has then run all the other GPU tests before this one.
"""
import ctypes

import numpy as np
import pytest

from adaptive_block_sparse_hilbert_b200 import synth
from tests import _common as C

pytestmark = pytest.mark.gpu


def _noalloc_mask(run, p, k_floor, use_pooled, m=None):
    """Route through fva_route_noalloc into mask `m` (a fresh one when None); returns the
    mask's contents and the mask."""
    import torch
    from adaptive_block_sparse_hilbert_b200 import fva
    if m is None:
        m = fva.Mask.allocate(run.shape)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    lay = run.layer
    if use_pooled:
        fva.fva_route_noalloc(run.shape, None, None, lay.pooled_q, lay.pooled_k, p, k_floor, m, lay.order, st)
    else:
        fva.fva_route_noalloc(run.shape, lay.qh, lay.kh, None, None, p, k_floor, m, lay.order, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    rp = m.row_ptr.cpu().numpy().astype(np.int64)
    tp = m.tile_ptr.cpu().numpy().astype(np.int64)
    return {
        "row_ptr": rp, "col_idx": m.col_idx[: int(rp[-1])].cpu().numpy().astype(np.int64),
        "head_kept": m.head_kept.cpu().numpy(), "tile_ptr": tp,
        "tile_col": m.tile_col[: int(tp[-1])].cpu().numpy().astype(np.int64),
        "tile_cost": m.tile_cost.cpu().numpy().astype(np.int64),
        "worklist": m.worklist.cpu().numpy().astype(np.int64),
    }, m


def test_noalloc_route_matches_workspace_route_twice():
    cases = [
        # (workload, p, k_floor, pass pooled Q/K in)
        (synth.custom_workload(6, 30, 45, 8, 64, "bf16", seed=41), 0.9, 2, True),
        (synth.custom_workload(8, 24, 24, 16, 128, "bf16", seed=42, tau=("logU", 1.0, 5.0)), 0.8, 4, False),
    ]
    for wl, p, kf, use_pooled in cases:
        L = synth.make_layer(wl)
        run = C.GpuRun(wl, L, p=p, k_floor=kf)          # fva_route with a caller workspace
        want = run.mask_np()
        got, m = _noalloc_mask(run, p, kf, use_pooled)   # the same inputs, no workspace
        again, _ = _noalloc_mask(run, p, kf, use_pooled, m)  # once more, into the filled mask
        for key in want:
            np.testing.assert_array_equal(got[key], want[key], err_msg=f"{wl.name}: {key}")
            np.testing.assert_array_equal(again[key], want[key], err_msg=f"{wl.name}: {key} (repeat)")


def test_noalloc_rejects_shapes_beyond_its_scratch():
    from adaptive_block_sparse_hilbert_b200 import fva
    wl = synth.WORKLOADS[1]  # 40 heads x 512 blocks: ~84 MB of block logits
    s = C.shape_of(wl)
    assert fva.fva_route_workspace_bytes(s, False) > fva.ROUTE_NOALLOC_SCRATCH_BYTES
    m = fva.fva_mask(16, 16, 1 << 40, 16, 16, 16, 1 << 40, 16, 16)  # never touched: rejected first
    rc = fva.call_raw("fva_route_noalloc", ctypes.byref(s), None, None, ctypes.c_void_p(256), ctypes.c_void_p(256),
                      0.9, 4, 2, ctypes.byref(m), None, None)
    assert rc == fva.FVA_ERR_TOO_LARGE
    assert "no-alloc" in fva.status_string(rc)
