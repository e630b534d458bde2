"""Failure detection on the GPU without a fault: the attention kernels' mbarrier waits are
bounded. With FVA_DIAG_WITHHOLD_Q each CTA never requests its Q tile, so the waits behind
it can never complete; with a 20 ms limit they run out, the kernel reports
FVA_DEVERR_TIMEOUT through dev_status, drains its own loads and MMAs, frees TMEM and
exits. The context stays usable and the next call (normal settings) is correct."""
import numpy as np
import pytest

from adaptive_block_sparse_hilbert_b200 import synth
import oracle as O
from tests import _common as C

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dense", [False, True])
def test_wait_timeout_reports_and_context_recovers(dense):
    import torch
    from adaptive_block_sparse_hilbert_b200 import fva
    wl = synth.custom_workload(4, 20, 20, 3, 128, "bf16", seed=51)
    L = synth.make_layer(wl)
    run = C.GpuRun(wl, L)
    lay = run.layer
    o = torch.zeros_like(lay.qh)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    fva.fva_set_diagnostics(20_000_000, fva.FVA_DIAG_WITHHOLD_Q)
    try:
        if dense:
            fva.fva_dense_attn(run.shape, lay.qh, lay.kh, lay.vh, o, 0.0, st)
        else:
            fva.fva_sparse_attn(run.shape, lay.qh, lay.kh, lay.vh, lay.mask, o, 0.0, st)
        torch.cuda.synchronize()
    finally:
        fva.fva_set_diagnostics(0, 0)
    assert int(st.item()) == fva.FVA_DEVERR_TIMEOUT
    # the device is still usable and the kernel is correct again with the default limit
    st.zero_()
    if dense:
        fva.fva_dense_attn(run.shape, lay.qh, lay.kh, lay.vh, o, 0.0, st)
    else:
        fva.fva_sparse_attn(run.shape, lay.qh, lay.kh, lay.vh, lay.mask, o, 0.0, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    perm, _ = O.hilbert_perm(wl.T, wl.Hg, wl.Wg)
    qh, kh, vh = C.hilbert_bhnd(L, perm)
    if dense:
        want = O.dense_attention(qh, kh, vh)
    else:
        g = run.mask_np()
        want = O.assemble(O.block_sparse_attention(qh, kh, vh, g["row_ptr"], g["col_idx"]), wl.B, wl.H, wl.N, wl.d)
    mx, mean = C.err_stats(o.float().cpu().numpy(), want)
    assert mx <= C.BF16_MAX_ABS and mean <= C.BF16_MEAN_ABS, (mx, mean)
