"""The per-CTA trace of the attention kernel: one record per launched tile, in work-list
order, with the SM it ran on, its list length and a start no later than its end; the
traced launch writes the same output as an untraced one, and a trace buffer that is too
small is refused before launch."""
import numpy as np
import pytest

from adaptive_block_sparse_hilbert_b200 import synth
from tests import _common as C

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dense", [False, True])
def test_cta_trace_records_every_tile(dense):
    import torch
    from adaptive_block_sparse_hilbert_b200 import fva
    wl = synth.custom_workload(4, 20, 20, 3, 128, "bf16", seed=61, tau=("logU", 1.0, 6.0))
    L = synth.make_layer(wl)
    run = C.GpuRun(wl, L)
    lay = run.layer
    tiles = fva.fva_num_tiles(run.shape)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")

    def attend(o):
        if dense:
            fva.fva_dense_attn(run.shape, lay.qh, lay.kh, lay.vh, o, 0.0, st)
        else:
            fva.fva_sparse_attn(run.shape, lay.qh, lay.kh, lay.vh, lay.mask, o, 0.0, st)

    o_plain = torch.zeros_like(lay.qh)
    attend(o_plain)
    trace = torch.full((tiles, 4), -1, dtype=torch.int64, device="cuda")
    o_traced = torch.zeros_like(lay.qh)
    fva.fva_set_cta_trace(trace)
    try:
        attend(o_traced)
        torch.cuda.synchronize()
    finally:
        fva.fva_set_cta_trace(None)
    assert int(st.item()) == 0
    assert torch.equal(o_plain, o_traced)
    t = trace.cpu().numpy()
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert (t[:, 0] >= 0).all() and (t[:, 0] < sms).all()
    assert (t[:, 2] > 0).all() and (t[:, 3] >= t[:, 2]).all()
    nB = wl.nB
    if dense:
        assert (t[:, 1] == nB).all()
    else:
        tp = lay.mask.tile_ptr.cpu().numpy().astype(np.int64)
        wlist = lay.mask.worklist.cpu().numpy().astype(np.int64)
        np.testing.assert_array_equal(t[:, 1], tp[wlist + 1] - tp[wlist])
    # a buffer one CTA short is refused before launch
    small = torch.zeros((tiles - 1, 4), dtype=torch.int64, device="cuda")
    fva.fva_set_cta_trace(small)
    try:
        with pytest.raises(fva.FvaError) as e:
            attend(o_traced)
        assert e.value.status == fva.FVA_ERR_CAPACITY
    finally:
        fva.fva_set_cta_trace(None)
