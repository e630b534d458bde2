"""The host-pipelined layer (head groups copied in, computed on two alternating compute
streams, or one, and copied out) writes the same output as the one-shot device layer, bit
for bit."""
import numpy as np
import pytest

from adaptive_block_sparse_hilbert_b200 import synth
from tests import _common as C

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,H,groups,streams", [(1, 5, 3, 2), (1, 4, 4, 2), (1, 6, 1, 2), (1, 7, None, 2),
                                                (2, 5, 2, 2), (1, 5, 3, 1), (1, 7, None, 3)])
def test_pipelined_equals_one_shot(B, H, groups, streams):
    import torch
    from adaptive_block_sparse_hilbert_b200 import fva, pipeline
    wl = synth.custom_workload(3, 10, 13, H, 128, "bf16", seed=81, B=B)
    L = synth.make_layer(wl)
    s = C.shape_of(wl)
    q, k, v = C.to_device(L)
    one = pipeline.SparseAttentionLayer(s, wl.p, wl.k_floor)
    o_ref = torch.empty_like(q)
    one.forward(q, k, v, o_ref)
    qh, kh, vh = (t.cpu().pin_memory() for t in (q, k, v))
    oh = torch.zeros_like(qh).pin_memory()
    pipe = pipeline.HostPipelinedLayer(s, wl.p, wl.k_floor, groups=groups, compute_streams=streams)
    pipe.forward(qh, kh, vh, oh)
    torch.cuda.synchronize()
    assert pipe.dev_status() == 0 and int(one.dev_status.item()) == 0
    assert torch.equal(oh, o_ref.cpu())


def test_consecutive_layers_overlap_without_races():
    # three layers with different inputs enqueued back to back (their copies and compute
    # overlap across calls), then one wait: each output equals its one-shot layer's
    import torch
    from adaptive_block_sparse_hilbert_b200 import pipeline
    wls = [synth.custom_workload(3, 10, 13, 5, 128, "bf16", seed=91 + i) for i in range(3)]
    s = C.shape_of(wls[0])
    one = pipeline.SparseAttentionLayer(s, wls[0].p, wls[0].k_floor)
    pipe = pipeline.HostPipelinedLayer(s, wls[0].p, wls[0].k_floor, groups=3)
    refs, hosts = [], []
    for wl in wls:
        q, k, v = C.to_device(synth.make_layer(wl))
        o_ref = torch.empty_like(q)
        one.forward(q, k, v, o_ref)
        refs.append(o_ref.cpu())
        hosts.append(tuple(t.cpu().pin_memory() for t in (q, k, v)) + (torch.zeros_like(q.cpu()).pin_memory(),))
    torch.cuda.synchronize()
    for rep in range(2):
        for qh, kh, vh, oh in hosts:
            pipe.forward(qh, kh, vh, oh)
        pipe.wait()
        torch.cuda.synchronize()
        assert pipe.dev_status() == 0
        for (_, _, _, oh), ref in zip(hosts, refs):
            assert torch.equal(oh, ref), rep
        for h in hosts:
            h[3].zero_()


def test_copy_strided_moves_a_head_slice():
    import torch
    from adaptive_block_sparse_hilbert_b200 import fva
    host = torch.arange(2 * 7 * 5 * 8, dtype=torch.float32).reshape(2, 7, 5, 8).pin_memory()
    dev = torch.empty((2, 7, 2, 8), dtype=torch.float32, device="cuda")
    fva.fva_copy_strided(dev, 2 * 8 * 4, host[:, :, 1:3, :], 5 * 8 * 4, 2 * 8 * 4, 14)
    back = torch.zeros_like(host).pin_memory()
    fva.fva_copy_strided(back[:, :, 3:5, :], 5 * 8 * 4, dev, 2 * 8 * 4, 2 * 8 * 4, 14)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(dev.cpu().numpy(), host[:, :, 1:3, :].numpy())
    np.testing.assert_array_equal(back[:, :, 3:5, :].numpy(), host[:, :, 1:3, :].numpy())
    assert (back[:, :, :3, :] == 0).all()
