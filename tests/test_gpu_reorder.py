"""GPU parity: Hilbert permutation, reorder with fused pooling, inverse reorder (C ABI vs oracle).

Integer and copy work is compared bit-exactly; the float64 pooled means up to the last
bit of a float64 sum (the GPU sums bf16/fp32 inputs exactly in float64 for these
inputs, the oracle with numpy).
"""
import numpy as np
import pytest

from adaptive_block_sparse_hilbert_b200 import synth
import oracle as O
from tests import _common as C

pytestmark = pytest.mark.gpu

GRIDS = [(4, 16, 16), (21, 30, 52), (21, 45, 80), (13, 30, 45), (1, 1, 1), (3, 5, 3), (2, 7, 130), (5, 129, 2)]


@pytest.mark.parametrize("T,Hg,Wg", GRIDS)
def test_hilbert_perm_exact(T, Hg, Wg):
    import torch
    from adaptive_block_sparse_hilbert_b200 import fva
    s = fva.make_shape(1, 1, 64, T, Hg, Wg, "bf16")
    N = T * Hg * Wg
    perm = torch.empty(N, dtype=torch.int32, device="cuda")
    inv = torch.empty(N, dtype=torch.int32, device="cuda")
    fva.fva_hilbert_perm(s, perm, inv)
    torch.cuda.synchronize()
    want_p, want_i = O.hilbert_perm(T, Hg, Wg)
    np.testing.assert_array_equal(perm.cpu().numpy(), want_p)
    np.testing.assert_array_equal(inv.cpu().numpy(), want_i)


# frames at the side limit (65536, an enclosing square of 4^16 cells), long strips and a
# large near-square frame; the oracle sorts the cells by their index on the curve
LARGE_FRAMES = [(1, 2, 65536), (1, 65536, 2), (2, 3, 40000), (1, 1, 65536), (1, 1500, 1300), (1, 4097, 5)]


@pytest.mark.parametrize("T,Hg,Wg", LARGE_FRAMES)
def test_hilbert_perm_exact_on_large_frames(T, Hg, Wg):
    import torch
    from adaptive_block_sparse_hilbert_b200 import fva
    s = fva.make_shape(1, 1, 64, T, Hg, Wg, "bf16")
    N = T * Hg * Wg
    perm = torch.empty(N, dtype=torch.int32, device="cuda")
    inv = torch.empty(N, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    fva.fva_hilbert_perm(s, perm, inv)
    torch.cuda.synchronize()
    want_p, want_i = O.hilbert_perm_by_index(T, Hg, Wg)
    np.testing.assert_array_equal(perm.cpu().numpy(), want_p)
    np.testing.assert_array_equal(inv.cpu().numpy(), want_i)
    if Hg * Wg <= 200000:
        fva.fva_curve_perm(s, fva.FVA_CURVE_RECT, perm, inv, st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        np.testing.assert_array_equal(perm.cpu().numpy(), O.rect_curve_perm(T, Hg, Wg)[0])


@pytest.mark.parametrize("T,Hg,Wg", GRIDS + [(1, 40, 40), (2, 1, 77), (3, 33, 17)])
def test_rect_curve_perm_exact(T, Hg, Wg):
    import torch
    from adaptive_block_sparse_hilbert_b200 import fva
    s = fva.make_shape(1, 1, 64, T, Hg, Wg, "bf16")
    N = T * Hg * Wg
    perm = torch.empty(N, dtype=torch.int32, device="cuda")
    inv = torch.empty(N, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    fva.fva_curve_perm(s, fva.FVA_CURVE_RECT, perm, inv, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    want_p, want_i = O.rect_curve_perm(T, Hg, Wg)
    np.testing.assert_array_equal(perm.cpu().numpy(), want_p)
    np.testing.assert_array_equal(inv.cpu().numpy(), want_i)
    # the plain curve through the same entry point is fva_hilbert_perm's order
    fva.fva_curve_perm(s, fva.FVA_CURVE_HILBERT, perm, inv, st)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(perm.cpu().numpy(), O.hilbert_perm(T, Hg, Wg)[0])


SMALL = [
    synth.WORKLOADS[0],
    synth.custom_workload(3, 10, 13, 3, 64, "bf16", seed=11),    # N = 390, tail block of 6
    synth.custom_workload(2, 9, 9, 2, 128, "bf16", seed=12),     # N = 162, tail of 34
    synth.custom_workload(1, 8, 8, 2, 128, "f32", seed=13),      # exactly one block
    synth.custom_workload(2, 5, 7, 2, 64, "f32", seed=14),       # N = 70
    synth.custom_workload(3, 12, 17, 3, 128, "bf16", seed=15, B=2),  # two batch entries
    synth.custom_workload(3, 5, 7, 2, 64, "f32", seed=16, B=3),     # three entries, fp32
    # rows shorter than 256 B move two or four adjacent heads per CTA
    synth.custom_workload(3, 10, 13, 4, 32, "bf16", seed=17),           # 64 B rows, 4 heads per CTA
    synth.custom_workload(3, 10, 13, 6, 32, "bf16", seed=18),           # 64 B rows, H = 6: 2 per CTA
    synth.custom_workload(2, 9, 11, 2, 64, "bf16", seed=19, B=2),       # 128 B rows, 2 per CTA, B = 2
    synth.custom_workload(2, 9, 11, 4, 32, "f32", seed=20),             # 128 B rows, 2 per CTA
    synth.custom_workload(3, 7, 9, 4, 16, "f32", seed=21),              # 64 B rows, 4 per CTA, N = 189
]


@pytest.mark.parametrize("wl", SMALL, ids=lambda w: w.name)
def test_reorder_pool_inverse_small(wl):
    import torch
    from adaptive_block_sparse_hilbert_b200 import fva
    L = synth.make_layer(wl)
    run = C.GpuRun(wl, L)
    perm, _ = O.hilbert_perm(wl.T, wl.Hg, wl.Wg)
    qh, kh, vh = C.hilbert_bhnd(L, perm)
    np.testing.assert_array_equal(run.layer.qh.float().cpu().numpy().astype(np.float64), qh)
    np.testing.assert_array_equal(run.layer.kh.float().cpu().numpy().astype(np.float64), kh)
    # bf16 layers hold V in fp16 (bf16 -> fp16 is exact except below fp16's normal range)
    want_v = vh.astype(np.float16).astype(np.float64) if run.layer.v_fp16 else vh
    np.testing.assert_array_equal(run.layer.vh.float().cpu().numpy().astype(np.float64), want_v)
    np.testing.assert_allclose(run.layer.pooled_q.cpu().numpy(), O.block_mean_pool(qh), rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(run.layer.pooled_k.cpu().numpy(), O.block_mean_pool(kh), rtol=1e-14, atol=1e-15)
    # inverse: Hilbert-ordered K back to raster equals the raster input
    out = torch.empty_like(run.k)
    fva.fva_reorder(run.shape, run.layer.kh, out, None, run.layer.perm, fva.FVA_INV)
    torch.cuda.synchronize()
    assert torch.equal(out, run.k)
    # fva_pool on the reordered tensor equals the fused pooling
    pooled = torch.empty_like(run.layer.pooled_q)
    fva.fva_pool(run.shape, run.layer.qh, pooled)
    torch.cuda.synchronize()
    assert torch.equal(pooled, run.layer.pooled_q)


@pytest.mark.parametrize("wid", [1, 2, 3])
def test_reorder_full_size_sampled(wid):
    """Full-size workloads: sampled rows exact, sampled pooled blocks to float64 rounding."""
    import torch
    from adaptive_block_sparse_hilbert_b200 import fva
    wl = synth.WORKLOADS[wid]
    L = C.layer(wid)
    run = C.GpuRun(wl, L)
    perm, _ = O.hilbert_perm(wl.T, wl.Hg, wl.Wg)
    rng = np.random.default_rng(wid)
    N, nB = wl.N, wl.nB
    heads = rng.choice(wl.H, size=min(4, wl.H), replace=False)
    positions = np.concatenate([rng.choice(N, size=200, replace=False), [0, N - 1]])
    qh = run.layer.qh
    for h in heads:
        got = qh[0, h, torch.as_tensor(positions, device="cuda")].float().cpu().numpy()
        np.testing.assert_array_equal(got, L.q[0, perm[positions], h])
    blocks = np.concatenate([rng.choice(nB, size=16, replace=False), [nB - 1]])
    for h in heads:
        for a in blocks:
            lo, hi = a * 64, min(a * 64 + 64, N)
            want = L.k[0, perm[lo:hi], h].astype(np.float64).sum(axis=0) / (hi - lo)
            np.testing.assert_allclose(run.layer.pooled_k[0, h, a].cpu().numpy(), want, rtol=1e-14, atol=1e-15)
    out = torch.empty_like(run.q)
    fva.fva_reorder(run.shape, run.layer.qh, out, None, run.layer.perm, fva.FVA_INV)
    torch.cuda.synchronize()
    assert torch.equal(out, run.q)
    # V went through the fp16 conversion (round to nearest even)
    vs = run.layer.vh[0, heads[0], torch.as_tensor(positions, device="cuda")].float().cpu().numpy()
    np.testing.assert_array_equal(vs, L.v[0, perm[positions], heads[0]].astype(np.float16).astype(np.float32))


def test_fwd_f16_conversion_exact_and_saturating():
    import torch
    from adaptive_block_sparse_hilbert_b200 import fva
    s = fva.make_shape(1, 2, 64, 1, 3, 43, "bf16")   # N = 129: a 1-token tail block
    N = 129
    x = torch.randn(1, N, 2, 64, device="cuda").to(torch.bfloat16)
    x[0, 5, 1, :8] = torch.tensor([1e5, -1e6, 65504.0, -65504.0, 3e38, 1e-7, -0.0, 2.0 ** -20],
                                  device="cuda").to(torch.bfloat16)
    perm = torch.empty(N, dtype=torch.int32, device="cuda")
    inv = torch.empty(N, dtype=torch.int32, device="cuda")
    fva.fva_hilbert_perm(s, perm, inv)
    y = torch.empty((1, 2, N, 64), dtype=torch.float16, device="cuda")
    fva.fva_reorder(s, x, y, None, perm, fva.FVA_FWD_F16)
    torch.cuda.synchronize()
    ref = x[0, perm.long()].permute(1, 0, 2).float().clamp(-65504.0, 65504.0).to(torch.float16)
    assert torch.equal(y[0], ref)
    pos = int(inv[5].item())
    got = y[0, 1, pos, :5].float().cpu().tolist()
    assert got == [65504.0, -65504.0, 65504.0, -65504.0, 65504.0]
