"""GPU parity: block-sparse and dense attention (C ABI vs oracle).

Tolerances: bf16 inputs max-abs 2e-2 and mean-abs 2e-3; fp32 inputs max-abs 1e-4. Both
sides use the same (GPU-routed) mask, so outputs are compared on every row; the masks
themselves are checked against the oracle in test_gpu_route.py.
"""
import numpy as np
import pytest

from adaptive_block_sparse_hilbert_b200 import synth
import oracle as O
from tests import _common as C

pytestmark = pytest.mark.gpu


def _run_sparse(run):
    import torch
    run.layer.attend()
    torch.cuda.synchronize()
    assert run.status() == 0
    return run.layer.oh.float().cpu().numpy().astype(np.float64)


def _run_dense(run):
    import torch
    from adaptive_block_sparse_hilbert_b200 import fva
    o = torch.empty_like(run.layer.qh)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    fva.fva_dense_attn(run.shape, run.layer.qh, run.layer.kh, run.layer.vh, o, 0.0, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return o.float().cpu().numpy().astype(np.float64)


def _tol(wl, got, want, what):
    mx, mean = C.err_stats(got, want)
    print(f"{wl.name} {what}: max-abs {mx:.3e} mean-abs {mean:.3e}")
    if wl.dtype == "bf16":
        assert mx <= C.BF16_MAX_ABS and mean <= C.BF16_MEAN_ABS, (mx, mean)
    else:
        assert mx <= C.F32_MAX_ABS, mx


SMALL = [
    synth.WORKLOADS[0],                                                  # fp32, 16 blocks
    synth.custom_workload(3, 10, 13, 3, 64, "bf16", seed=31),            # nB = 7 (odd), tail of 6
    synth.custom_workload(2, 9, 9, 2, 128, "bf16", seed=32),             # nB = 3, tail of 34
    synth.custom_workload(4, 20, 20, 2, 128, "bf16", seed=33, tau=("logU", 2.0, 6.0)),  # sparse
    synth.custom_workload(1, 8, 8, 1, 64, "bf16", seed=34),              # a single block
    synth.custom_workload(2, 5, 7, 2, 64, "f32", seed=35),               # fp32 ragged
    synth.custom_workload(5, 16, 16, 2, 128, "bf16", seed=36, p=0.7, k_floor=1),
    synth.custom_workload(3, 12, 17, 3, 128, "bf16", seed=42, B=2, p=0.8, k_floor=1),  # two batch entries
    synth.custom_workload(3, 12, 17, 2, 64, "f32", seed=43, B=3, p=0.8, k_floor=1),    # fp32, three entries
    synth.custom_workload(2, 9, 11, 2, 32, "f32", seed=44, p=0.8, k_floor=1),          # fp32 d = 32
    synth.custom_workload(2, 9, 11, 2, 128, "f32", seed=45, p=0.8, k_floor=1),         # fp32 d = 128
]


@pytest.mark.parametrize("wl", SMALL, ids=lambda w: w.name)
def test_sparse_and_dense_small(wl):
    L = synth.make_layer(wl)
    run = C.GpuRun(wl, L)
    g = run.mask_np()
    perm, _ = O.hilbert_perm(wl.T, wl.Hg, wl.Wg)
    qh, kh, vh = C.hilbert_bhnd(L, perm)
    want = O.assemble(O.block_sparse_attention(qh, kh, vh, g["row_ptr"], g["col_idx"]), wl.B, wl.H, wl.N, wl.d)
    _tol(wl, _run_sparse(run), want, "sparse")
    _tol(wl, _run_dense(run), O.dense_attention(qh, kh, vh), "dense")


@pytest.mark.parametrize("d", [64, 128])
def test_bf16_v_path(d):
    """The kernel variant that rounds P to bf16 (V kept in bf16) also meets the tolerance."""
    import torch
    from adaptive_block_sparse_hilbert_b200 import fva
    wl = synth.custom_workload(3, 10, 13, 2, d, "bf16", seed=40)
    L = synth.make_layer(wl)
    run = C.GpuRun(wl, L)
    vb = torch.empty(run.layer.vh.shape, dtype=torch.bfloat16, device="cuda")
    fva.fva_reorder(run.shape, run.v, vb, None, run.layer.perm, fva.FVA_FWD)
    o = torch.empty_like(run.layer.qh)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    fva.fva_sparse_attn(run.shape, run.layer.qh, run.layer.kh, vb, run.layer.mask, o, 0.0, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    g = run.mask_np()
    perm, _ = O.hilbert_perm(wl.T, wl.Hg, wl.Wg)
    qh, kh, vh = C.hilbert_bhnd(L, perm)
    want = O.assemble(O.block_sparse_attention(qh, kh, vh, g["row_ptr"], g["col_idx"]), wl.B, wl.H, wl.N, wl.d)
    _tol(wl, o.float().cpu().numpy().astype(np.float64), want, "sparse-bf16V")


def test_end_to_end_raster_output():
    """forward(): reorder -> route -> attention -> inverse reorder equals the oracle in raster order."""
    import torch
    wl = synth.custom_workload(3, 10, 13, 3, 64, "bf16", seed=37)
    L = synth.make_layer(wl)
    run = C.GpuRun(wl, L)
    out = torch.empty_like(run.q)
    run.layer.forward(run.q, run.k, run.v, out)
    torch.cuda.synchronize()
    g = run.mask_np()
    perm, _ = O.hilbert_perm(wl.T, wl.Hg, wl.Wg)
    qh, kh, vh = C.hilbert_bhnd(L, perm)
    want_h = O.assemble(O.block_sparse_attention(qh, kh, vh, g["row_ptr"], g["col_idx"]), wl.B, wl.H, wl.N, wl.d)
    _tol(wl, out.float().cpu().numpy().astype(np.float64), O.inverse_reorder(want_h, perm), "forward")


def _custom_mask_run(wl, lists_fn):
    """Run the sparse kernel with a hand-made CSR mask (tiles built by fva_build_tiles)."""
    import torch
    from adaptive_block_sparse_hilbert_b200 import fva
    L = synth.make_layer(wl)
    run = C.GpuRun(wl, L)
    BH, nB = wl.B * wl.H, wl.nB
    lists = [np.array(sorted(lists_fn(bh, a)), dtype=np.int32) for bh in range(BH) for a in range(nB)]
    rp = np.concatenate([[0], np.cumsum([x.size for x in lists])]).astype(np.int32)
    ci = np.concatenate(lists).astype(np.int32)
    m = fva.Mask.allocate(run.shape)
    m.row_ptr.copy_(torch.from_numpy(rp))
    m.col_idx[: ci.size].copy_(torch.from_numpy(ci))
    ws = torch.empty(fva.fva_tiles_workspace_bytes(run.shape), dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    fva.fva_build_tiles(run.shape, m, ws, fva.FVA_ORDER_LPT, st)
    o = torch.empty_like(run.layer.qh)
    fva.fva_sparse_attn(run.shape, run.layer.qh, run.layer.kh, run.layer.vh, m, o, 0.0, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    perm, _ = O.hilbert_perm(wl.T, wl.Hg, wl.Wg)
    qh, kh, vh = C.hilbert_bhnd(L, perm)
    want = O.assemble(O.block_sparse_attention(qh, kh, vh, rp.astype(np.int64), ci.astype(np.int64)),
                      wl.B, wl.H, wl.N, wl.d)
    return o.float().cpu().numpy().astype(np.float64), want, vh


@pytest.mark.parametrize("d", [64, 128])
def test_single_key_block_returns_its_value(d):
    # N = 64*4 + 1: every row keeps only the 1-key tail block, so o = v[last] (bf16-rounded)
    wl = synth.custom_workload(1, 1, 257, 2, d, "bf16", seed=38)
    got, want, vh = _custom_mask_run(wl, lambda bh, a: [4])
    _tol(wl, got, want, "one-key")
    np.testing.assert_allclose(got[:, :, :, :], np.broadcast_to(vh[:, :, 256:257, :], got.shape), rtol=0, atol=1e-2)


@pytest.mark.parametrize("d", [64, 128])
def test_disjoint_pair_lists_and_all_blocks(d):
    # rows 2t and 2t+1 keep disjoint lists (worst case for the pair union), plus all-block rows
    wl = synth.custom_workload(3, 12, 12, 2, d, "bf16", seed=39)   # N = 432, nB = 7
    got, want, _ = _custom_mask_run(wl, lambda bh, a: [a] if a % 2 == 0 else ([b for b in range(7) if b != a - 1]))
    _tol(wl, got, want, "disjoint")
    got, want, _ = _custom_mask_run(wl, lambda bh, a: list(range(7)))
    _tol(wl, got, want, "all-blocks")


@pytest.mark.parametrize("d,dtype", [(64, "bf16"), (128, "bf16"), (64, "f32")])
def test_empty_rows_and_empty_pair_tiles(d, dtype):
    # a caller-made mask where rows 0, 2, 3 and 6 keep nothing: tile 1 (rows 2, 3) and
    # tile 3 (row 6 and the missing row 7) have no work at all; empty rows come out as
    # zeros and the other rows are unaffected
    wl = synth.custom_workload(3, 12, 12, 2, d, dtype, seed=40)   # N = 432, nB = 7
    keep = {1: [0, 3], 4: [4, 6], 5: [1]}
    got, want, _ = _custom_mask_run(wl, lambda bh, a: keep.get(a, []))
    _tol(wl, got, want, "empty rows")
    for a in (0, 2, 3, 6):
        assert np.all(got[:, :, a * 64:min(a * 64 + 64, wl.N)] == 0.0), a


def _sampled_check(wl, L, n_per_head, seed):
    """Route and attend one layer in the benchmark's launch configuration, then compare
    sampled query blocks (always the densest and the sparsest rows) with the oracle."""
    run = C.GpuRun(wl, L)
    mx, mean, n_rows = C.sampled_attention_errors(run, wl, L, run.mask_np(), n_per_head, seed)
    print(f"{wl.name}: sampled {n_rows} query blocks max-abs {mx:.3e} mean-abs {mean:.3e}")
    assert mx <= C.BF16_MAX_ABS and mean <= C.BF16_MEAN_ABS


@pytest.mark.parametrize("wid", [1, 3, 2])
def test_sparse_full_size_sampled(wid):
    """Full-size workloads in the benchmark's launch configuration; sampled query blocks."""
    _sampled_check(synth.WORKLOADS[wid], C.layer(wid), 6, wid)


def test_sparse_at_largest_routable_shape():
    """One head of 724,842 tokens (nB = 11326, the routing limit), 5,663 pair tiles."""
    wl = C.largest_routable_workload()
    _sampled_check(wl, synth.make_layer(wl), 10, 41)


def test_dense_full_size_sampled_480p():
    import torch
    from adaptive_block_sparse_hilbert_b200 import fva
    wl = synth.WORKLOADS[1]
    L = C.layer(1)
    run = C.GpuRun(wl, L)
    o = torch.empty_like(run.layer.qh)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    fva.fva_dense_attn(run.shape, run.layer.qh, run.layer.kh, run.layer.vh, o, 0.0, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    perm, _ = O.hilbert_perm(wl.T, wl.Hg, wl.Wg)
    rng = np.random.default_rng(5)
    for bh in rng.choice(wl.H, size=3, replace=False):
        qh = O.reorder(L.q[:, :, bh:bh + 1], perm)[0, 0]
        kh = O.reorder(L.k[:, :, bh:bh + 1], perm)[0, 0]
        vh = O.reorder(L.v[:, :, bh:bh + 1], perm)[0, 0]
        rows = np.concatenate([rng.choice(wl.N, size=64, replace=False), [wl.N - 1]])
        want = O.attention_rows(qh[rows], kh, vh, np.arange(wl.N), 1.0 / np.sqrt(wl.d))
        gv = o[0, bh, torch.as_tensor(rows, device="cuda")].float().cpu().numpy()
        mx, mean = C.err_stats(gv, want)
        assert mx <= C.BF16_MAX_ABS and mean <= C.BF16_MEAN_ABS, (mx, mean)


@pytest.mark.parametrize("d", [64, 128])
def test_sparse_attn_range_slices_the_work_list(d):
    """fva_sparse_attn_range: two ranges that cover the work list give fva_sparse_attn's
    output bit for bit; a range leaves the rows of every tile outside it untouched."""
    import torch
    from adaptive_block_sparse_hilbert_b200 import fva
    wl = synth.custom_workload(3, 12, 17, 3, d, "bf16", seed=46)   # nB = 10, 15 pair tiles
    run = C.GpuRun(wl, synth.make_layer(wl))
    lay = run.layer
    lay.attend()
    torch.cuda.synchronize()
    full = lay.oh.clone()
    tiles = fva.fva_num_tiles(run.shape)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    o = torch.full_like(full, float("nan"))
    for first, n in ((0, 6), (6, tiles - 6)):
        fva.fva_sparse_attn_range(run.shape, lay.qh, lay.kh, lay.vh, lay.mask, o, first, n, 0.0, st)
    fva.fva_sparse_attn_range(run.shape, lay.qh, lay.kh, lay.vh, lay.mask, o, 3, 0, 0.0, st)  # empty: no launch
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert torch.equal(o, full)
    # only the first 6 slots: their tiles' rows are written, every other row keeps its NaN
    o = torch.full_like(full, float("nan"))
    fva.fva_sparse_attn_range(run.shape, lay.qh, lay.kh, lay.vh, lay.mask, o, 0, 6, 0.0, st)
    torch.cuda.synchronize()
    wlist = lay.mask.worklist.cpu().numpy()
    n_pairs = (wl.nB + 1) // 2
    written = torch.zeros(wl.H, wl.N, dtype=torch.bool)
    for tile in wlist[:6]:
        h, t = divmod(int(tile), n_pairs)
        written[h, t * 128:min(t * 128 + 128, wl.N)] = True
    got = o[0].cpu()
    assert torch.equal(got[written], full[0].cpu()[written])
    assert torch.isnan(got[~written].float()).all()


def test_work_list_entry_out_of_range_is_reported_not_followed():
    """A work-list entry that names no tile: the kernel reports FVA_DEVERR_BAD_LIST, its CTA
    writes nothing, and every other tile's rows are still computed."""
    import torch
    from adaptive_block_sparse_hilbert_b200 import fva
    wl = synth.custom_workload(3, 12, 17, 2, 128, "bf16", seed=47)   # nB = 10, 10 pair tiles
    run = C.GpuRun(wl, synth.make_layer(wl))
    lay = run.layer
    lay.attend()
    torch.cuda.synchronize()
    full = lay.oh.clone()
    bad_slot = 4
    victim = int(lay.mask.worklist[bad_slot].item())
    lay.mask.worklist[bad_slot] = fva.fva_num_tiles(run.shape) + 7   # no such tile
    o = torch.full_like(full, float("nan"))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    fva.fva_sparse_attn(run.shape, lay.qh, lay.kh, lay.vh, lay.mask, o, 0.0, st)
    torch.cuda.synchronize()
    assert int(st.item()) == fva.FVA_DEVERR_BAD_LIST
    n_pairs = (wl.nB + 1) // 2
    h, t = divmod(victim, n_pairs)
    skipped = torch.zeros(wl.H, wl.N, dtype=torch.bool)
    skipped[h, t * 128:min(t * 128 + 128, wl.N)] = True
    got = o[0].cpu()
    assert torch.isnan(got[skipped].float()).all()                  # the named-nothing CTA wrote nothing
    assert torch.equal(got[~skipped], full[0].cpu()[~skipped])     # the rest is intact
