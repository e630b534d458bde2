"""GPU: the head-sharded step with RLB head migration (migrate.ShardRank) on ranks emulated
in one process on one GPU (run_virtual_step: the phases run rank after rank and the
transfers are device copies into the receivers' own buffers).

Heads are independent along the whole path, so every rank's output must equal the
unsharded layer's output for its heads bit for bit, whether a head was computed at home
or routed and attended on the rank it migrated to; and a donor's attention launches must
leave exactly its migrated head's tiles out of the work list.
"""
import numpy as np
import pytest

from adaptive_block_sparse_hilbert_b200 import synth
from tests import _common as C

pytestmark = pytest.mark.gpu


def _layers(wl, world):
    import torch
    from adaptive_block_sparse_hilbert_b200 import fva, migrate, pipeline
    L = synth.make_layer(wl)
    q, k, v = C.to_device(L)
    s = C.shape_of(wl)
    whole = pipeline.SparseAttentionLayer(s, wl.p, wl.k_floor)
    o_whole = torch.empty_like(q)
    whole.forward(q, k, v, o_whole)
    ranks, qs, ks, vs, os_ = [], [], [], [], []
    for r in range(world):
        hs = migrate.heads_of_rank(r, world, wl.H)
        ranks.append(migrate.ShardRank(s, wl.p, wl.k_floor, r, world, ms_per_step=1e-3))
        for lst, x in ((qs, q), (ks, k), (vs, v)):
            lst.append(x[:, :, hs.start:hs.stop].contiguous())
        os_.append(torch.full_like(qs[-1], float("nan")))
    return whole, o_whole, ranks, qs, ks, vs, os_


CASES = [
    # (workload, ranks): heads of very different density so that the planner moves some
    (synth.custom_workload(4, 16, 24, 6, 64, "bf16", seed=94, tau=("logU", 0.3, 8.0), p=0.9, k_floor=1), 3),
    (synth.custom_workload(5, 24, 30, 8, 128, "bf16", seed=96, tau=("logU", 0.3, 8.0), p=0.9, k_floor=2), 4),
]


@pytest.mark.parametrize("wl,world", CASES, ids=lambda c: getattr(c, "name", str(c)))
def test_virtual_ranks_match_the_unsharded_layer(wl, world):
    import torch
    from adaptive_block_sparse_hilbert_b200 import migrate
    whole, o_whole, ranks, qs, ks, vs, os_ = _layers(wl, world)
    loads, rank_of, moves = migrate.run_virtual_step(ranks, qs, ks, vs, os_, comm_ms=0.0)
    torch.cuda.synchronize()
    print(f"{wl.name}: loads {np.round(loads, 3).tolist()} moves {[(m.head, m.src, m.dst) for m in moves]}")
    assert all(r.dev_status() == 0 for r in ranks)
    assert len({m.src for m in moves}) == len(moves)
    # per-head loads: the whole layer's issued tile steps of each head
    steps = whole.mask.tile_cost.cpu().numpy().reshape(wl.B, wl.H, -1).sum(axis=(0, 2))
    np.testing.assert_allclose(loads, steps * 1e-3)
    got = torch.cat(os_, dim=2)
    assert torch.equal(got, o_whole), "sharded output differs from the unsharded layer"


def test_given_moves_with_two_batch_entries():
    """B = 2 (a head's slices of both entries travel, and both come back): moves given to
    the step instead of planned -- head 0 from rank 0 to rank 2, head 3 from rank 1 to 0."""
    import torch
    from adaptive_block_sparse_hilbert_b200 import migrate
    wl = synth.custom_workload(3, 16, 20, 6, 128, "bf16", seed=97, tau=("logU", 0.3, 8.0), B=2)
    whole, o_whole, ranks, qs, ks, vs, os_ = _layers(wl, 3)
    moves = [migrate.Move(0, 0, 2, 0.0), migrate.Move(3, 1, 0, 0.0)]
    _, rank_of, got_moves = migrate.run_virtual_step(ranks, qs, ks, vs, os_, comm_ms=0.0, moves=moves)
    torch.cuda.synchronize()
    assert got_moves == moves and rank_of.tolist() == [2, 0, 1, 0, 2, 2]
    assert all(r.dev_status() == 0 for r in ranks)
    assert torch.equal(torch.cat(os_, dim=2), o_whole)


def test_donor_skips_exactly_its_migrated_heads_tiles():
    import torch
    from adaptive_block_sparse_hilbert_b200 import migrate
    wl, world = CASES[1]
    _, _, ranks, qs, ks, vs, _ = _layers(wl, world)
    r = ranks[0]
    r.prepare(qs[0], ks[0], vs[0])
    r.local_loads()
    wlist = r._worklist
    n_pairs = r.n_pairs
    for li, h in enumerate(r.heads):
        runs = r.slot_ranges([h])
        slots = np.concatenate([np.arange(a, a + n) for a, n in runs])
        heads_left = np.unique(wlist[slots] // n_pairs % r.Hr)
        assert li not in heads_left and len(heads_left) == r.Hr - 1
        assert slots.size == wlist.size - n_pairs * wl.B
        assert len(runs) <= 2 * wl.B  # one head's tiles are consecutive per batch entry
    assert r.slot_ranges([]) == [(0, wlist.size)]
    torch.cuda.synchronize()
