"""Head-sharded step with RLB head migration (adaptive_block_sparse_hilbert_b200.migrate)
on the CPU: the protocol (gathered loads, one plan on every rank, inputs to the receiver,
outputs back to the donor) run by ranks whose compute is the float64 oracle.

  * R ranks emulated in one process (run_virtual_step);
  * 3 real processes over gloo (run_step with DistExchange), one of them a bystander.

Either way every rank's output must equal the unsharded oracle attention of its heads
exactly (the migrated head is routed and attended from the same values on the receiver),
and the moves must be the planner's on the gathered loads.
"""
import os
import socket

import numpy as np
import pytest
import torch

import oracle as O
from adaptive_block_sparse_hilbert_b200 import migrate, synth

# 6 heads over 3 ranks, tau drawn from logU(0.3, 8): with this seed heads 0, 1 and 3 are
# flat (about 250 issued tile steps each) and 2, 4, 5 concentrated (about 30), so ranks 0
# and 2 start far apart and the planner moves a head each way
WL = synth.custom_workload(4, 16, 24, 6, 64, "f32", seed=94, tau=("logU", 0.3, 8.0), p=0.9, k_floor=1)
MS_PER_STEP = 1e-3


class OracleRank:
    """The compute of one rank done by the oracle (float64, CPU tensors)."""

    def __init__(self, wl, rank, world, device="cpu"):
        self.wl, self.H, self.rank, self.world = wl, wl.H, rank, world
        self.heads = migrate.heads_of_rank(rank, world, wl.H)
        self.Hr = len(self.heads)
        self.device = torch.device(device)
        self.perm, _ = O.hilbert_perm(wl.T, wl.Hg, wl.Wg)
        self.guests = {}

    def _route(self, pq, pk):
        return O.route(pq, pk, self.wl.d, self.wl.p, self.wl.k_floor)

    def prepare(self, q, k, v):
        self.qh = torch.from_numpy(O.reorder(q.numpy(), self.perm))
        self.kh = torch.from_numpy(O.reorder(k.numpy(), self.perm))
        self.vh = torch.from_numpy(O.reorder(v.numpy(), self.perm))
        self.pq = torch.from_numpy(O.block_mean_pool(self.qh.numpy()))
        self.pk = torch.from_numpy(O.block_mean_pool(self.kh.numpy()))
        self.R = self._route(self.pq.numpy(), self.pk.numpy())
        self.oh = torch.zeros_like(self.qh)

    def local_loads(self):
        nB = self.wl.nB
        cost = O.tile_costs(self.R["row_ptr"], self.R["col_idx"], self.wl.B * self.Hr, nB)
        steps = cost.reshape(self.wl.B, self.Hr, -1).sum(axis=(0, 2))
        return steps.astype(np.float64) * MS_PER_STEP

    def _li(self, h):
        return h - self.heads.start

    def input_tensors(self, m):
        li = self._li(m.head)
        return [x[b, li].contiguous() for b in range(self.wl.B) for x in (self.qh, self.kh, self.vh, self.pq, self.pk)]

    def input_buffers(self, m):
        g = self.guests.setdefault(m.head, {})
        N, nB, d = self.wl.N, self.wl.nB, self.wl.d
        bufs = []
        for b in range(self.wl.B):
            for name, rows in (("q", N), ("k", N), ("v", N), ("pq", nB), ("pk", nB)):
                g[(name, b)] = torch.zeros((rows, d), dtype=torch.float64)
                bufs.append(g[(name, b)])
        return bufs

    def output_tensors(self, m):
        g = self.guests[m.head]
        return [g[("o", b)] for b in range(self.wl.B)]

    def output_buffers(self, m):
        li = self._li(m.head)
        return [self.oh[b, li] for b in range(self.wl.B)]

    def _attend_head(self, q, k, v, rp, ci, row0):
        B, N, d = 1, self.wl.N, self.wl.d
        out = O.block_sparse_attention(q[None, None], k[None, None], v[None, None],
                                       rp[row0:row0 + self.wl.nB + 1] - rp[row0], ci[rp[row0]:], rows=None)
        return torch.from_numpy(O.assemble(out, B, 1, N, d)[0, 0])

    def attend_own(self, skip=()):
        nB = self.wl.nB
        rp, ci = self.R["row_ptr"], self.R["col_idx"]
        for b in range(self.wl.B):
            for li, h in enumerate(self.heads):
                if h in skip:
                    continue
                row0 = (b * self.Hr + li) * nB
                self.oh[b, li] = self._attend_head(self.qh[b, li].numpy(), self.kh[b, li].numpy(),
                                                   self.vh[b, li].numpy(), rp, ci, row0)

    def attend_received(self, heads=()):
        for h in heads:
            g = self.guests[h]
            for b in range(self.wl.B):
                R = self._route(g[("pq", b)].numpy()[None, None], g[("pk", b)].numpy()[None, None])
                g[("o", b)] = self._attend_head(g[("q", b)].numpy(), g[("k", b)].numpy(), g[("v", b)].numpy(),
                                                R["row_ptr"], R["col_idx"], 0)

    def finish(self, o):
        o.copy_(torch.from_numpy(O.inverse_reorder(self.oh.numpy(), self.perm)))


def _expected_all_heads(wl, L):
    """The unsharded oracle output of the whole layer, raster [B, N, H, d]."""
    perm, _ = O.hilbert_perm(wl.T, wl.Hg, wl.Wg)
    qh, kh, vh = O.reorder(L.q, perm), O.reorder(L.k, perm), O.reorder(L.v, perm)
    R = O.route(O.block_mean_pool(qh), O.block_mean_pool(kh), wl.d, wl.p, wl.k_floor)
    oh = O.assemble(O.block_sparse_attention(qh, kh, vh, R["row_ptr"], R["col_idx"]), wl.B, wl.H, wl.N, wl.d)
    return O.inverse_reorder(oh, perm), R


def _slices(L, world):
    out = []
    for r in range(world):
        hs = migrate.heads_of_rank(r, world, L.q.shape[2])
        out.append(tuple(torch.from_numpy(np.ascontiguousarray(x[:, :, hs.start:hs.stop], np.float64))
                         for x in (L.q, L.k, L.v)))
    return out


def test_virtual_ranks_migrate_and_match_the_unsharded_layer():
    L = synth.make_layer(WL)
    want, R_all = _expected_all_heads(WL, L)
    world = 3
    ranks = [OracleRank(WL, r, world) for r in range(world)]
    parts = _slices(L, world)
    outs = [torch.zeros_like(p[0]) for p in parts]
    loads, rank_of, moves = migrate.run_virtual_step(ranks, [p[0] for p in parts], [p[1] for p in parts],
                                                     [p[2] for p in parts], outs, comm_ms=0.0)
    # the gathered loads are the heads' issued tile steps; the plan is the planner's on them
    cost = O.tile_costs(R_all["row_ptr"], R_all["col_idx"], WL.H, WL.nB).reshape(WL.H, -1).sum(axis=1)
    np.testing.assert_allclose(loads, cost * MS_PER_STEP)
    r2, m2 = migrate.plan_moves(loads, world, 0.0, 0.0)
    assert moves == m2 and np.array_equal(rank_of, r2)
    assert moves, "the flat and concentrated heads should give the planner a paying move"
    assert len({m.src for m in moves}) == len(moves)  # at most one exported head per rank
    for r in range(world):
        hs = migrate.heads_of_rank(r, world, WL.H)
        np.testing.assert_array_equal(outs[r].numpy(), want[:, :, hs.start:hs.stop])
    # without migration the outputs are the same (every head computed at home)
    outs2 = [torch.zeros_like(p[0]) for p in parts]
    migrate.run_virtual_step([OracleRank(WL, r, world) for r in range(world)], [p[0] for p in parts],
                             [p[1] for p in parts], [p[2] for p in parts], outs2, comm_ms=0.0, migrate=False)
    for a, b in zip(outs, outs2):
        np.testing.assert_array_equal(a.numpy(), b.numpy())


def test_transfers_pair_up_in_issue_order():
    moves = [migrate.Move(4, 2, 0, 1.0), migrate.Move(1, 0, 1, 0.5), migrate.Move(5, 1, 0, 0.2)]
    s0, r0 = migrate.transfers(moves, 0, "inputs")
    assert [(p, m.head) for p, m in s0] == [(1, 1)]
    assert [(p, m.head) for p, m in r0] == [(2, 4), (1, 5)]
    s0, r0 = migrate.transfers(moves, 0, "outputs")
    assert [(p, m.head) for p, m in s0] == [(2, 4), (1, 5)]
    assert [(p, m.head) for p, m in r0] == [(1, 1)]
    # every send has exactly one matching receive at its peer, in the same order
    for what in ("inputs", "outputs"):
        for a in range(3):
            for b in range(3):
                sa = [m for p, m in migrate.transfers(moves, a, what)[0] if p == b]
                rb = [m for p, m in migrate.transfers(moves, b, what)[1] if p == a]
                assert sa == rb


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _gloo_rank(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        L = synth.make_layer(WL)
        q, k, v = _slices(L, world)[rank]
        o = torch.zeros_like(q)
        obj = OracleRank(WL, rank, world)
        phases = []
        rank_of, moves = migrate.run_step(obj, migrate.DistExchange(), q, k, v, o, comm_ms=0.0, sched_ms=0.0,
                                          timer=lambda phase, fn: (phases.append(phase), fn()))
        dist.barrier()
        # the same step with every head kept at home: same collective steps, same output
        o2 = torch.zeros_like(q)
        _, moves2 = migrate.run_step(OracleRank(WL, rank, world), migrate.DistExchange(), q, k, v, o2, comm_ms=0.0,
                                     sched_ms=0.0, migrate=False)
        dist.barrier()
        out[rank] = (o.numpy().copy(), [(m.head, m.src, m.dst) for m in moves], rank_of.tolist(), phases,
                     bool(torch.equal(o, o2)), len(moves2))
    finally:
        dist.destroy_process_group()


def test_gloo_ranks_migrate_and_match_the_unsharded_layer():
    import torch.multiprocessing as mp
    world = 3
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_gloo_rank, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
        res = dict(out)
    L = synth.make_layer(WL)
    want, _ = _expected_all_heads(WL, L)
    plans = {tuple(map(tuple, res[r][1])) for r in range(world)}
    assert len(plans) == 1, "every rank must hold the same moves"
    moves = res[0][1]
    assert moves
    for r in range(world):
        hs = migrate.heads_of_rank(r, world, WL.H)
        np.testing.assert_array_equal(res[r][0], want[:, :, hs.start:hs.stop])
        assert res[r][3] == ["prepare", "attend", "attend_received", "finish"]
        assert res[r][4] and res[r][5] == 0  # without migration: no moves, the same output
    # the same plan as the in-process emulation
    ranks = [OracleRank(WL, r, world) for r in range(world)]
    parts = _slices(L, world)
    outs = [torch.zeros_like(p[0]) for p in parts]
    _, _, vmoves = migrate.run_virtual_step(ranks, [p[0] for p in parts], [p[1] for p in parts],
                                            [p[2] for p in parts], outs, comm_ms=0.0)
    assert [(m.head, m.src, m.dst) for m in vmoves] == [tuple(x) for x in moves]


class _DyingDonor(OracleRank):
    """A rank that fails on the host after the plan, before it sends its migrated head."""

    def input_tensors(self, m):
        raise RuntimeError("donor failed before sending")


def _gloo_failing_rank(rank, world, port, out):
    import datetime
    import time
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=3))
    L = synth.make_layer(WL)
    q, k, v = _slices(L, world)[rank]
    o = torch.zeros_like(q)
    obj = (_DyingDonor if rank == 0 else OracleRank)(WL, rank, world)
    t0 = time.time()
    try:
        migrate.run_step(obj, migrate.DistExchange(), q, k, v, o, comm_ms=0.0, sched_ms=0.0)
        out[rank] = ("finished", time.time() - t0, "")
    except Exception as e:  # noqa: BLE001 -- the outcome is what the test checks
        out[rank] = (type(e).__name__, time.time() - t0, str(e)[:200])
    if rank == 0:
        time.sleep(6.0)  # the failed rank stays up but silent, so the others' waits must time out
    # no barrier or destroy: rank 0 is gone as far as the others are concerned


def test_gloo_rank_failing_mid_step_ends_the_receivers_wait():
    """A donor that fails after the plan never sends its head and stays silent; the
    receiver's wait for it ends with the process group's timeout (3 s here) as an error, not
    a hang, and a rank with no transfer finishes its own heads."""
    import torch.multiprocessing as mp
    world = 3
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_gloo_failing_rank, args=(world, port, out), nprocs=world, start_method="spawn",
                           join=True)
        res = dict(out)
    # the plan of this layer moves head 0 from rank 0 to rank 2 and head 4 from rank 2 to 0
    assert res[0][0] == "RuntimeError" and "donor failed" in res[0][2]
    assert res[2][0] == "RuntimeError" and 2.5 < res[2][1] < 30.0, res[2]
    assert "Timed out" in res[2][2], res[2]
    assert res[1][0] == "finished", res[1]
