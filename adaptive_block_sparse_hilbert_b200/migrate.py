"""Head-sharded attention with Runtime Load Balancing head migration between GPUs.

Method: aixai.ru FVAttn blog, "Runtime Load Balancing (RLB)" -- under Ulysses sequence
parallelism every rank attends its own heads over the full sequence; per-head load comes
from the routing pass, the most loaded rank hands its heaviest head to the least loaded
one when the move pays (G = K - P - C > 0), at most one local head per rank, and the head's
data travels point to point while the ranks compute. PaperDaily FVAttn article, 方法揭秘 --
the plan runs on the CPU while the GPU computes, moving the heaviest head from the most
to the least loaded rank until the imbalance falls below a threshold.

One step on rank r (heads [r H / R, (r + 1) H / R) of the layer, Q, K, V in raster
[B, N, H_r, d] as the sequence-parallel all-to-all leaves them):
  1. reorder + pool + route its own heads (libfva); per-head load = the head's issued tile
     steps x the measured time per step;
  2. the per-head loads are all-gathered (one small collective);
  3. every rank runs the same planner (fva_rlb_plan) on the same loads, so all ranks hold
     the same moves without further agreement;
  4. each donor sends its migrated head's Hilbert-ordered Q, K, V and pooled Q, K to the
     receiver, which lands them in its own buffers (NCCL send/recv between GPUs; nothing
     reads another GPU's memory in place);
  5. meanwhile every rank attends its remaining heads -- a donor launches the work-list
     slots around its migrated head's tiles (heads are contiguous in the head-grouped
     longest-first list);
  6. a receiver routes and attends each head once it has landed and sends its O back; the
     donor inverse-reorders all its heads once that O has arrived.

The protocol is written once (`run_step` for one rank of a process group, `run_virtual_step`
for R ranks emulated in one process, whose transfers are copies); the per-rank compute is
an object with the methods of `ShardRank` (libfva on a GPU). The bench runs the virtual
form on one GPU, which measures each rank's own compute time; the NCCL form needs one GPU
per rank.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

from . import fva, pipeline


# ------------------------------------------------------------------------------ plan

def heads_of_rank(rank: int, world: int, H: int) -> range:
    """Contiguous head slice of a rank (the planner's starting placement)."""
    return range(rank * H // world, (rank + 1) * H // world)


@dataclasses.dataclass(frozen=True)
class Move:
    head: int       # global head index
    src: int        # donor rank (the head's owner)
    dst: int        # receiver rank
    gain_ms: float  # net gain G of the move


def plan_moves(all_loads_ms: np.ndarray, world: int, comm_ms: float, sched_ms: float,
               threshold: float = 1.10, max_per_rank: int = 1):
    """The RLB plan over the gathered per-head loads (host C planner in libfva); the same
    inputs give the same moves on every rank."""
    rank_of, moves = fva.fva_rlb_plan(np.asarray(all_loads_ms, np.float64), world, comm_ms, sched_ms, threshold,
                                      max_per_rank)
    return rank_of, [Move(int(h), int(a), int(b), float(g)) for h, a, b, g in moves]


def transfers(moves, rank: int, what: str):
    """The point-to-point transfers of `rank` for one direction of the moves, in the order
    both ends issue them: what="inputs" (donor -> receiver) or "outputs" (receiver ->
    donor). Returns (sends, recvs) as lists of (peer, move)."""
    sends, recvs = [], []
    for m in moves:
        a, b = (m.src, m.dst) if what == "inputs" else (m.dst, m.src)
        if a == rank:
            sends.append((b, m))
        if b == rank:
            recvs.append((a, m))
    return sends, recvs


# ------------------------------------------------------------------------------ exchanges

class _Done:
    def wait(self):
        pass


class _Works:
    def __init__(self, works):
        self.works = works

    def wait(self):
        for w in self.works:
            w.wait()


class DistExchange:
    """The step's communication over a torch.distributed group: NCCL between GPUs (tensors
    on the device), gloo on CPU. All ranks take the same collective steps in the same
    order; the P2P transfers of a step come after the all-gather, so a batch may involve a
    subset of the ranks."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)

    def all_gather_loads(self, local_ms: np.ndarray, H: int, device) -> np.ndarray:
        """Every rank's per-head loads, in global head order (slices padded to one size)."""
        width = -(-H // self.world)
        t = torch.full((width,), -1.0, dtype=torch.float64, device=device)
        t[: local_ms.size] = torch.as_tensor(local_ms, dtype=torch.float64)
        out = [torch.empty_like(t) for _ in range(self.world)]
        self.dist.all_gather(out, t, group=self.group)
        full = torch.cat(out).cpu().numpy().reshape(self.world, width)
        return np.concatenate([full[r, : len(heads_of_rank(r, self.world, H))] for r in range(self.world)])

    def transfer(self, sends, recvs):
        """sends / recvs: lists of (peer, tensor) in issue order; returns a handle whose
        wait() orders the caller's stream (or host, for gloo) after the transfers."""
        d = self.dist
        ops = [d.P2POp(d.isend, t, peer, self.group) for peer, t in sends]
        ops += [d.P2POp(d.irecv, t, peer, self.group) for peer, t in recvs]
        if not ops:
            return _Done()
        return _Works(d.batch_isend_irecv(ops))


# ------------------------------------------------------------------------------ protocol

def _flatten(pairs, tensors_of):
    return [(peer, t) for peer, m in pairs for t in tensors_of(m)]


def run_step(rank_obj, exchange: DistExchange, q, k, v, o, comm_ms: float, sched_ms: float = 0.1,
             threshold: float = 1.10, migrate: bool = True, timer=None):
    """One step of one rank of a process group. q, k, v, o: this rank's raster [B, N, H_r, d]
    slices. comm_ms (P: moving one head) and sched_ms (C: the planner's time) enter the plan,
    so they must be the same on every rank -- constants, not per-rank measurements.
    migrate=False keeps every head at home (the same collective steps are still taken);
    `timer`, if given, is called as timer(phase, fn) around the rank's compute phases.
    Returns (rank_of, moves); o holds the rank's output when the call returns (its stream
    ordered after everything the step enqueued)."""
    H, R, r = rank_obj.H, exchange.world, exchange.rank
    run = timer if timer is not None else (lambda phase, fn: fn())
    run("prepare", lambda: rank_obj.prepare(q, k, v))
    loads = exchange.all_gather_loads(rank_obj.local_loads(), H, rank_obj.device)
    if migrate:
        rank_of, moves = plan_moves(loads, R, comm_ms, sched_ms, threshold)
    else:
        rank_of, moves = np.array([x for x in range(R) for _ in heads_of_rank(x, R, H)], np.int32), []
    s_in, r_in = transfers(moves, r, "inputs")
    h_in = exchange.transfer(_flatten(s_in, rank_obj.input_tensors), _flatten(r_in, rank_obj.input_buffers))
    run("attend", lambda: rank_obj.attend_own(skip=[m.head for _, m in s_in]))
    h_in.wait()
    run("attend_received", lambda: rank_obj.attend_received([m.head for _, m in r_in]))
    s_out, r_out = transfers(moves, r, "outputs")
    h_out = exchange.transfer(_flatten(s_out, rank_obj.output_tensors), _flatten(r_out, rank_obj.output_buffers))
    h_out.wait()
    run("finish", lambda: rank_obj.finish(o))
    return rank_of, moves


def run_virtual_step(ranks, qs, ks, vs, os_, comm_ms: float, sched_ms: float = 0.0, threshold: float = 1.10,
                     migrate: bool = True, timer=None, moves=None):
    """The same step for R ranks emulated in one process (one device): the phases run rank
    after rank and the transfers are copies into the receivers' own buffers. `timer`, if
    given, is called as timer(phase, rank, fn) around each rank's compute phase (the bench
    times them with CUDA events). migrate=False keeps every head at home; `moves` replaces
    the planner's moves by given ones (each from the head's owner, at most one per donor)."""
    R = len(ranks)
    H = ranks[0].H
    run = timer if timer is not None else (lambda phase, r, fn: fn())
    for r, obj in enumerate(ranks):
        run("prepare", r, lambda: obj.prepare(qs[r], ks[r], vs[r]))
    loads = np.concatenate([obj.local_loads() for obj in ranks])
    home = np.array([r for r in range(R) for _ in heads_of_rank(r, R, H)], np.int32)
    if moves is not None:
        moves = list(moves)
        if any(home[m.head] != m.src for m in moves) or len({m.src for m in moves}) != len(moves):
            raise ValueError("each move must start at the head's owner, one move per donor")
        rank_of = home.copy()
        for m in moves:
            rank_of[m.head] = m.dst
    elif migrate:
        rank_of, moves = plan_moves(loads, R, comm_ms, sched_ms, threshold)
    else:
        rank_of, moves = home, []

    def copy_phase(what, tensors_of, buffers_of):
        for r, obj in enumerate(ranks):
            _, recvs = transfers(moves, r, what)
            for peer, m in recvs:
                for dst, src in zip(buffers_of(obj, m), tensors_of(ranks[peer], m)):
                    dst.copy_(src)

    copy_phase("inputs", lambda o, m: o.input_tensors(m), lambda o, m: o.input_buffers(m))
    for r, obj in enumerate(ranks):
        skip = [m.head for m in moves if m.src == r]
        got = [m.head for m in moves if m.dst == r]
        run("attend", r, lambda: (obj.attend_own(skip=skip), obj.attend_received(got)))
    copy_phase("outputs", lambda o, m: o.output_tensors(m), lambda o, m: o.output_buffers(m))
    for r, obj in enumerate(ranks):
        run("finish", r, lambda: obj.finish(os_[r]))
    return loads, rank_of, moves


# ------------------------------------------------------------------------------ GPU rank

class ShardRank:
    """One rank's heads of a layer on a GPU, with buffers for the heads it may receive.

    shape: the whole layer (all H heads); this rank owns heads_of_rank(rank, world, H).
    ms_per_step: time of one issued tile step (64 keys x 128 query rows) on this GPU; the
    per-head load the planner sees is the head's issued steps times it."""

    def __init__(self, shape: fva.fva_shape, p: float, k_floor: int, rank: int, world: int, ms_per_step: float,
                 device="cuda", stream=None):
        s = shape
        self.full = s
        self.H = s.H
        self.rank, self.world = rank, world
        self.heads = heads_of_rank(rank, world, s.H)
        self.Hr = len(self.heads)
        self.p, self.k_floor = float(p), int(k_floor)
        self.ms_per_step = float(ms_per_step)
        self.device = torch.device(device)
        self.stream = stream
        self.shape = fva.make_shape(s.B, self.Hr, s.d, s.T, s.Hg, s.Wg, s.dtype)
        self.layer = pipeline.SparseAttentionLayer(self.shape, p, k_floor, fva.FVA_ORDER_HEAD_LPT, device)
        self.n_pairs = (self.layer.nB + 1) // 2
        self.one = fva.make_shape(s.B, 1, s.d, s.T, s.Hg, s.Wg, s.dtype)
        self.guests = {}      # global head -> 1-head layer holding a received head
        self._worklist = None

    # -- phase 1
    def prepare(self, q, k, v):
        self.layer.reorder_inputs(q, k, v, self.stream)
        self.layer.route(self.stream)

    def local_loads(self) -> np.ndarray:
        """Per-head load (ms) of the own heads; reads the tile costs and the work list back."""
        m = self.layer.mask
        cost = m.tile_cost.cpu().numpy().astype(np.int64)
        self._worklist = m.worklist.cpu().numpy().astype(np.int64)
        steps = cost.reshape(self.shape.B, self.Hr, self.n_pairs).sum(axis=(0, 2))
        return steps.astype(np.float64) * self.ms_per_step

    # -- transfers: tensors are contiguous [N, d] / [nB, d] slices, one per batch entry
    def _local(self, head: int) -> int:
        return head - self.heads.start

    def input_tensors(self, m: Move):
        li, L = self._local(m.head), self.layer
        return [x[b, li] for b in range(self.shape.B) for x in (L.qh, L.kh, L.vh, L.pooled_q, L.pooled_k)]

    def _guest(self, head: int):
        g = self.guests.get(head)
        if g is None:
            g = pipeline.SparseAttentionLayer(self.one, self.p, self.k_floor, fva.FVA_ORDER_HEAD_LPT, self.device)
            self.guests[head] = g
        return g

    def input_buffers(self, m: Move):
        g = self._guest(m.head)
        return [x[b, 0] for b in range(self.shape.B) for x in (g.qh, g.kh, g.vh, g.pooled_q, g.pooled_k)]

    def output_tensors(self, m: Move):
        g = self.guests[m.head]
        return [g.oh[b, 0] for b in range(self.shape.B)]

    def output_buffers(self, m: Move):
        li = self._local(m.head)
        return [self.layer.oh[b, li] for b in range(self.shape.B)]

    # -- phase 2
    def slot_ranges(self, skip) -> list:
        """Maximal runs of work-list slots whose tiles belong to heads not in `skip`."""
        if not skip:
            return [(0, int(self._worklist.size))]
        bh = self._worklist // self.n_pairs
        keep = ~np.isin(bh % self.Hr, [self._local(h) for h in skip])
        runs, start = [], None
        for i, k in enumerate(keep):
            if k and start is None:
                start = i
            elif not k and start is not None:
                runs.append((start, i - start))
                start = None
        if start is not None:
            runs.append((start, int(keep.size) - start))
        return runs

    def attend_own(self, skip=()):
        L = self.layer
        for first, n in self.slot_ranges(list(skip)):
            fva.fva_sparse_attn_range(self.shape, L.qh, L.kh, L.vh, L.mask, L.oh, first, n, 0.0, L.dev_status,
                                      self.stream)

    def attend_received(self, heads=()):
        for h in heads:
            g = self.guests[h]
            g.route(self.stream)
            g.attend(self.stream)

    # -- phase 3
    def finish(self, o):
        self.layer.restore_output(o, self.stream)

    def dev_status(self) -> int:
        return max([int(self.layer.dev_status.item())] + [int(g.dev_status.item()) for g in self.guests.values()])
