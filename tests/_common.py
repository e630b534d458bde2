"""Shared helpers for the GPU parity tests (CUDA path through the C ABI vs the oracle)."""
from __future__ import annotations

import functools
import math

import numpy as np

from adaptive_block_sparse_hilbert_b200 import synth
import oracle as O

# acceptance tolerances for attention outputs (bf16 inputs / fp32 inputs)
BF16_MAX_ABS = 2e-2
BF16_MEAN_ABS = 2e-3
F32_MAX_ABS = 1e-4


def torch_dev():
    import torch
    return torch


@functools.lru_cache(maxsize=4)
def layer(wid: int, step: int = 0):
    return synth.make_layer(synth.WORKLOADS[wid], step)


def shape_of(wl):
    from adaptive_block_sparse_hilbert_b200 import fva
    return fva.make_shape(wl.B, wl.H, wl.d, wl.T, wl.Hg, wl.Wg, wl.dtype)


def to_device(L):
    """Q, K, V of a Layer as CUDA tensors [B, N, H, d] of the workload dtype."""
    torch = torch_dev()
    out = []
    for vals, bits in ((L.q, L.q_bits), (L.k, L.k_bits), (L.v, L.v_bits)):
        if bits is not None:
            t = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)
        else:
            t = torch.from_numpy(np.ascontiguousarray(vals, dtype=np.float32))
        out.append(t.cuda())
    return out


class GpuRun:
    """Runs the CUDA path step by step and keeps every intermediate (on the device)."""

    def __init__(self, wl, L, p=None, k_floor=None, order=None, need_pool=False, curve=None):
        torch = torch_dev()
        from adaptive_block_sparse_hilbert_b200 import fva, pipeline
        self.fva = fva
        self.wl = wl
        s = shape_of(wl)
        self.shape = s
        kw = {}
        if order is not None:
            kw["order"] = order
        if curve is not None:
            kw["curve"] = curve
        self.layer = pipeline.SparseAttentionLayer(s, wl.p if p is None else p,
                                                   wl.k_floor if k_floor is None else k_floor, **kw)
        self.q, self.k, self.v = to_device(L)
        self.layer.reorder_inputs(self.q, self.k, self.v)
        if need_pool:
            ws = torch.empty(fva.fva_route_workspace_bytes(s, True), dtype=torch.uint8, device="cuda")
            fva.fva_route(s, self.layer.qh, self.layer.kh, None, None, self.layer.p, self.layer.k_floor,
                          self.layer.mask, ws, self.layer.order, self.layer.dev_status)
        else:
            self.layer.route()
        torch.cuda.synchronize()

    def mask_np(self):
        m = self.layer.mask
        rp = m.row_ptr.cpu().numpy().astype(np.int64)
        ci = m.col_idx[: int(rp[-1])].cpu().numpy().astype(np.int64)
        tp = m.tile_ptr.cpu().numpy().astype(np.int64)
        tc = m.tile_col[: int(tp[-1])].cpu().numpy().astype(np.int64)
        return {
            "row_ptr": rp, "col_idx": ci, "head_kept": m.head_kept.cpu().numpy(),
            "tile_ptr": tp, "tile_col": tc, "tile_cost": m.tile_cost.cpu().numpy().astype(np.int64),
            "worklist": m.worklist.cpu().numpy().astype(np.int64),
        }

    def status(self):
        return int(self.layer.dev_status.item())


def hilbert_bhnd(L, perm):
    """Oracle-side reorder of Q, K, V (float64 [B,H,N,d])."""
    return O.reorder(L.q, perm), O.reorder(L.k, perm), O.reorder(L.v, perm)


def oracle_pooled(L, perm):
    """Pooled Q and K [B,H,nB,d] computed head by head (bounded memory)."""
    B, N, H, d = L.q.shape
    nB = O.n_blocks(N)
    pq = np.empty((B, H, nB, d))
    pk = np.empty((B, H, nB, d))
    for h in range(H):
        pq[:, h] = O.block_mean_pool(O.reorder(L.q[:, :, h:h + 1], perm))[:, 0]
        pk[:, h] = O.block_mean_pool(O.reorder(L.k[:, :, h:h + 1], perm))[:, 0]
    return pq, pk


def compare_masks(gpu: dict, orc: dict, nrows: int):
    """Rows where the CSR lists differ, and the oracle's ambiguity flags for them."""
    grp, gci = gpu["row_ptr"], gpu["col_idx"]
    orp, oci = orc["row_ptr"], orc["col_idx"]
    mismatch = []
    for r in range(nrows):
        a = gci[grp[r]:grp[r + 1]]
        b = oci[orp[r]:orp[r + 1]]
        if a.size != b.size or np.any(a != b):
            mismatch.append(r)
    amb = orc["ambiguous_mass"] | orc["ambiguous_tie"]
    return np.array(mismatch, dtype=np.int64), amb


def expected_tiles(row_ptr, col_idx, BH, nB):
    """Union lists with membership bits, per tile (host recomputation from the CSR)."""
    n_pairs = (nB + 1) // 2
    out = []
    for bh in range(BH):
        for t in range(n_pairs):
            a = set(O.row_list(row_ptr, col_idx, bh * nB + 2 * t).tolist())
            b = set(O.row_list(row_ptr, col_idx, bh * nB + 2 * t + 1).tolist()) if 2 * t + 1 < nB else set()
            out.append([(blk << 2) | (blk in a) | ((blk in b) << 1) for blk in sorted(a | b)])
    return out


def expected_worklist(cost: np.ndarray, BH: int, n_pairs: int, order: int) -> np.ndarray:
    ids = np.arange(cost.size)
    if order == 0:
        return ids
    if order == 1:
        return np.lexsort((ids, -cost))
    load = cost.reshape(BH, n_pairs).sum(axis=1)
    heads = np.lexsort((np.arange(BH), -load))
    parts = []
    for bh in heads:
        c = cost[bh * n_pairs:(bh + 1) * n_pairs]
        parts.append(bh * n_pairs + np.lexsort((np.arange(n_pairs), -c)))
    return np.concatenate(parts)


def err_stats(got: np.ndarray, want: np.ndarray):
    diff = np.abs(got.astype(np.float64) - want)
    return float(diff.max()), float(diff.mean())


def sample_rows(row_ptr, BH, nB, n_per_head, seed):
    """Seeded (bh, a) sample per head, always including its densest and sparsest rows."""
    rng = np.random.default_rng(seed)
    cnt = np.diff(row_ptr).reshape(BH, nB)
    rows = []
    for bh in range(BH):
        pick = set(rng.choice(nB, size=min(n_per_head, nB), replace=False).tolist())
        pick.add(int(np.argmax(cnt[bh])))
        pick.add(int(np.argmin(cnt[bh])))
        pick.add(nB - 1)  # the ragged tail block
        rows.extend((bh, a) for a in sorted(pick))
    return rows


def default_scale(d):
    return 1.0 / math.sqrt(d)


def largest_routable_workload():
    """One head at the routing kernel's largest block count: 837 x 866 = 724,842 tokens,
    nB = 11326 (a ragged tail of 42), d = 64. Heads drawn with tau in logU(2, 2.5) give a
    low density with row lengths from a few dozen to thousands of blocks."""
    return synth.custom_workload(1, 837, 866, 1, 64, "bf16", seed=41, tau=("logU", 2.0, 2.5))


def sampled_attention_errors(run, wl, L, g, n_per_head, seed, curve=0):
    """Attend with the run's routed mask `g` (from run.mask_np()) and compare sampled query
    blocks of every head -- seeded ones plus each head's densest, sparsest and ragged tail
    rows -- with the oracle's attention over the same kept blocks. Returns (max-abs error,
    mean-abs error, query blocks compared)."""
    torch = torch_dev()
    run.layer.attend()
    torch.cuda.synchronize()
    assert run.status() == 0
    BH, nB = wl.B * wl.H, wl.nB
    rows = sample_rows(g["row_ptr"], BH, nB, n_per_head, seed=seed)
    perm, _ = (O.rect_curve_perm if curve == 1 else O.hilbert_perm)(wl.T, wl.Hg, wl.Wg)
    max_err, sum_err, n = 0.0, 0.0, 0
    oh = run.layer.oh
    for bh in sorted({bh for bh, _ in rows}):
        b, h = divmod(bh, wl.H)
        qh = O.reorder(L.q[b:b + 1, :, h:h + 1], perm)[0, 0]
        kh = O.reorder(L.k[b:b + 1, :, h:h + 1], perm)[0, 0]
        vh = O.reorder(L.v[b:b + 1, :, h:h + 1], perm)[0, 0]
        for (b2, a) in rows:
            if b2 != bh:
                continue
            keys = O.block_keys(O.row_list(g["row_ptr"], g["col_idx"], bh * nB + a), wl.N)
            lo, hi = a * 64, min(a * 64 + 64, wl.N)
            want = O.attention_rows(qh[lo:hi], kh, vh, keys, 1.0 / np.sqrt(wl.d))
            gv = oh[b, h, lo:hi].float().cpu().numpy().astype(np.float64)
            diff = np.abs(gv - want)
            max_err = max(max_err, float(diff.max()))
            sum_err += float(diff.sum())
            n += diff.size
    return max_err, sum_err / n, len(rows)
