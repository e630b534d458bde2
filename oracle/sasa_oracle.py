"""Float64 CPU oracle for FVAttn's Slack-Aware Sparse Augmentation (SASA).

TEST INFRASTRUCTURE ONLY, like fva_oracle.py: only the tests and bench.py's reference
leg may call it, and it shares no code with the library.

Sources, cited by page and section:

* [aixai] aixai.ru blog post on FVAttn -- section "Slack-Aware Sparse Augmentation
  (SASA)": after balancing, non-critical ranks wait for the critical path; SASA spends
  that slack on additional high-value blocks without lengthening the critical path;
  thresholds k1 = 1.05 and k2 = 1.10 pick the mode (SASA alone for k1 <= imbalance < k2,
  RLB + SASA for imbalance >= k2); the augmentation coefficient n1 = 0.8 and the trigger
  threshold n2 = 0.07 set how much is added. Section "Sparse-routing frontend": the one
  routing pass yields the per-head density (for RLB) and the importance order of key
  blocks (for SASA).
* [PD] longzhangge.com PaperDaily article -- section 方法揭秘: SASA computes each rank's
  idle-time budget and, from the blocks the sparse mask skipped, picks some in order of
  importance, keeping the extra compute within that budget.

Readings where the pages leave a step open:

* The mode is chosen on the imbalance (slowest / fastest rank load) of the starting
  placement; below k1 nothing is added.
* A rank's slack is (critical load - its load), measured after RLB when RLB runs; the
  rank is augmented when slack >= n2 x critical load, with a budget of
  floor(n1 x slack / c) blocks, c the compute time of one block.
* Importance is the routing softmax P_ab of the row; a rank's budget goes to the skipped
  (row, block) entries of its heads with the largest P, ties to the lower head, then the
  lower query block, then the lower key block (equal logits are ordered by block index in
  the routing order too). Within a row, the taken entries then continue the row's routing
  order, so every row keeps a prefix of that order.
"""
from __future__ import annotations

import numpy as np

from . import fva_oracle as F

K1 = 1.05
K2 = 1.10
N1 = 0.8
N2 = 0.07


def mode(rank_load: np.ndarray) -> str:
    """'none' below k1, 'sasa' for k1 <= slowest/fastest < k2, 'rlb+sasa' from k2 on."""
    L = np.asarray(rank_load, dtype=np.float64)
    rho = float(L.max() / L.min()) if L.min() > 0 else float("inf")
    if rho < K1:
        return "none"
    return "sasa" if rho < K2 else "rlb+sasa"


def budgets(rank_load: np.ndarray, block_ms: float, n1: float = N1, n2: float = N2) -> np.ndarray:
    """Blocks each rank may add: floor(n1 * slack / c) where slack >= n2 * critical load."""
    L = np.asarray(rank_load, dtype=np.float64)
    crit = float(L.max())
    out = np.zeros(L.size, dtype=np.int64)
    for r in range(L.size):
        slack = crit - float(L[r])
        if crit > 0.0 and slack >= n2 * crit:
            out[r] = int(np.floor(n1 * slack / block_ms))
    return out


def _row_tables(logits: np.ndarray, kept_len: np.ndarray):
    """Per row: the importance P of every key block (block order) and whether the block is
    outside the kept prefix of the routing order (skipped)."""
    BH, nB, _ = logits.shape
    P = np.empty((BH, nB, nB), dtype=np.float64)
    skipped = np.ones((BH, nB, nB), dtype=bool)
    for h in range(BH):
        for a in range(nB):
            s = logits[h, a]
            P[h, a] = F.importance(s)
            skipped[h, a, F.routing_order(s)[: kept_len[h, a]]] = False
    return P, skipped


def augment(logits: np.ndarray, kept_len: np.ndarray, rank_of_head: np.ndarray, budget: np.ndarray,
            with_threshold: bool = False):
    """New kept lengths per row after SASA.

    logits: float64 [BH, nB, nB] block logits; kept_len: int [BH * nB], the routed prefix
    length L of every row; rank_of_head: int [BH]; budget: int [R] blocks per rank.
    Each rank's skipped entries are ranked by (importance desc, head, query block, key
    block) and the first budget[r] of them are taken; a row's taken blocks continue its
    routing order, so the row keeps a prefix. Returns new_len [BH * nB] (and, with
    with_threshold, the importance of the last entry taken per rank, or None)."""
    logits = np.asarray(logits, dtype=np.float64)
    BH, nB, _ = logits.shape
    L = np.asarray(kept_len, dtype=np.int64).reshape(BH, nB)
    P, skipped = _row_tables(logits, L)
    new_len = L.copy()
    rank_of_head = np.asarray(rank_of_head, dtype=np.int64)
    last_p = [None] * len(budget)
    for r in range(len(budget)):
        if budget[r] <= 0:
            continue
        heads = np.nonzero(rank_of_head == r)[0]
        if heads.size == 0:
            continue
        hh, aa, bb = np.nonzero(skipped[heads])                          # head, row, block order
        pv = P[heads[hh], aa, bb]
        rank_key = np.lexsort((bb, aa, heads[hh], -pv))                  # importance first
        take = rank_key[: int(budget[r])]
        np.add.at(new_len, (heads[hh[take]], aa[take]), 1)
        if take.size:
            last_p[r] = float(pv[take[-1]])
    new_len = new_len.reshape(-1)
    return (new_len, last_p) if with_threshold else new_len


def kept_mass(logits: np.ndarray, kept_len: np.ndarray) -> np.ndarray:
    """Per row, the routing importance the kept prefix holds (sum of P over it)."""
    logits = np.asarray(logits, dtype=np.float64)
    BH, nB, _ = logits.shape
    L = np.asarray(kept_len, dtype=np.int64).reshape(BH, nB)
    out = np.zeros((BH, nB))
    for h in range(BH):
        for a in range(nB):
            s = logits[h, a]
            order = F.routing_order(s)
            out[h, a] = F.importance(s)[order[: L[h, a]]].sum()
    return out.reshape(-1)
