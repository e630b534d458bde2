"""Float64 CPU oracle for FVAttn's Runtime Load Balancing (RLB) planner.

TEST INFRASTRUCTURE ONLY, like fva_oracle.py: only the tests and the reference leg of
bench.py may call it, and it shares no code with the library's planner.

Sources, cited by page and section:

* [aixai] aixai.ru blog post on FVAttn -- section "Runtime Load Balancing (RLB)": the
  planner runs on the materialised mask; the critical-path benefit of a plan is
  K = c * (max_r L_r - max_r L_r_new) with c the compute time of one sparse block; the
  cost is the communication overhead P of moving head state plus the scheduling
  overhead C; the net gain is G = K - P - C; each rank migrates at most one local head
  (20% of the local heads in the 8-GPU setting), which takes the average imbalance from
  1.34 to 1.08. Section "Slack-Aware Sparse Augmentation": the regime thresholds
  k1 = 1.05 and k2 = 1.10 (RLB + SASA when the imbalance is >= k2).
* [PD] longzhangge.com PaperDaily article -- section 方法揭秘 (method): compute each
  rank's total load, find the most and the least loaded rank, move the heaviest head of
  the most loaded rank to the least loaded one, and repeat until the imbalance factor is
  below a threshold or the migration budget is used up; the imbalance factor is the
  slowest rank's compute time over the fastest rank's.

Readings where the pages leave a step open:

* Heads start in the contiguous Ulysses split: rank r owns heads [r H / R, (r+1) H / R).
* The imbalance factor that stops the planner is max/min (the [PD] definition); the stop
  threshold defaults to k2 = 1.10, the boundary of the RLB regime.
* A move takes the heaviest of the most loaded rank's own (never received) heads whose
  move has positive net gain G; if the heaviest one's move does not pay (it would make
  the receiving rank the new maximum), the next heaviest is tried. No positive-gain move
  from the most loaded rank ends the plan, as does its export budget.
* Ties: the lowest rank index is the most / least loaded; equal head loads go to the
  lower head index.
* Loads are in milliseconds (blocks times c); K is in milliseconds too.
"""
from __future__ import annotations

import numpy as np

K1 = 1.05
K2 = 1.10


def contiguous_split(H: int, R: int) -> np.ndarray:
    """rank_of[h] for the Ulysses head split: rank r owns heads [r H // R, (r+1) H // R)."""
    rank_of = np.empty(H, dtype=np.int64)
    for r in range(R):
        rank_of[(r * H) // R:((r + 1) * H) // R] = r
    return rank_of


def rank_loads(head_load: np.ndarray, rank_of: np.ndarray, R: int) -> np.ndarray:
    """L_r = sum of the loads of the heads on rank r, added in head order."""
    L = np.zeros(R, dtype=np.float64)
    for h in range(len(head_load)):
        L[rank_of[h]] += float(head_load[h])
    return L


def imbalance(L: np.ndarray) -> tuple[float, float]:
    """(max / mean, max / min) of the rank loads ([PD] defines the factor as max / min)."""
    mx, mn, mean = float(L.max()), float(L.min()), float(L.mean())
    return (mx / mean if mean > 0 else 1.0), (mx / mn if mn > 0 else float("inf"))


def rlb_plan(head_load: np.ndarray, R: int, comm_ms: float, sched_ms: float, threshold: float = K2,
             max_per_rank: int = 1):
    """The RLB planner: returns (rank_of, moves), moves = [(head, from, to, gain_ms)] in
    the order they are applied. head_load: per-head compute time in ms (blocks * c)."""
    head_load = np.asarray(head_load, dtype=np.float64)
    H = len(head_load)
    home = contiguous_split(H, R)
    rank_of = home.copy()
    exported = np.zeros(R, dtype=np.int64)
    moves = []
    while True:
        L = rank_loads(head_load, rank_of, R)
        if imbalance(L)[1] < threshold:
            break
        r_max = int(np.argmax(L))  # first maximum: lowest rank index
        r_min = int(np.argmin(L))
        if r_max == r_min or exported[r_max] >= max_per_rank:
            break
        # the most loaded rank's own heads, heaviest first (ties: lower head index)
        own = [h for h in range(H) if rank_of[h] == r_max and home[h] == r_max]
        own.sort(key=lambda h: (-head_load[h], h))
        chosen = None
        for h in own:
            trial = rank_of.copy()
            trial[h] = r_min
            L_new = rank_loads(head_load, trial, R)
            gain = (float(L.max()) - float(L_new.max())) - comm_ms - sched_ms
            if gain > 0.0:
                chosen = (h, gain)
                break
        if chosen is None:
            break
        h, gain = chosen
        rank_of[h] = r_min
        exported[r_max] += 1
        moves.append((h, r_max, r_min, gain))
    return rank_of, moves
