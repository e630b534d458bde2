"""Float64 CPU oracle for the FVAttn sparse-routing frontend and block-sparse attention.

TEST INFRASTRUCTURE ONLY. Nothing in the library imports this module; only the tests,
``__graft_entry__.smoke()`` and the CPU-baseline / reference legs of ``bench.py`` call
it. It shares no code with the CUDA path (no common helpers, tables or constants) and
takes plain numpy arrays. Everything is computed in float64 in the order the pages
state the method, with no blocking or fusion beyond that.

Sources (the five pages about FVAttn, arXiv 2607.16190), cited by page and section:

* [aixai]  aixai.ru blog post on FVAttn -- sections "Top-p vs Top-k", "Sparse-routing
  frontend", "Runtime Load Balancing (RLB)".
* [PD]     longzhangge.com PaperDaily article "腾讯+中山大学新方法：视频生成提速2.11倍" --
  sections 方法揭秘 (method) and 龙迷三问 (Q&A).
* [wiki]   "FVAttn: Adaptive Sparse Attention with Runtime Load Balancing" (AI research
  wiki) -- "What it is".
* [abs]    "FVAttn: Adaptive Sparse Attention with Runtime Load Balancing for Video
  Generation" (mlsanity.com) -- arXiv abstract.

Readings taken where the pages leave a step open:

* Hilbert order: per frame, the 2-D curve over (y, x) on the enclosing 2^m square,
  out-of-grid cells skipped, frames concatenated in t order.
* Pooling: arithmetic mean over the valid tokens of a 64-token block.
* Block importance: softmax over key blocks of (pooled q_a . pooled k_b) / sqrt(d).
* Order: logit descending, ties to the lower block index.
* Top-p cut: the minimal prefix whose cumulative importance is >= p; p >= 1 keeps all.
* Top-k floor: the first min(k_floor, nB) blocks of the same order; the kept set is the
  union, i.e. the longer of the two prefixes.
* Attention: softmax over the valid keys of the kept blocks only, no causal mask. A row
  that keeps no block (only a caller-made mask can have one) outputs zeros.

Parity pins: every function here is pinned in tests/test_oracle_*.py against
something other than itself (an independent L-system construction of the Hilbert
curve, closed forms, brute-force subset enumeration, and torch's float64
scaled_dot_product_attention). See the per-function docstrings.
"""
from __future__ import annotations

import math

import numpy as np

BLOCK = 64

# --------------------------------------------------------------------------------------
# Step 1: Hilbert-curve token order ("video-aware block organization")
# [aixai] "Sparse-routing frontend": blocks are reordered along a Hilbert curve so that
# spatially close tokens land in neighbouring blocks at several scales.
# [PD] 方法揭秘: Hilbert curve organises the blocks so adjacent tokens share blocks.
# --------------------------------------------------------------------------------------


def hilbert_curve(m: int) -> np.ndarray:
    """Cells of the 2^m x 2^m square in Hilbert visiting order, as an int array [4^m, 2] of (x, y).

    Recursive quadrant construction: the order-m curve is four copies of the
    order-(m-1) curve, visiting the quadrants lower-left, upper-left, upper-right,
    lower-right (y grows "up"). The lower-left copy is reflected about the main
    diagonal, the lower-right copy about the anti-diagonal, the two upper copies are
    only translated. The order-1 curve is (0,0) -> (0,1) -> (1,1) -> (1,0).
    """
    if m < 0:
        raise ValueError("m must be >= 0")
    curve = [(0, 0)]
    for level in range(1, m + 1):
        h = 1 << (level - 1)
        ll = [(y, x) for (x, y) in curve]                          # reflect about y = x
        ul = [(x, y + h) for (x, y) in curve]                      # translate up
        ur = [(x + h, y + h) for (x, y) in curve]                  # translate up-right
        lr = [(h - 1 - y + h, h - 1 - x) for (x, y) in curve]      # reflect about anti-diagonal, shift right
        curve = ll + ul + ur + lr
    return np.array(curve, dtype=np.int64).reshape(-1, 2)


def hilbert_order_m(Hg: int, Wg: int) -> int:
    """Smallest m with 2^m >= max(Hg, Wg)."""
    side = max(Hg, Wg)
    m = 0
    while (1 << m) < side:
        m += 1
    return m


def hilbert_perm(T: int, Hg: int, Wg: int):
    """perm[i] = raster index of the token placed at Hilbert position i; inv = perm^-1.

    Raster index n = t*Hg*Wg + y*Wg + x. Within a frame, cells are visited in the
    order of ``hilbert_curve`` on the enclosing 2^m square, skipping cells with
    x >= Wg or y >= Hg; frames follow one another in t order.
    """
    curve = hilbert_curve(hilbert_order_m(Hg, Wg))
    frame = [y * Wg + x for (x, y) in curve if x < Wg and y < Hg]
    assert len(frame) == Hg * Wg
    frame = np.array(frame, dtype=np.int64)
    hw = Hg * Wg
    perm = np.concatenate([t * hw + frame for t in range(T)]) if T > 0 else np.zeros(0, np.int64)
    inv = np.empty_like(perm)
    inv[perm] = np.arange(perm.size, dtype=np.int64)
    return perm, inv


def hilbert_index(m: int, x, y) -> np.ndarray:
    """Distance along the 2^m x 2^m Hilbert curve of each cell (x, y), int64.

    A second construction of the curve above, read digit by digit from the top: at the
    level of half-side s the cell lies in one of four quadrants, visited in the order
    lower-left, upper-left, upper-right, lower-right, so it is preceded by
    (quadrant number) * s^2 cells; the coordinates are then mapped into that quadrant's
    own frame (lower-left: swap axes; lower-right: reflect about the anti-diagonal; the
    upper quadrants keep their orientation) and the next level reads the next bit.
    Works on frames far too large to enumerate (m up to 16)."""
    x = np.asarray(x, dtype=np.int64).copy()
    y = np.asarray(y, dtype=np.int64).copy()
    d = np.zeros(np.broadcast(x, y).shape, dtype=np.int64)
    for level in range(m - 1, -1, -1):
        s = 1 << level
        right = (x >> level) & 1
        up = (y >> level) & 1
        quadrant = np.where(right == 0, up, 3 - up)        # LL 0, UL 1, UR 2, LR 3
        d += quadrant * s * s
        low_x, low_y = x & (s - 1), y & (s - 1)
        ll = quadrant == 0
        lr = quadrant == 3
        x = np.where(ll, low_y, np.where(lr, s - 1 - low_y, low_x))
        y = np.where(ll, low_x, np.where(lr, s - 1 - low_x, low_y))
    return d


def hilbert_perm_by_index(T: int, Hg: int, Wg: int):
    """hilbert_perm's order built the other way round: the frame's cells sorted by
    hilbert_index on the enclosing square (no enumeration of the square's other cells)."""
    m = hilbert_order_m(Hg, Wg)
    yy, xx = np.divmod(np.arange(Hg * Wg, dtype=np.int64), Wg)
    frame = (yy * Wg + xx)[np.argsort(hilbert_index(m, xx, yy), kind="stable")]
    hw = Hg * Wg
    perm = np.concatenate([t * hw + frame for t in range(T)]) if T > 0 else np.zeros(0, np.int64)
    inv = np.empty_like(perm)
    inv[perm] = np.arange(perm.size, dtype=np.int64)
    return perm, inv


# Variant of step 1 (a next step of the build, not the pages' own): a generalized
# Hilbert curve that covers a W x H rectangle directly instead of the enclosing 2^m
# square, following Jakub Cerveny's published generalized-Hilbert ("gilbert")
# construction: a rectangle is split along its longer side into two halves, or across
# it into three parts whose middle part runs the other way, with half lengths rounded to
# even so that the pieces join by unit steps. On 2^m squares it is the curve above.


def rect_hilbert_curve(W: int, H: int) -> np.ndarray:
    """Cells of the W x H rectangle in generalized-Hilbert visiting order, int [W*H, 2] of (x, y).

    A region is given by its first cell (x, y), a major vector a (along which the curve
    leaves the region) and a minor vector b, both axis-parallel. A region one cell thick
    is walked straight. A region at least 1.5 times longer than thick is cut across a into
    two regions with the same a direction. Otherwise it is cut into three: a first region
    whose major vector is the first half of b (and minor vector the first half of a), the
    far part along b with the original vectors, and a last region that returns along -b.
    """
    cells = []

    def sign(v):
        return (v > 0) - (v < 0)

    def region(x, y, ax, ay, bx, by):
        w, h = abs(ax + ay), abs(bx + by)
        ux, uy, vx, vy = sign(ax), sign(ay), sign(bx), sign(by)
        if h == 1:
            cells.extend((x + i * ux, y + i * uy) for i in range(w))
            return
        if w == 1:
            cells.extend((x + i * vx, y + i * vy) for i in range(h))
            return
        na, nb = w // 2, h // 2
        if 2 * w > 3 * h:
            if na % 2 == 1 and w > 2:
                na += 1
            region(x, y, ux * na, uy * na, bx, by)
            region(x + ux * na, y + uy * na, ax - ux * na, ay - uy * na, bx, by)
        else:
            if nb % 2 == 1 and h > 2:
                nb += 1
            a2x, a2y, b2x, b2y = ux * na, uy * na, vx * nb, vy * nb
            region(x, y, b2x, b2y, a2x, a2y)
            region(x + b2x, y + b2y, ax, ay, bx - b2x, by - b2y)
            region(x + (ax - ux) + (b2x - vx), y + (ay - uy) + (b2y - vy), -b2x, -b2y, -(ax - a2x), -(ay - a2y))

    if W >= H:
        region(0, 0, W, 0, 0, H)
    else:
        region(0, 0, 0, H, W, 0)
    return np.array(cells, dtype=np.int64).reshape(-1, 2)


def rect_curve_perm(T: int, Hg: int, Wg: int):
    """As ``hilbert_perm`` with the frame order of ``rect_hilbert_curve(Wg, Hg)``."""
    frame = np.array([y * Wg + x for (x, y) in rect_hilbert_curve(Wg, Hg)], dtype=np.int64)
    hw = Hg * Wg
    perm = np.concatenate([t * hw + frame for t in range(T)]) if T > 0 else np.zeros(0, np.int64)
    inv = np.empty_like(perm)
    inv[perm] = np.arange(perm.size, dtype=np.int64)
    return perm, inv


def reorder(x_bnhd: np.ndarray, perm: np.ndarray) -> np.ndarray:
    """[B, N, H, d] raster -> [B, H, N, d] Hilbert order: out[b, h, i] = x[b, perm[i], h] (float64)."""
    x = np.asarray(x_bnhd, dtype=np.float64)
    return np.ascontiguousarray(x[:, perm, :, :].transpose(0, 2, 1, 3))


def inverse_reorder(o_bhnd: np.ndarray, perm: np.ndarray) -> np.ndarray:
    """[B, H, N, d] Hilbert order -> [B, N, H, d] raster: out[b, perm[i], h] = o[b, h, i]."""
    o = np.asarray(o_bhnd, dtype=np.float64)
    out = np.empty((o.shape[0], o.shape[2], o.shape[1], o.shape[3]), dtype=np.float64)
    out[:, perm, :, :] = o.transpose(0, 2, 1, 3)
    return out


# --------------------------------------------------------------------------------------
# Step 2: block pooling of Q and K ("pooled Q/K")
# [PD] 方法揭秘: the router estimates block importance from pooled Q/K.
# --------------------------------------------------------------------------------------


def n_blocks(N: int, block: int = BLOCK) -> int:
    return (N + block - 1) // block


def block_mean_pool(x_hnd: np.ndarray, block: int = BLOCK) -> np.ndarray:
    """Mean of each block's valid rows. x: [..., N, d] -> [..., nB, d] (float64).

    Block a covers rows [a*block, min((a+1)*block, N)); the last block averages only
    the rows it holds.
    """
    x = np.asarray(x_hnd, dtype=np.float64)
    N = x.shape[-2]
    nB = n_blocks(N, block)
    out = np.empty(x.shape[:-2] + (nB, x.shape[-1]), dtype=np.float64)
    for a in range(nB):
        lo, hi = a * block, min((a + 1) * block, N)
        out[..., a, :] = x[..., lo:hi, :].sum(axis=-2) / (hi - lo)
    return out


# --------------------------------------------------------------------------------------
# Steps 3-7: block importance, Top-p routing with a Top-k safety floor, CSR mask,
# per-head kept counts.
# [aixai] "Top-p vs Top-k": Top-k keeps a fixed number of key blocks per query block,
#   Top-p adapts the number to the importance distribution (concentrated heads keep
#   few, flat heads many).
# [aixai] "Sparse-routing frontend": Top-p routing combined with a Top-k safety floor
#   that keeps a minimum budget; one routing pass yields per-head density.
# [PD] 方法揭秘: Top-k floor = keep at least the k most important blocks.
# [PD] 龙迷三问: Top-p keeps blocks until the cumulative importance reaches the
#   threshold; Top-k keeps a fixed first k.
# --------------------------------------------------------------------------------------


def block_logits(pq: np.ndarray, pk: np.ndarray, d: int) -> np.ndarray:
    """s[a, b] = pooled_q[a] . pooled_k[b] / sqrt(d) for one head (float64, [nB, nB])."""
    return (np.asarray(pq, np.float64) @ np.asarray(pk, np.float64).T) / math.sqrt(d)


def importance(s_row: np.ndarray) -> np.ndarray:
    """Row softmax of the block logits: P_b = exp(s_b - max) / sum."""
    e = np.exp(s_row - s_row.max())
    return e / e.sum()


def routing_order(s_row: np.ndarray) -> np.ndarray:
    """Key blocks by logit descending, ties broken by the lower block index."""
    idx = np.arange(s_row.size)
    return np.lexsort((idx, -s_row))


def route_row(s_row: np.ndarray, p: float, k_floor: int) -> dict:
    """Top-p union Top-k for one (head, query-block) row of logits.

    Returns kept (sorted ascending), L_p, L_k, L, and the order/cumulative mass used.
    L_p = 1 + min{j : c_j >= p} with c_j the running sum of P over the order
    (sequential float64); p >= 1 keeps every block. The floor keeps the first
    min(k_floor, nB) blocks of the same order, so the union is the longer prefix.
    """
    nB = s_row.size
    order = routing_order(s_row)
    P = importance(s_row)
    c = np.cumsum(P[order])  # sequential running sum
    if p >= 1.0:
        L_p = nB
    else:
        hit = np.nonzero(c >= p)[0]
        L_p = int(hit[0]) + 1 if hit.size else nB
    L_k = min(max(int(k_floor), 0), nB)
    L = max(L_p, L_k)
    kept = np.sort(order[:L])
    return {"kept": kept, "L_p": L_p, "L_k": L_k, "L": L, "order": order, "c": c, "P": P}


def row_ambiguity(s_row: np.ndarray, info: dict, p: float, mass_tol: float = 1e-6,
                  logit_rel_tol: float = 1e-9) -> dict:
    """How close a row's decision is to a rounding-sensitive boundary.

    * mass: the cut L_p changes if c_{L_p-1} falls below p or c_{L_p-2} rises to p;
      the distance to p of those two cumulative masses (only when L_p decides L).
    * tie: the kept set changes if two logits around the boundary swap; the smallest
      gap between consecutive ordered logits at positions L-2, L-1, L.
    """
    nB = s_row.size
    L, L_p, L_k, c = info["L"], info["L_p"], info["L_k"], info["c"]
    mass_margin = math.inf
    if p < 1.0 and L_p >= L_k:
        if L_p - 1 < nB:
            mass_margin = min(mass_margin, abs(c[L_p - 1] - p))
        if L_p - 2 >= 0:
            mass_margin = min(mass_margin, abs(p - c[L_p - 2]))
    tie_margin = math.inf
    srt = s_row[info["order"]]
    for j in (L - 2, L - 1):
        if 0 <= j and j + 1 < nB:
            gap = srt[j] - srt[j + 1]
            tol = logit_rel_tol * max(1.0, abs(srt[j]))
            tie_margin = min(tie_margin, gap / tol)
    return {
        "mass_margin": mass_margin,
        "ambiguous_mass": mass_margin < mass_tol,
        # tie_margin in units of the tolerance; < 1 means the two logits are closer than it
        "ambiguous_tie": tie_margin < 1.0,
    }


def route(pq_bhnd: np.ndarray, pk_bhnd: np.ndarray, d: int, p: float, k_floor: int,
          with_ambiguity: bool = False) -> dict:
    """Route every (batch, head, query-block) row; build the CSR block mask.

    Rows are ordered r = (b*H + h)*nB + a. row_ptr[r+1] - row_ptr[r] = |kept(r)|,
    col_idx holds each row's kept key blocks ascending. head_kept[b*H + h] is the
    number of kept (query-block, key-block) pairs of that head (its load L_h, [aixai]
    "Runtime Load Balancing (RLB)").
    """
    pq = np.asarray(pq_bhnd, np.float64)
    pk = np.asarray(pk_bhnd, np.float64)
    B, H, nB, _ = pq.shape
    row_ptr = np.zeros(B * H * nB + 1, dtype=np.int64)
    cols = []
    head_kept = np.zeros(B * H, dtype=np.int64)
    amb_mass = np.zeros(B * H * nB, dtype=bool)
    amb_tie = np.zeros(B * H * nB, dtype=bool)
    L_p_all = np.zeros(B * H * nB, dtype=np.int64)
    r = 0
    for b in range(B):
        for h in range(H):
            s = block_logits(pq[b, h], pk[b, h], d)
            for a in range(nB):
                info = route_row(s[a], p, k_floor)
                cols.append(info["kept"])
                row_ptr[r + 1] = row_ptr[r] + info["kept"].size
                head_kept[b * H + h] += info["kept"].size
                L_p_all[r] = info["L_p"]
                if with_ambiguity:
                    amb = row_ambiguity(s[a], info, p)
                    amb_mass[r] = amb["ambiguous_mass"]
                    amb_tie[r] = amb["ambiguous_tie"]
                r += 1
    col_idx = np.concatenate(cols).astype(np.int64) if cols else np.zeros(0, np.int64)
    out = {"row_ptr": row_ptr, "col_idx": col_idx, "head_kept": head_kept, "L_p": L_p_all}
    if with_ambiguity:
        out["ambiguous_mass"] = amb_mass
        out["ambiguous_tie"] = amb_tie
    return out


def row_list(row_ptr: np.ndarray, col_idx: np.ndarray, r: int) -> np.ndarray:
    return col_idx[row_ptr[r]:row_ptr[r + 1]]


# --------------------------------------------------------------------------------------
# Longest-first work list (scheduling of the attention tiles)
# Not a step of the pages' method: the single-GPU stand-in for their observation that
# a few heavy heads dominate the load ([aixai] "Runtime Load Balancing (RLB)"). A tile
# is a pair of adjacent query blocks (2t, 2t+1) of one head; its cost is the number of
# key blocks in the union of the two rows' lists. Tiles are sorted by cost
# descending, ties by tile id ascending.
# --------------------------------------------------------------------------------------


def tile_costs(row_ptr: np.ndarray, col_idx: np.ndarray, BH: int, nB: int) -> np.ndarray:
    n_pairs = (nB + 1) // 2
    cost = np.zeros(BH * n_pairs, dtype=np.int64)
    for bh in range(BH):
        for t in range(n_pairs):
            rows = [bh * nB + a for a in (2 * t, 2 * t + 1) if a < nB]
            u = set()
            for r in rows:
                u.update(row_list(row_ptr, col_idx, r).tolist())
            cost[bh * n_pairs + t] = len(u)
    return cost


def lpt_order(cost: np.ndarray) -> np.ndarray:
    """Tile ids sorted by cost descending, ties by id ascending (stable)."""
    ids = np.arange(cost.size)
    return np.lexsort((ids, -cost))


# --------------------------------------------------------------------------------------
# Step 8: block-sparse attention over the mask
# [aixai] sparse attention section: for most queries only a small subset of key blocks
#   contributes; block masks skip the low-importance interactions.
# Reading: within a (head, query block) the softmax runs over the valid keys of the
# kept blocks only; there is no causal mask (bidirectional video DiT).
# --------------------------------------------------------------------------------------


def attention_rows(q_nd: np.ndarray, k_nd: np.ndarray, v_nd: np.ndarray, keys: np.ndarray,
                   scale: float) -> np.ndarray:
    """softmax(q k^T * scale) v over the given key rows, float64.

    An empty key set (a caller-made mask row that keeps no block; routing always keeps
    at least one) has no softmax; its output is taken to be zero."""
    q = np.asarray(q_nd, np.float64)
    if len(keys) == 0:
        return np.zeros((q.shape[0], np.asarray(v_nd).shape[-1]), dtype=np.float64)
    k = np.asarray(k_nd, np.float64)[keys]
    v = np.asarray(v_nd, np.float64)[keys]
    s = (q @ k.T) * scale
    s -= s.max(axis=1, keepdims=True)
    w = np.exp(s)
    w /= w.sum(axis=1, keepdims=True)
    return w @ v


def block_keys(blocks: np.ndarray, N: int, block: int = BLOCK) -> np.ndarray:
    """Valid key row indices covered by a list of key blocks."""
    parts = [np.arange(b * block, min((b + 1) * block, N)) for b in blocks]
    return np.concatenate(parts) if parts else np.zeros(0, np.int64)


def block_sparse_attention(q_bhnd, k_bhnd, v_bhnd, row_ptr, col_idx, scale=None,
                           rows=None, block: int = BLOCK) -> dict:
    """Attention of each requested (b, h, a) query block over its kept key blocks.

    Returns {(b, h, a): O rows [n_a, d]}; rows=None computes every query block.
    """
    B, H, N, d = q_bhnd.shape
    nB = n_blocks(N, block)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if rows is None:
        rows = [(b, h, a) for b in range(B) for h in range(H) for a in range(nB)]
    out = {}
    for (b, h, a) in rows:
        r = (b * H + h) * nB + a
        keys = block_keys(row_list(row_ptr, col_idx, r), N, block)
        lo, hi = a * block, min((a + 1) * block, N)
        out[(b, h, a)] = attention_rows(q_bhnd[b, h, lo:hi], k_bhnd[b, h], v_bhnd[b, h], keys, scale)
    return out


def dense_attention(q_bhnd, k_bhnd, v_bhnd, scale=None) -> np.ndarray:
    """Full softmax attention per (b, h), float64: the density-1 case."""
    B, H, N, d = q_bhnd.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out = np.empty((B, H, N, d), dtype=np.float64)
    keys = np.arange(N)
    for b in range(B):
        for h in range(H):
            out[b, h] = attention_rows(q_bhnd[b, h], k_bhnd[b, h], v_bhnd[b, h], keys, scale)
    return out


def assemble(blocks: dict, B: int, H: int, N: int, d: int, block: int = BLOCK) -> np.ndarray:
    """Place per-block outputs into a [B, H, N, d] array (all blocks must be present)."""
    o = np.empty((B, H, N, d), dtype=np.float64)
    for (b, h, a), val in blocks.items():
        o[b, h, a * block:a * block + val.shape[0]] = val
    return o


def kept_flops(row_ptr, col_idx, B: int, H: int, N: int, d: int, block: int = BLOCK) -> int:
    """Algorithmic FLOPs of the sparse attention: sum over kept (a, b) of 4 d n_a n_b."""
    nB = n_blocks(N, block)
    sizes = np.array([min(block, N - a * block) for a in range(nB)], dtype=np.int64)
    total = 0
    for r in range(B * H * nB):
        a = r % nB
        total += int(4 * d * sizes[a] * sizes[row_list(row_ptr, col_idx, r)].sum())
    return total
