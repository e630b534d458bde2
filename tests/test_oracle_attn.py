"""Pins for the oracle's block-sparse and dense attention (CPU only).

Pinned by torch's float64 scaled_dot_product_attention (the library routine), with an
additive -inf block mask built from the CSR for the sparse case; by permutation
equivariance of dense attention under the Hilbert reorder; by the one-key case
(output = that key's value); and by the p = 1 case collapsing to dense attention.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O


def _sdpa(q, k, v, mask=None):
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(torch.float64)
    m = None if mask is None else t(mask)
    return torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), attn_mask=m).numpy()


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def test_dense_matches_sdpa():
    B, H, N, d = 1, 2, 64 * 3 + 9, 32
    q, k, v = _rand((B, H, N, d), 1, 2.0), _rand((B, H, N, d), 2, 2.0), _rand((B, H, N, d), 3)
    np.testing.assert_allclose(O.dense_attention(q, k, v), _sdpa(q, k, v), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("p,kf", [(0.5, 1), (0.8, 2), (0.3, 0)])
def test_sparse_matches_masked_sdpa(p, kf):
    B, H, N, d = 1, 2, 64 * 5 + 20, 16
    q, k, v = _rand((B, H, N, d), 4, 3.0), _rand((B, H, N, d), 5, 3.0), _rand((B, H, N, d), 6)
    pq, pk = O.block_mean_pool(q), O.block_mean_pool(k)
    R = O.route(pq, pk, d, p, kf)
    nB = O.n_blocks(N)
    mask = np.full((B, H, N, N), -np.inf)
    for h in range(H):
        for a in range(nB):
            for b in O.row_list(R["row_ptr"], R["col_idx"], h * nB + a):
                mask[0, h, a * 64:(a + 1) * 64, b * 64:(b + 1) * 64] = 0.0
    got = O.assemble(O.block_sparse_attention(q, k, v, R["row_ptr"], R["col_idx"]), B, H, N, d)
    np.testing.assert_allclose(got, _sdpa(q, k, v, mask), rtol=1e-12, atol=1e-12)
    # the mask is genuinely sparse here, so the result differs from dense attention
    assert R["row_ptr"][-1] < H * nB * nB
    assert np.abs(got - O.dense_attention(q, k, v)).max() > 1e-3


def test_empty_rows_give_zeros_and_leave_other_rows_alone():
    # a caller-made mask: rows 0 and 3 keep nothing, the others keep scattered blocks
    B, H, N, d = 1, 1, 64 * 5 + 11, 16
    q, k, v = _rand((B, H, N, d), 21, 2.0), _rand((B, H, N, d), 22, 2.0), _rand((B, H, N, d), 23)
    lists = [[], [0, 4], [2], [], [1, 3, 5], [5]]
    nB = O.n_blocks(N)
    assert nB == len(lists)
    row_ptr = np.concatenate([[0], np.cumsum([len(x) for x in lists])]).astype(np.int64)
    col_idx = np.array([b for x in lists for b in x], dtype=np.int64)
    got = O.assemble(O.block_sparse_attention(q, k, v, row_ptr, col_idx), B, H, N, d)
    mask = np.full((B, H, N, N), -np.inf)
    for a, keep in enumerate(lists):
        for b in keep:
            mask[0, 0, a * 64:(a + 1) * 64, b * 64:(b + 1) * 64] = 0.0
    want = _sdpa(q, k, v, mask)
    for a, keep in enumerate(lists):
        lo, hi = a * 64, min(a * 64 + 64, N)
        if keep:
            np.testing.assert_allclose(got[0, 0, lo:hi], want[0, 0, lo:hi], rtol=1e-12, atol=1e-12)
        else:
            assert np.all(got[0, 0, lo:hi] == 0.0)


def test_p_one_equals_dense():
    B, H, N, d = 1, 1, 64 * 4 + 3, 16
    q, k, v = _rand((B, H, N, d), 7, 2.0), _rand((B, H, N, d), 8, 2.0), _rand((B, H, N, d), 9)
    R = O.route(O.block_mean_pool(q), O.block_mean_pool(k), d, 1.0, 0)
    got = O.assemble(O.block_sparse_attention(q, k, v, R["row_ptr"], R["col_idx"]), B, H, N, d)
    np.testing.assert_allclose(got, _sdpa(q, k, v), rtol=1e-12, atol=1e-12)


def test_permutation_equivariance_under_hilbert_reorder():
    T, Hg, Wg, H, d = 2, 6, 11, 2, 8
    N = T * Hg * Wg
    x = [_rand((1, N, H, d), s, 1.5) for s in (10, 11, 12)]
    perm, _ = O.hilbert_perm(T, Hg, Wg)
    o_h = O.dense_attention(*[O.reorder(a, perm) for a in x])
    o_raster = _sdpa(*[a.transpose(0, 2, 1, 3) for a in x]).transpose(0, 2, 1, 3)
    np.testing.assert_allclose(O.inverse_reorder(o_h, perm), o_raster, rtol=1e-12, atol=1e-12)


def test_single_valid_key_returns_its_value():
    # N = 64*2 + 1: the tail block holds one key; route every row to it alone
    B, H, N, d = 1, 1, 129, 8
    q, k, v = _rand((B, H, N, d), 13), _rand((B, H, N, d), 14), _rand((B, H, N, d), 15)
    nB = 3
    rp = np.arange(nB + 1)
    ci = np.full(nB, 2)
    out = O.block_sparse_attention(q, k, v, rp, ci)
    for a in range(nB):
        np.testing.assert_allclose(out[(0, 0, a)], np.broadcast_to(v[0, 0, 128], out[(0, 0, a)].shape), rtol=0, atol=1e-15)


def test_scale_argument():
    B, H, N, d = 1, 1, 70, 8
    q, k, v = _rand((B, H, N, d), 16), _rand((B, H, N, d), 17), _rand((B, H, N, d), 18)
    got = O.dense_attention(q, k, v, scale=0.5)
    want = O.dense_attention(q * (0.5 * math.sqrt(d)), k, v)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def test_kept_flops_counts_valid_tokens():
    # 2 blocks, N = 64 + 10: row 0 keeps {0,1}, row 1 keeps {1}
    rp = np.array([0, 2, 3])
    ci = np.array([0, 1, 1])
    d = 4
    want = 4 * d * (64 * 64 + 64 * 10 + 10 * 10)
    assert O.kept_flops(rp, ci, 1, 1, 74, d) == want
