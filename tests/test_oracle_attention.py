"""Pins for the oracle's masked attention (CPU only).

The oracle's softmax path is checked against independent library routines
(torch's scaled_dot_product_attention and logsumexp in float64), against the
row-sum invariant, and against the special cases the pages fix: an all-ones
mask and a sliding-tile window covering the whole grid are dense attention.
"""
import math

import numpy as np
import pytest
import torch

from oracle import attention, layout, masks


def _rand(n, d, seed):
    g = np.random.default_rng(seed)
    return [g.standard_normal((n, d)).astype(np.float32) for _ in range(3)]


def _sdpa(q, k, v, keep=None):
    tq, tk, tv = (torch.from_numpy(x.astype(np.float64))[None, None] for x in (q, k, v))
    m = None if keep is None else torch.from_numpy(keep)[None, None]
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=m)
    s = (tq @ tk.transpose(-1, -2)) / math.sqrt(q.shape[1])
    if keep is not None:
        s = s.masked_fill(~m, -math.inf)
    return o[0, 0].numpy(), torch.logsumexp(s, dim=-1)[0, 0].numpy()


def test_all_ones_mask_is_dense_sdpa():
    q, k, v = _rand(96, 64, 1)
    rows = np.arange(96)
    o, lse = attention.masked_attention_rows(q, k, v, rows, np.ones((96, 96), bool))
    o_ref, lse_ref = _sdpa(q, k, v)
    np.testing.assert_allclose(o, o_ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, rtol=1e-12, atol=1e-12)


def test_random_mask_matches_sdpa_boolean_mask():
    q, k, v = _rand(80, 32, 2)
    g = np.random.default_rng(3)
    keep = g.random((80, 80)) < 0.3
    keep[np.arange(80), g.integers(0, 80, 80)] = True      # no empty row
    o, lse = attention.masked_attention_rows(q, k, v, np.arange(80), keep)
    o_ref, lse_ref = _sdpa(q, k, v, keep)
    np.testing.assert_allclose(o, o_ref, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, rtol=1e-12, atol=1e-12)


def test_weights_rows_sum_to_one_and_masked_entries_zero():
    q, k, _ = _rand(50, 16, 4)
    g = np.random.default_rng(5)
    keep = g.random((50, 50)) < 0.5
    keep[:, 0] = True
    w = attention.masked_attention_weights(q, k, np.arange(50), keep)
    np.testing.assert_allclose(w.sum(axis=1), 1.0, atol=1e-12)
    assert np.all(w[~keep] == 0.0)


def test_empty_row_gives_zero_output_and_minus_inf_lse():
    q, k, v = _rand(8, 16, 6)
    keep = np.ones((8, 8), bool)
    keep[3] = False
    o, lse = attention.masked_attention_rows(q, k, v, np.arange(8), keep)
    assert np.all(o[3] == 0.0) and lse[3] == -np.inf
    assert np.all(np.isfinite(lse[np.arange(8) != 3]))


def test_duplicated_keys_add_ln2_to_lse():
    # Listing every key twice doubles each exponential: O is unchanged and the
    # log-sum-exp grows by exactly ln 2.
    q, k, v = _rand(20, 16, 7)
    rows = np.arange(20)
    o1, l1 = attention.masked_attention_rows(q, k, v, rows, np.ones((20, 20), bool))
    k2, v2 = np.concatenate([k, k]), np.concatenate([v, v])
    o2, l2 = attention.masked_attention_rows(q, k2, v2, rows, np.ones((20, 40), bool))
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(l2 - l1, math.log(2.0), atol=1e-12)


def test_sta_window_covering_whole_grid_is_dense():
    # Sliding Tile Attention review: a window at least as large as the tile grid
    # keeps every tile, so block-sparse attention equals dense attention.
    T, H, W, tile = 3, 5, 6, (2, 2, 4)
    n = T * H * W
    q, k, v = _rand(n, 32, 8)
    order = layout.tile_order(T, H, W, *tile)
    blk = layout.blocks(order, 16)
    dims = layout.tile_grid_dims(T, H, W, *tile)
    valid = masks.valid_blocks(blk)
    win = tuple(2 * x + 1 for x in dims)
    bm = masks.tile_window(dims, win, valid, valid)
    o, lse = attention.block_sparse_attention(q, k, v, blk, bm)
    o_ref, lse_ref = _sdpa(q, k, v)
    np.testing.assert_allclose(o, o_ref, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, rtol=1e-12, atol=1e-12)


def test_block_sparse_equals_token_level_brute_force():
    # Blocks -> per-token keep sets, done here by an independent route:
    # slot of every token via the inverse order, block = slot // BS.
    T, H, W, tile = 2, 4, 4, (1, 2, 4)
    n, bs = T * H * W, 8
    q, k, v = _rand(n, 16, 9)
    order = layout.tile_order(T, H, W, *tile)
    blk = layout.blocks(order, bs)
    g = np.random.default_rng(10)
    bm = g.random((blk.shape[0], blk.shape[0])) < 0.5
    bm[np.arange(blk.shape[0]), np.arange(blk.shape[0])] = True
    o, lse = attention.block_sparse_attention(q, k, v, blk, bm)
    inv = layout.inverse(order, n)
    for i in range(n):
        ks = [j for j in range(n) if bm[inv[i] // bs, inv[j] // bs]]
        s = np.array([float(np.dot(q[i].astype(np.float64), k[j])) / 4.0 for j in ks])
        p = np.exp(s - s.max())
        o_i = (p[:, None] * v[ks].astype(np.float64)).sum(0) / p.sum()
        np.testing.assert_allclose(o[i], o_i, rtol=1e-11, atol=1e-12)
        assert abs(lse[i] - (s.max() + math.log(p.sum()))) < 1e-12


@pytest.mark.parametrize("group", [4, 5])
def test_slice_attention_matches_per_group_keep(group):
    n = 23
    q, k, v = _rand(n, 8, 11)
    g = np.random.default_rng(12)
    G = -(-n // group)
    keep = g.random((G, n)) < 0.4
    keep[:, 0] = True
    o, lse = attention.slice_attention(q, k, v, keep, group)
    for i in range(n):
        kk = np.broadcast_to(keep[i // group], (1, n))
        oi, li = attention.masked_attention_rows(q, k, v, np.array([i]), kk)
        np.testing.assert_allclose(o[i], oi[0], rtol=1e-13)
