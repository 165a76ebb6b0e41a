"""Pins for the oracle's working-order permutations (CPU only).

Each permutation is checked to be a bijection on the valid tokens, and checked
slot by slot against an independent construction: reshaping the padded grid of
token indices and transposing its axes.
"""
import numpy as np
import pytest

from oracle import layout


def _padded_grid(T, H, W, PT, PH, PW):
    g = np.full((PT, PH, PW), -1, dtype=np.int64)
    g[:T, :H, :W] = np.arange(T * H * W).reshape(T, H, W)
    return g


@pytest.mark.parametrize("dims,tile", [((4, 8, 8), (2, 4, 8)), ((21, 30, 52), (4, 4, 8)),
                                       ((5, 7, 9), (2, 4, 4)), ((21, 45, 80), (8, 4, 4))])
def test_tile_order_matches_axis_transpose(dims, tile):
    T, H, W = dims
    bt, bh, bw = tile
    nt, nh, nw = layout.tile_grid_dims(T, H, W, bt, bh, bw)
    g = _padded_grid(T, H, W, nt * bt, nh * bh, nw * bw)
    ref = g.reshape(nt, bt, nh, bh, nw, bw).transpose(0, 2, 4, 1, 3, 5).reshape(-1)
    np.testing.assert_array_equal(layout.tile_order(T, H, W, bt, bh, bw), ref)


@pytest.mark.parametrize("dims", [(4, 8, 8), (30, 48, 80), (3, 5, 7)])
def test_frame_major_matches_axis_transpose(dims):
    T, H, W = dims
    n = T * H * W
    ref = np.arange(n).reshape(T, H, W).transpose(1, 2, 0).reshape(-1)
    got = layout.frame_major_order(T, H, W, 128)
    np.testing.assert_array_equal(got[:n], ref)
    assert np.all(got[n:] == -1) and len(got) % 128 == 0


@pytest.mark.parametrize("maker", [
    lambda: (layout.tile_order(5, 7, 9, 2, 4, 4), 315),
    lambda: (layout.frame_major_order(5, 7, 9, 64), 315),
    lambda: (layout.identity_order(5, 7, 9, 64), 315),
])
def test_bijection_and_inverse(maker):
    order, n = maker()
    valid = order[order >= 0]
    assert sorted(valid.tolist()) == list(range(n))
    inv = layout.inverse(order, n)
    np.testing.assert_array_equal(order[inv], np.arange(n))        # forward(inverse) = id
    slots = np.nonzero(order >= 0)[0]
    np.testing.assert_array_equal(inv[order[slots]], slots)         # inverse(forward) = id


def test_tile_order_coordinates_token_by_token():
    # Slot m = tile_id*(bt*bh*bw) + (lt*bh + lh)*bw + lw holds token (t*H+h)*W+w.
    T, H, W, bt, bh, bw = 3, 5, 6, 2, 2, 4
    order = layout.tile_order(T, H, W, bt, bh, bw)
    nt, nh, nw = 2, 3, 2
    for t in range(T):
        for h in range(H):
            for w in range(W):
                tid = ((t // bt) * nh + h // bh) * nw + w // bw
                m = tid * bt * bh * bw + ((t % bt) * bh + h % bh) * bw + w % bw
                assert order[m] == (t * H + h) * W + w
