"""Working-order permutations of the T x H x W token grid (test infrastructure).

Original order of a token is n = (t*H + h)*W + w. A "working layout" is a
sequence of token slots, grouped into blocks of consecutive slots; each slot
holds an original token index or -1 for a padding slot.
"""
import numpy as np


def _ceil_div(a, b):
    return -(-a // b)


def identity_order(T, H, W, block):
    """Original order, padded with -1 to a multiple of ``block`` slots."""
    n = T * H * W
    n_pad = _ceil_div(n, block) * block
    out = np.full(n_pad, -1, dtype=np.int64)
    out[:n] = np.arange(n)
    return out


def tile_order(T, H, W, bt, bh, bw):
    """3D tile order.

    Sliding Tile Attention review, key machinery: tokens are grouped into
    bt x bh x bw cubes whose size equals one attention block, and the tokens of
    one tile are kept consecutive. The grid is tiled from the origin and padded
    at the high end of each axis. Tiles are visited in raster order (tw
    fastest); inside a tile, tokens are in raster order (lw fastest).
    Slot m = tile_id * (bt*bh*bw) + (lt*bh + lh)*bw + lw.
    """
    nt, nh, nw = _ceil_div(T, bt), _ceil_div(H, bh), _ceil_div(W, bw)
    out = []
    for tt in range(nt):
        for th in range(nh):
            for tw in range(nw):
                for lt in range(bt):
                    for lh in range(bh):
                        for lw in range(bw):
                            t, h, w = tt * bt + lt, th * bh + lh, tw * bw + lw
                            if t < T and h < H and w < W:
                                out.append((t * H + h) * W + w)
                            else:
                                out.append(-1)
    return np.array(out, dtype=np.int64)


def frame_major_order(T, H, W, block):
    """Token-major to frame-major transpose.

    Sparse VideoGen review, key machinery: activations are transposed from
    token-major to frame-major order, so the tokens at one spatial position in
    all frames become consecutive. Slot m = (h*W + w)*T + t holds token
    n = (t*H + h)*W + w. Padded with -1 to a multiple of ``block``.
    """
    n = T * H * W
    out = np.full(_ceil_div(n, block) * block, -1, dtype=np.int64)
    for h in range(H):
        for w in range(W):
            for t in range(T):
                out[(h * W + w) * T + t] = (t * H + h) * W + w
    return out


def blocks(order, block):
    """[n_blocks, block] view of a working order (slot -> original index or -1)."""
    assert len(order) % block == 0
    return order.reshape(-1, block)


def inverse(order, n):
    """Original index -> slot. Every original token appears exactly once."""
    inv = np.full(n, -1, dtype=np.int64)
    valid = order >= 0
    inv[order[valid]] = np.nonzero(valid)[0]
    return inv


def tile_grid_dims(T, H, W, bt, bh, bw):
    return _ceil_div(T, bt), _ceil_div(H, bh), _ceil_div(W, bw)
