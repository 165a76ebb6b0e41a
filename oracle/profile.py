"""SVG online head profiler, written out plainly (test infrastructure).

Sparse VideoGen review, key machinery (Algorithm 1): for every head, on a
random 1 % of its query rows, attention is computed three times -- over all
keys, over the keys of the spatial pattern and over the keys of the temporal
pattern -- and the head is given the pattern whose output has the lower mean
squared error against the full output.

Readings (the pages leave these open):
* the two patterns are the block masks of the spatial/temporal heads built by
  ``oracle.masks`` (spatial: identity layout, frames within +-frame_radius;
  temporal: frame-major layout, a shared spatial position), both with the
  sink blocks;
* the error is the mean over the sampled rows and the head dimension of
  (O_pattern - O_full)^2;
* a tie goes to the spatial pattern;
* the sampled rows are an input (``synthetic.sample_rows`` draws them).
"""
import numpy as np

from . import attention, layout, masks


def pattern_keep(rows, T, H, W, block, sink_tokens, frame_radius, temporal):
    """[len(rows), N] bool: the keys each sampled query keeps under one pattern."""
    n = T * H * W
    order = (layout.frame_major_order(T, H, W, block) if temporal
             else layout.identity_order(T, H, W, block))
    blk = layout.blocks(order, block)
    bm = (masks.temporal_rule(blk, T, H, W) if temporal
          else masks.spatial_rule(blk, T, H, W, frame_radius))
    bm = masks.add_sinks(bm, blk, sink_tokens, block)
    slot = layout.inverse(order, n)
    keep = np.zeros((len(rows), n), dtype=bool)
    for r, tok in enumerate(rows):
        keys = blk[np.nonzero(bm[slot[tok] // block])[0]].reshape(-1)
        keep[r, keys[keys >= 0]] = True
    return keep


def profile_head(q, k, v, rows, T, H, W, block, sink_tokens, frame_radius=1, chunk=256):
    """Outputs on the sampled rows, the two errors and the decision for one head.

    q, k, v: float32 [N, d] (bf16 values); rows: sampled token indices.
    """
    rows = np.asarray(rows)
    n = T * H * W
    keep_s = pattern_keep(rows, T, H, W, block, sink_tokens, frame_radius, temporal=False)
    keep_t = pattern_keep(rows, T, H, W, block, sink_tokens, frame_radius, temporal=True)
    outs = {"full": [], "spatial": [], "temporal": []}
    for a in range(0, len(rows), chunk):
        r = rows[a:a + chunk]
        outs["full"].append(attention.masked_attention_rows(q, k, v, r, np.ones((len(r), n), bool))[0])
        outs["spatial"].append(attention.masked_attention_rows(q, k, v, r, keep_s[a:a + chunk])[0])
        outs["temporal"].append(attention.masked_attention_rows(q, k, v, r, keep_t[a:a + chunk])[0])
    o = {key: np.concatenate(val) for key, val in outs.items()}
    mse_s = float(np.mean((o["spatial"] - o["full"]) ** 2))
    mse_t = float(np.mean((o["temporal"] - o["full"]) ** 2))
    return dict(mse_spatial=mse_s, mse_temporal=mse_t, temporal=mse_t < mse_s,
                o_full=o["full"], o_spatial=o["spatial"], o_temporal=o["temporal"])


def window_keep(rows, T, H, W, tile, win):
    """[len(rows), N] bool: the keys a sampled query keeps under one tile window.

    The block mask of the sliding tile window (Sliding Tile Attention review,
    core discovery; ``masks.tile_window``) on the 3D tile layout, read per
    query token through the tile that holds it.
    """
    n = T * H * W
    order = layout.tile_order(T, H, W, *tile)
    blk = layout.blocks(order, tile[0] * tile[1] * tile[2])
    valid = masks.valid_blocks(blk)
    bm = masks.tile_window(layout.tile_grid_dims(T, H, W, *tile), win, valid, valid)
    slot = layout.inverse(order, n)
    bs = blk.shape[1]
    keep = np.zeros((len(rows), n), dtype=bool)
    for r, tok in enumerate(rows):
        keys = blk[np.nonzero(bm[slot[tok] // bs])[0]].reshape(-1)
        keep[r, keys[keys >= 0]] = True
    return keep


def sta_window_search(q, k, v, rows, T, H, W, tile, candidates, chunk=256):
    """Per-head window search (Sliding Tile Attention review, key machinery:
    Algorithm 1 picks each head's window by the mask minimizing the MSE to full
    attention). Reading: the candidate windows are the caller's; the error is
    the mean over the sampled rows and head_dim of (O_window - O_full)^2; the
    lowest error wins, ties to the earlier candidate.
    """
    rows = np.asarray(rows)
    n = T * H * W
    keeps = [window_keep(rows, T, H, W, tile, c) for c in candidates]
    full, outs = [], [[] for _ in candidates]
    for a in range(0, len(rows), chunk):
        r = rows[a:a + chunk]
        full.append(attention.masked_attention_rows(q, k, v, r, np.ones((len(r), n), bool))[0])
        for ci, kp in enumerate(keeps):
            outs[ci].append(attention.masked_attention_rows(q, k, v, r, kp[a:a + chunk])[0])
    o_full = np.concatenate(full)
    o = [np.concatenate(x) for x in outs]
    mse = [float(np.mean((oc - o_full) ** 2)) for oc in o]
    best = 0
    for ci in range(1, len(mse)):
        if mse[ci] < mse[best]:
            best = ci
    return dict(mse=mse, choice=best, o_full=o_full, o=o)
