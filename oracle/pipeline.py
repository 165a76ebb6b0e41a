"""Per-head mask construction for each workload kind (test infrastructure).

``head_mask(wl, q, k, head)`` takes one head's q and k as float32 [N, d]
(bf16 values, original token order) and returns the working order, the block
mask and the intermediate values that decide it.
"""
import numpy as np

from . import layout, masks


def working_order(wl, head, tile=None):
    """Slot -> original token for this head's working layout."""
    if wl.kind in ("topk", "sta", "spade"):
        bt, bh, bw = tile if tile is not None else wl.tile
        return layout.tile_order(wl.T, wl.H, wl.W, bt, bh, bw)
    if wl.kind == "spatiotemporal" and head in wl.temporal_heads:
        return layout.frame_major_order(wl.T, wl.H, wl.W, wl.block)
    return layout.identity_order(wl.T, wl.H, wl.W, wl.block)


def head_mask(wl, q, k, head, force_choice=None):
    """``force_choice`` (SPADE) evaluates the given candidate instead of the
    argmax, for a head whose summed SICS scores tie within the tolerance."""
    d = wl.head_dim
    info = {}
    if wl.kind == "fg" and wl.fg_rule == "cached":
        tau = 0.5 / k.shape[0]
        info.update(tau=tau)
        return dict(keep_groups=masks.fg_cached_keep(q, k, wl.fg_group, tau), info=info)
    if wl.kind == "fg":
        s = masks.fg_scores(q, k, wl.fg_group)
        tau, r = masks.fg_threshold(s, wl.fg_keep_fraction)
        info.update(scores=s, tau=tau, rank=r)
        return dict(keep_groups=masks.fg_keep(s, tau), info=info)

    tile = None
    if wl.kind == "spade":
        totals = []
        for cand in wl.candidates:
            blk_c = layout.blocks(working_order(wl, head, cand), wl.block)
            totals.append(float(masks.sics(k, blk_c).astype(np.float64).sum()))
        choice = masks.choose_candidate(totals)
        info.update(sics_totals=totals, choice=choice)
        if force_choice is not None:
            choice = force_choice
        tile = wl.candidates[choice]

    order = working_order(wl, head, tile)
    blk = layout.blocks(order, wl.block)
    valid = masks.valid_blocks(blk)

    if wl.kind == "topk":
        s = masks.pooled_scores(masks.block_summaries(q, blk, wl.summarizer),
                                masks.block_summaries(k, blk, wl.summarizer), d)
        info["scores"] = s
        bm = masks.topk_with_diagonal(s, wl.topk, wl.keep_diagonal, valid, valid)
    elif wl.kind == "sta":
        dims = layout.tile_grid_dims(wl.T, wl.H, wl.W, *wl.tile)
        # Sliding Tile Attention review: heads specialize in different window
        # sizes; a per-head window replaces the policy's one for its head
        win = wl.head_windows[head] if wl.head_windows else wl.window
        bm = masks.tile_window(dims, win, valid, valid)
    elif wl.kind == "spatiotemporal":
        if head in wl.temporal_heads:
            bm = masks.temporal_rule(blk, wl.T, wl.H, wl.W)
        else:
            bm = masks.spatial_rule(blk, wl.T, wl.H, wl.W)
        bm = masks.add_sinks(bm, blk, wl.sink_tokens, wl.block)
    elif wl.kind == "spade":
        s = masks.pooled_scores(masks.block_summaries(q, blk, wl.summarizer),
                                masks.block_summaries(k, blk, wl.summarizer), d)
        info["scores"] = s
        dims = layout.tile_grid_dims(wl.T, wl.H, wl.W, *tile)
        bm = masks.tile_window(dims, wl.window, valid, valid)
        for i in range(blk.shape[0]):
            if valid[i]:
                bm[i] |= masks.top_p_row(s[i], valid, wl.top_p)
    else:
        raise ValueError(wl.kind)
    return dict(order=order, order_blocks=blk, bmask=bm, tile=tile, info=info)
