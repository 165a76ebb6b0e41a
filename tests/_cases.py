"""Helpers shared by the GPU parity tests: workload -> policy, small variants
of each workload, and the mask / output comparisons with their tolerances."""
import math

import numpy as np

from synthetic import CONFIGS, Workload

# Output tolerances for unit-scale bf16 inputs (the workload statement's bar).
O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3
LSE_MAX_ABS = 1e-3
# A mask decision whose deciding value is within this relative distance of the
# cut-off may go either way.
REL_TIE = 1e-4


def policy_kwargs(wl: Workload):
    if wl.kind == "topk":
        return dict(kind="topk", block=wl.block, tile=wl.tile, topk=wl.topk,
                    keep_diagonal=wl.keep_diagonal, summarizer=wl.summarizer)
    if wl.kind == "sta":
        return dict(kind="sta", block=wl.block, tile=wl.tile, window=wl.window,
                    head_windows=wl.head_windows or None)
    if wl.kind == "spatiotemporal":
        return dict(kind="spatiotemporal", block=wl.block, temporal_heads=wl.temporal_heads,
                    heads=wl.heads, sink_tokens=wl.sink_tokens, frame_radius=1)
    if wl.kind == "spade":
        return dict(kind="spade", block=wl.block, candidates=wl.candidates, top_p=wl.top_p,
                    window=wl.window, summarizer=wl.summarizer)
    if wl.kind == "fg":
        return dict(kind="fg", block=wl.block, fg_group=wl.fg_group,
                    fg_keep_fraction=wl.fg_keep_fraction)
    raise ValueError(wl.kind)


# Small variants: several tiles, ragged grids (padding on every axis where the
# tile allows), head_dim 64 and 128. config_id 100+ keeps their seeds apart.
SMALL = {
    "tiny_topk": CONFIGS["tiny_topk"],
    "topk_ragged_d128": Workload(name="topk_ragged_d128", config_id=101, T=7, H=9, W=13, heads=2,
                                 head_dim=128, kind="topk", tile=(2, 8, 8), block=128, topk=3,
                                 keep_diagonal=True),
    "sta_ragged": Workload(name="sta_ragged", config_id=102, T=9, H=10, W=19, heads=3,
                           head_dim=128, kind="sta", tile=(4, 4, 8), block=128, window=(3, 3, 3)),
    "sta_d64": Workload(name="sta_d64", config_id=103, T=6, H=8, W=16, heads=2, head_dim=64,
                        kind="sta", tile=(2, 4, 8), block=64, window=(3, 3, 3)),
    "spatiotemporal_ragged": Workload(name="spatiotemporal_ragged", config_id=104, T=6, H=12,
                                      W=20, heads=4, head_dim=128, kind="spatiotemporal",
                                      block=128, sink_tokens=226, temporal_heads=(1, 3)),
    "spade_ragged": Workload(name="spade_ragged", config_id=105, T=7, H=13, W=24, heads=3,
                             head_dim=128, kind="spade", block=128,
                             candidates=((1, 8, 16), (8, 4, 4), (2, 8, 8)), top_p=0.9,
                             window=(3, 3, 3)),
    "spade_d64": Workload(name="spade_d64", config_id=106, T=5, H=9, W=16, heads=2, head_dim=64,
                          kind="spade", block=128, candidates=((1, 8, 16), (8, 4, 4), (2, 8, 8)),
                          top_p=0.9, window=(3, 3, 3)),
    # candidates whose common region holds 1,024 atoms: the pooling falls back
    # to the per-candidate kernel
    "spade_pool_fallback": Workload(name="spade_pool_fallback", config_id=107, T=8, H=6, W=136,
                                    heads=2, head_dim=128, kind="spade", block=128,
                                    candidates=((1, 1, 128), (8, 4, 4)), top_p=0.9,
                                    window=(3, 3, 3)),
    # max / min block summaries (SPADE review, minor comment 3): the atom
    # pooling kernel, the per-candidate kernel and Top-K
    "spade_max": Workload(name="spade_max", config_id=108, T=7, H=13, W=24, heads=3,
                          head_dim=128, kind="spade", block=128,
                          candidates=((1, 8, 16), (8, 4, 4), (2, 8, 8)), top_p=0.9,
                          window=(3, 3, 3), summarizer="max"),
    "spade_fallback_min": Workload(name="spade_fallback_min", config_id=109, T=8, H=6, W=136,
                                   heads=2, head_dim=128, kind="spade", block=128,
                                   candidates=((1, 1, 128), (8, 4, 4)), top_p=0.9,
                                   window=(3, 3, 3), summarizer="min"),
    "topk_max_d64": CONFIGS["tiny_topk"].with_(name="topk_max_d64", config_id=110,
                                               summarizer="max"),
    # head_dim 64 with 128-token blocks on the one-warpgroup kernel
    "spatiotemporal_d64": Workload(name="spatiotemporal_d64", config_id=112, T=5, H=9, W=16,
                                   heads=2, head_dim=64, kind="spatiotemporal", block=128,
                                   sink_tokens=100, temporal_heads=(1,)),
    # a window per head (Sliding Tile Attention review: head specialization)
    "sta_head_windows": Workload(name="sta_head_windows", config_id=111, T=9, H=10, W=19, heads=3,
                                 head_dim=128, kind="sta", tile=(4, 4, 8), block=128,
                                 window=(3, 3, 3), head_windows=((1, 1, 1), (3, 5, 3), (5, 1, 1))),
}


def bits_to_bool(words, nb):
    """[nb, W32] uint32 rows -> [nb, nb] bool."""
    words = np.asarray(words, dtype=np.uint32).reshape(-1, (nb + 31) // 32)
    bits = np.unpackbits(words.view(np.uint8), bitorder="little").reshape(words.shape[0], -1)
    return bits[:, :nb].astype(bool)


def pack_rows(dense):
    """[..., nb] bool -> [..., ceil(nb/32)] uint32 with bit b of word w = column 32w+b."""
    nb = dense.shape[-1]
    w32 = (nb + 31) // 32
    pad = np.zeros(dense.shape[:-1] + (w32 * 32,), bool)
    pad[..., :nb] = dense
    b = pad.reshape(dense.shape[:-1] + (w32, 32)).astype(np.uint64)
    return (b << np.arange(32, dtype=np.uint64)).sum(-1).astype(np.uint32)


def ambiguous_topk(scores_row, k, valid):
    """Blocks whose rank against the k-th score is within REL_TIE may differ."""
    cols = np.nonzero(valid)[0]
    v = np.sort(scores_row[cols].astype(np.float64))[::-1]
    if len(v) <= k:
        return np.zeros(len(valid), bool)
    cut = 0.5 * (v[k - 1] + v[k])
    band = REL_TIE * max(abs(v[k - 1]), abs(v[k]), 1e-30)
    amb = np.zeros(len(valid), bool)
    if abs(v[k - 1] - v[k]) <= 2 * band:
        amb[cols] = np.abs(scores_row[cols].astype(np.float64) - cut) <= 2 * band
    return amb


def ambiguous_top_p(scores_row, valid, p):
    """Blocks whose Top-P membership is within REL_TIE of the cut."""
    cols = np.nonzero(valid)[0]
    s = scores_row[cols].astype(np.float64)
    e = np.exp(s - s.max())
    pr = e / e.sum()
    order = sorted(range(len(cols)), key=lambda a: (-pr[a], cols[a]))
    c = np.cumsum(pr[order])
    L = int(np.searchsorted(c, p * (1 - 1e-12))) + 1          # prefix length reaching p
    L = min(L, len(order))
    amb = np.zeros(len(valid), bool)
    p_cut = pr[order[L - 1]]
    amb[cols] = np.abs(pr - p_cut) <= REL_TIE * p_cut
    # a running sum that reaches p within REL_TIE at the crossing makes the
    # crossing block and its neighbour either way
    for pos in (L - 2, L - 1):
        if 0 <= pos < len(c) and abs(c[pos] - p) <= REL_TIE * p:
            for a in (pos, pos + 1):
                if 0 <= a < len(order):
                    amb[cols[order[a]]] = True
    return amb


def attention_errors(o_gpu, lse_gpu, o_ref, lse_ref):
    o_err = np.abs(o_gpu.astype(np.float64) - o_ref)
    fin = np.isfinite(lse_ref)
    lse_err = np.abs(lse_gpu[fin].astype(np.float64) - lse_ref[fin]) if fin.any() else np.zeros(1)
    assert np.all(np.isneginf(lse_gpu[~fin])), "rows with no kept key must have LSE = -inf"
    return float(o_err.max()), float(o_err.mean()), float(lse_err.max())


def check_errors(o_max, o_mean, lse_max, where=""):
    assert o_max <= O_MAX_ABS, f"{where}: O max-abs {o_max:.3e} > {O_MAX_ABS}"
    assert o_mean <= O_MEAN_ABS, f"{where}: O mean-abs {o_mean:.3e} > {O_MEAN_ABS}"
    assert lse_max <= LSE_MAX_ABS, f"{where}: LSE max-abs {lse_max:.3e} > {LSE_MAX_ABS}"


def n_blocks(wl, tile=None):
    if wl.kind in ("topk", "sta", "spade"):
        bt, bh, bw = tile if tile is not None else wl.tile
        return math.ceil(wl.T / bt) * math.ceil(wl.H / bh) * math.ceil(wl.W / bw)
    return math.ceil(wl.N / wl.block)
