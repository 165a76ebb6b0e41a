"""The five workloads, described by shape and mask policy.

Shapes follow the latent grids of the video DiTs the pages evaluate on:
Wan 2.1 1.3B at 480p (21x30x52), HunyuanVideo at 720p (30x48x80) and Wan 2.1
14B at 720p (21x45x80), plus a tiny grid small enough for brute force.

Mask kinds:
  "topk"     keep the diagonal block plus the Top-K key blocks by mean-pooled
             q.k score (SPADE review, "Core claim": head-wise Top-K/Top-P).
  "sta"      sliding tile window of neighbouring 3D tiles (Sliding Tile
             Attention review, key machinery).
  "spatiotemporal"  spatial heads keep their own frame +-1, temporal heads keep
             the same (h,w) positions across frames in a frame-major layout,
             plus sink tokens (Sparse VideoGen review, key machinery and
             core discovery).
  "spade"    per-head choice of 3D blocking by SICS, then Top-P of softmaxed
             pooled scores plus a local tile window (SPADE review, "What
             carries the argument", Eqs. 3-5).
  "fg"       M x 1 key slices: groups of M contiguous queries keep the keys
             whose score against the group's mean query passes a per-head
             threshold (FG-Attn review, skeptic critique on Sec. 4.4). With
             fg_rule "cached", the groups instead keep every key that one of
             their queries gives a full-attention probability above 0.5/N
             (FG-Attn review, the cached strategy).
"""
from dataclasses import dataclass, field
from typing import Optional, Tuple


@dataclass(frozen=True)
class Workload:
    name: str
    config_id: int
    T: int
    H: int
    W: int
    heads: int
    head_dim: int
    batch: int = 1
    kind: str = "topk"
    tile: Tuple[int, int, int] = (1, 1, 128)        # (bt, bh, bw) of the working layout
    topk: int = 0
    keep_diagonal: bool = False
    window: Tuple[int, int, int] = (0, 0, 0)       # (win_t, win_h, win_w) in tiles, odd
    sink_tokens: int = 0
    temporal_heads: Tuple[int, ...] = ()           # spatiotemporal: which heads are temporal
    candidates: Tuple[Tuple[int, int, int], ...] = ()
    top_p: float = 0.0
    fg_group: int = 0
    fg_keep_fraction: float = 0.0
    fg_rule: str = "pooled"                        # fg: "pooled" (q_avg scores) or "cached" (full map)
    block: int = 128                               # tokens per block in the working layout
    summarizer: str = "mean"                       # topk, spade: block summary ("mean", "max", "min")
    head_windows: Tuple[Tuple[int, int, int], ...] = ()   # sta: a window per head (empty: window)

    @property
    def N(self) -> int:
        return self.T * self.H * self.W

    def with_(self, **kw) -> "Workload":
        d = dict(self.__dict__)
        d.update(kw)
        return Workload(**d)


CONFIGS = {
    "tiny_topk": Workload(
        name="tiny_topk", config_id=1, T=4, H=8, W=8, heads=2, head_dim=64,
        kind="topk", tile=(2, 4, 8), block=64, topk=2, keep_diagonal=True),
    "sta_wan21_1p3b_480p": Workload(
        name="sta_wan21_1p3b_480p", config_id=2, T=21, H=30, W=52, heads=12, head_dim=128,
        kind="sta", tile=(4, 4, 8), block=128, window=(3, 3, 3)),
    "spatiotemporal_hunyuan_720p": Workload(
        name="spatiotemporal_hunyuan_720p", config_id=3, T=30, H=48, W=80, heads=24,
        head_dim=128, kind="spatiotemporal", block=128, sink_tokens=226,
        temporal_heads=tuple(range(12, 24))),
    "spade_wan21_14b_720p": Workload(
        name="spade_wan21_14b_720p", config_id=4, T=21, H=45, W=80, heads=40, head_dim=128,
        kind="spade", block=128, candidates=((1, 8, 16), (8, 4, 4), (2, 8, 8)),
        top_p=0.9, window=(3, 3, 3)),
    "fg_slices_hunyuan_720p": Workload(
        name="fg_slices_hunyuan_720p", config_id=5, T=30, H=48, W=80, heads=24, head_dim=128,
        kind="fg", block=128, fg_group=64, fg_keep_fraction=0.15),
}


def get_config(name: str) -> Workload:
    return CONFIGS[name]
