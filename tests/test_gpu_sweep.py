"""Small-case sweeps through the C ABI against the oracle (B200 only).

Seeded random tiny grids over every block mask kind, both head sizes, ragged
extents down to a single token and grids smaller than one tile; the
comparison is the block-sparse parity of test_gpu_block_sparse (masks bit
for bit outside the cut band, O and LSE within tolerance).
"""
import numpy as np
import pytest

from synthetic import Workload
from tests.test_gpu_block_sparse import run_block_case

pytestmark = pytest.mark.gpu

TILES = {128: [(1, 1, 128), (2, 8, 8), (4, 4, 8), (1, 8, 16), (8, 4, 4), (2, 4, 16)],
         64: [(1, 1, 64), (2, 4, 8), (4, 4, 4), (1, 8, 8)]}


def random_workload(seed):
    g = np.random.default_rng(seed)
    kind = ["topk", "sta", "spatiotemporal", "spade"][seed % 4]
    d = int(g.choice([64, 128]))
    block = 64 if (d == 64 and kind in ("topk", "sta") and g.random() < 0.5) else 128
    T, H, W = int(g.integers(1, 9)), int(g.integers(1, 13)), int(g.integers(1, 41))
    heads = int(g.integers(1, 4))
    odd = lambda: int(g.choice([1, 3, 5]))
    kw = dict(name=f"sweep_{seed}", config_id=2000 + seed, T=T, H=H, W=W, heads=heads,
              head_dim=d, kind=kind, block=block)
    tiles = TILES[block]
    if kind == "topk":
        kw.update(tile=tiles[int(g.integers(len(tiles)))], topk=int(g.integers(1, 5)),
                  keep_diagonal=bool(g.random() < 0.5))
    elif kind == "sta":
        kw.update(tile=tiles[int(g.integers(len(tiles)))], window=(odd(), odd(), odd()))
    elif kind == "spatiotemporal":
        kw.update(sink_tokens=int(g.integers(0, 300)),
                  temporal_heads=tuple(h for h in range(heads) if g.random() < 0.5))
    else:
        pick = g.choice(len(TILES[128]), size=int(g.integers(1, 4)), replace=False)
        kw.update(candidates=tuple(TILES[128][i] for i in sorted(pick)),
                  top_p=float(g.uniform(0.5, 0.95)), window=(odd(), odd(), odd()))
    return Workload(**kw)


@pytest.mark.parametrize("seed", range(24))
def test_random_tiny_grid(seed):
    run_block_case(random_workload(seed))


@pytest.mark.parametrize("T,H,W,kind", [
    (1, 1, 1, "sta"), (1, 1, 1, "spatiotemporal"), (1, 1, 1, "topk"),
    (2, 3, 7, "spade"), (1, 1, 128, "topk"), (1, 1, 127, "spatiotemporal"),
])
def test_single_tile_grid(T, H, W, kind):
    kw = dict(name=f"one_tile_{T}x{H}x{W}_{kind}", config_id=2100 + T * 1000 + H * 100 + W,
              T=T, H=H, W=W, heads=2, head_dim=128, kind=kind, block=128)
    if kind == "topk":
        kw.update(tile=(1, 1, 128), topk=1, keep_diagonal=True)
    elif kind == "sta":
        kw.update(tile=(2, 8, 8), window=(1, 1, 1))
    elif kind == "spatiotemporal":
        kw.update(sink_tokens=16, temporal_heads=(1,))
    else:
        kw.update(candidates=((1, 8, 16), (2, 8, 8)), top_p=0.9, window=(3, 3, 3))
    run_block_case(Workload(**kw))
