"""Pins for the SVG head profiler oracle (Sparse VideoGen review, key
machinery): cases whose answer is fixed by the definition of the patterns."""
import numpy as np
import pytest

from oracle import profile
from synthetic import sample_rows

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _qkv(n, d, seed):
    g = np.random.default_rng(seed)
    return [g.standard_normal((n, d)).astype(np.float32) for _ in range(3)]


def test_single_frame_spatial_pattern_is_full_attention():
    # T = 1: every key is in the query's frame, so the spatial output is the
    # full output and its error is exactly zero.
    T, H, W, d = 1, 16, 16, 32
    q, k, v = _qkv(T * H * W, d, 0)
    rows = np.array([0, 17, 100, 255])
    keep = profile.pattern_keep(rows, T, H, W, 128, 0, 1, temporal=False)
    assert keep.all()
    r = profile.profile_head(q, k, v, rows, T, H, W, 128, 0)
    assert r["mse_spatial"] == 0.0 and r["mse_temporal"] > 0.0
    assert r["temporal"] is False


def test_single_position_temporal_pattern_is_full_attention():
    # H = W = 1: every token sits at the same spatial position, so the temporal
    # output is the full output, while the spatial pattern (16-frame blocks)
    # sees the query's block and its neighbours only.
    T, H, W, d = 256, 1, 1, 32
    q, k, v = _qkv(T, d, 1)
    rows = np.array([5, 64, 200])
    assert profile.pattern_keep(rows, T, H, W, 16, 0, 1, temporal=True).all()
    assert not profile.pattern_keep(rows, T, H, W, 16, 0, 1, temporal=False).all()
    r = profile.profile_head(q, k, v, rows, T, H, W, 16, 0)
    assert r["mse_temporal"] == 0.0 and r["mse_spatial"] > 0.0
    assert r["temporal"] is True


def test_constant_values_tie_goes_to_spatial():
    T, H, W, d = 4, 8, 8, 16
    q, k, _ = _qkv(T * H * W, d, 2)
    v = np.ones((T * H * W, d), np.float32) * 0.75
    r = profile.profile_head(q, k, v, np.array([3, 70, 200]), T, H, W, 64, 0)
    np.testing.assert_allclose(r["o_spatial"], 0.75)
    np.testing.assert_allclose(r["o_temporal"], 0.75)
    assert r["mse_spatial"] < 1e-28 and r["mse_temporal"] < 1e-28
    if r["mse_spatial"] == r["mse_temporal"]:
        assert r["temporal"] is False


def test_patterns_match_their_plain_definitions_at_unit_granularity():
    # One frame per identity block and radius 0: the spatial keys are the
    # query's own frame; one position per frame-major block: the temporal
    # keys are the query's own (h, w). Plus the sink tokens in both.
    T, H, W = 6, 4, 4                        # H*W = 16 tokens per frame
    n, sinks = T * H * W, 16
    rows = np.array([0, 21, 47, 50, 95])
    ks = profile.pattern_keep(rows, T, H, W, H * W, sinks, 0, temporal=False)
    kt = profile.pattern_keep(rows, T, H, W, T, sinks, 0, temporal=True)
    tok = np.arange(n)
    frame, pos = tok // (H * W), tok % (H * W)
    # sinks: the first 16 slots of each working layout, rounded up to whole
    # blocks (16 tokens = frame 0 in identity order; 18 slots = positions 0-2
    # in frame-major order, slot = pos * T + frame)
    for r, t in enumerate(rows):
        want_s = (frame == frame[t]) | (tok < sinks)
        np.testing.assert_array_equal(ks[r], want_s)
        sink_t = (pos * T + frame) < -(-sinks // T) * T
        want_t = (pos == pos[t]) | sink_t
        np.testing.assert_array_equal(kt[r], want_t)


def test_sample_rows_are_distinct_sorted_and_seeded():
    a = sample_rows(115200, 3, 0.01, seed=7)
    assert a.shape == (3, 1152)
    for h in range(3):
        assert np.all(np.diff(a[h]) > 0) and a[h].min() >= 0 and a[h].max() < 115200
    np.testing.assert_array_equal(a, sample_rows(115200, 3, 0.01, seed=7))
    assert not np.array_equal(a[0], a[1])


def test_window_covering_the_grid_is_full_attention_and_wins():
    # Sliding Tile Attention review, Algorithm 1: a window that spans the
    # whole tile grid keeps every key, so its error is exactly zero.
    T, H, W, d = 4, 8, 16, 16
    tile = (2, 4, 8)                                      # tile grid 2 x 2 x 2
    q, k, v = _qkv(T * H * W, d, 8)
    rows = np.array([1, 77, 300, 511])
    cands = [(1, 1, 1), (3, 3, 3), (1, 3, 1)]
    assert profile.window_keep(rows, T, H, W, tile, (3, 3, 3)).all()
    r = profile.sta_window_search(q, k, v, rows, T, H, W, tile, cands)
    assert r["mse"][1] == 0.0 and r["mse"][0] > 0.0 and r["choice"] == 1


def test_window_keep_matches_its_plain_definition():
    # unit tiles (1, 1, 1) would make blocks of one token; with tiles of one
    # frame row (1, 1, W) the kept keys of a query at (t, h, w) under window
    # (wt, wh, 1) are the tokens with |dt| <= wt//2 and |dh| <= wh//2
    T, H, W = 5, 6, 8
    tile = (1, 1, W)
    rows = np.array([0, 13, 100, 239])
    keep = profile.window_keep(rows, T, H, W, tile, (3, 1, 1))
    tok = np.arange(T * H * W)
    t, h = tok // (H * W), (tok // W) % H
    for r, q_tok in enumerate(rows):
        want = (np.abs(t - t[q_tok]) <= 1) & (h == h[q_tok])
        np.testing.assert_array_equal(keep[r], want)


def test_per_head_windows_equal_single_window_masks():
    from oracle import pipeline
    from synthetic import CONFIGS, Workload, make_qkv, bf16_bits_to_f32
    base = Workload(name="hw", config_id=130, T=4, H=8, W=16, heads=2, head_dim=32, kind="sta",
                    tile=(2, 4, 8), block=64, window=(3, 3, 3))
    per_head = base.with_(head_windows=((1, 1, 1), (1, 3, 3)))
    x = make_qkv(base)
    for h, win in enumerate(per_head.head_windows):
        qf, kf = (bf16_bits_to_f32(x[n][0, h]) for n in "qk")
        a = pipeline.head_mask(per_head, qf, kf, h)["bmask"]
        b = pipeline.head_mask(base.with_(window=win), qf, kf, h)["bmask"]
        np.testing.assert_array_equal(a, b)
