"""GPU parity of the SVG online head profiler (Sparse VideoGen review, key
machinery) against the CPU oracle, through the C ABI.

Compared per head: the mean squared errors of the spatial and temporal
outputs against the full output (relative 5 %: the GPU's P is bf16 on the
tensor cores), the per-row errors, and the decision, which must agree unless
the oracle's two errors are within 10 % of each other. Where one pattern keeps
every key it is full attention again, computed by the masked-pass kernel
while the full pass runs on the tcgen05 attention kernel: its error is
rounding only, below 1e-3 of the other pattern's.
"""
import numpy as np
import pytest
import torch

from oracle import profile
from synthetic import CONFIGS, Workload, bf16_bits_to_f32, make_qkv, sample_rows
from tests import _cases as C

pytestmark = pytest.mark.gpu


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _run(wl, rows, sink_tokens, frame_radius=1, block=128):
    from sparse_attention_video_b200 import profile_heads
    x = make_qkv(wl)
    q, k, v = (_dev(x[n]) for n in "qkv")
    rows_d = torch.from_numpy(rows).cuda()
    is_t, mse, row_err = profile_heads(q, k, v, rows_d, wl.T, wl.H, wl.W, block=block,
                                       sink_tokens=sink_tokens, frame_radius=frame_radius)
    torch.cuda.synchronize()
    return x, is_t.cpu().numpy(), mse.cpu().numpy(), row_err.cpu().numpy()


def _check_heads(wl, x, rows, is_t, mse, row_err, sink_tokens, heads, block=128):
    for h in heads:
        qf, kf, vf = (bf16_bits_to_f32(x[n][0, h]) for n in "qkv")
        ref = profile.profile_head(qf, kf, vf, rows[h], wl.T, wl.H, wl.W, block, sink_tokens)
        got = (float(mse[h, 0]), float(mse[h, 1]))
        want = (ref["mse_spatial"], ref["mse_temporal"])
        for g_, w_ in zip(got, want):
            assert abs(g_ - w_) <= 0.05 * w_ + 1e-7, (h, got, want)
        d = wl.head_dim
        re_s = ((ref["o_spatial"] - ref["o_full"]) ** 2).sum(axis=1)
        re_t = ((ref["o_temporal"] - ref["o_full"]) ** 2).sum(axis=1)
        np.testing.assert_allclose(row_err[h, :, 0], re_s, rtol=0.1, atol=0.02 * re_s.max() + 1e-6)
        np.testing.assert_allclose(row_err[h, :, 1], re_t, rtol=0.1, atol=0.02 * re_t.max() + 1e-6)
        near_tie = abs(want[0] - want[1]) <= 0.1 * max(want)
        if not near_tie:
            assert bool(is_t[h]) == ref["temporal"], (h, got, want)
        assert abs(np.mean(row_err[h, :, 0]) / d - got[0]) <= 1e-5 * max(got[0], 1e-12) + 1e-9


def test_profile_small_grid_matches_oracle():
    wl = C.SMALL["spatiotemporal_ragged"]           # 6 x 12 x 20, 4 heads, d 128, 226 sinks
    rows = sample_rows(wl.N, wl.heads, fraction=0.1, seed=11)
    x, is_t, mse, row_err = _run(wl, rows, wl.sink_tokens)
    _check_heads(wl, x, rows, is_t, mse, row_err, wl.sink_tokens, range(wl.heads))


def test_profile_ragged_rows_and_head_dim_64():
    # 37 rows (not a multiple of a warp's 16), head_dim 64, no sinks
    wl = Workload(name="profile_d64", config_id=120, T=5, H=8, W=16, heads=2, head_dim=64,
                  kind="spatiotemporal", block=64, sink_tokens=0, temporal_heads=(1,))
    rows = np.ascontiguousarray(sample_rows(wl.N, wl.heads, fraction=0.1, seed=3)[:, :37])
    x, is_t, mse, row_err = _run(wl, rows, 0, block=64)
    _check_heads(wl, x, rows, is_t, mse, row_err, 0, range(wl.heads), block=64)


def test_profile_exact_patterns():
    # one frame: the spatial pattern is every key -> spatial error at rounding level
    wl = Workload(name="profile_one_frame", config_id=121, T=1, H=16, W=24, heads=2,
                  head_dim=64, kind="spatiotemporal", block=64, sink_tokens=0)
    rows = sample_rows(wl.N, wl.heads, fraction=0.2, seed=5)
    _, is_t, mse, row_err = _run(wl, rows, 0, block=64)
    assert np.all(mse[:, 0] <= 1e-3 * mse[:, 1])
    assert np.all(row_err[:, :, 0] <= 1e-3 * row_err[:, :, 1].mean(axis=1, keepdims=True) + 1e-9)
    assert np.all(is_t == 0)
    # one position per frame: the temporal pattern is every key -> temporal
    # error at rounding level
    wl = Workload(name="profile_one_position", config_id=122, T=256, H=1, W=1, heads=2,
                  head_dim=64, kind="spatiotemporal", block=64, sink_tokens=0)
    rows = sample_rows(wl.N, wl.heads, fraction=0.25, seed=6)
    _, is_t, mse, row_err = _run(wl, rows, 0, block=64)
    assert np.all(mse[:, 1] <= 1e-3 * mse[:, 0])
    assert np.all(row_err[:, :, 1] <= 1e-3 * row_err[:, :, 0].mean(axis=1, keepdims=True) + 1e-9)
    assert np.all(mse[:, 0] > 0.0) and np.all(is_t == 1)


def test_profile_full_size_sampled():
    # the 115,200-token grid, two heads, 64 sampled rows each
    wl = CONFIGS["spatiotemporal_hunyuan_720p"]
    wl2 = wl.with_(heads=2, temporal_heads=(1,))
    rows = np.ascontiguousarray(sample_rows(wl2.N, wl2.heads, fraction=0.01, seed=9)[:, ::18][:, :64])
    x, is_t, mse, row_err = _run(wl2, rows, wl2.sink_tokens)
    _check_heads(wl2, x, rows, is_t, mse, row_err, wl2.sink_tokens, range(wl2.heads))


def _run_search(wl, rows, cands):
    from sparse_attention_video_b200 import sta_window_search
    x = make_qkv(wl)
    q, k, v = (_dev(x[n]) for n in "qkv")
    choice, mse, row_err = sta_window_search(q, k, v, torch.from_numpy(rows).cuda(), wl.T, wl.H,
                                             wl.W, wl.tile, cands, block=wl.block)
    torch.cuda.synchronize()
    return x, choice.cpu().numpy(), mse.cpu().numpy(), row_err.cpu().numpy()


def test_sta_window_search_matches_oracle():
    # Sliding Tile Attention review, Algorithm 1: per head, the candidate
    # window whose output is closest (MSE) to full attention
    wl = C.SMALL["sta_ragged"]                      # 9 x 10 x 19, tiles 4 x 4 x 8, 3 heads
    cands = [(1, 1, 1), (3, 3, 3), (1, 3, 5), (3, 1, 1)]
    rows = sample_rows(wl.N, wl.heads, fraction=0.1, seed=13)
    x, choice, mse, row_err = _run_search(wl, rows, cands)
    for h in range(wl.heads):
        qf, kf, vf = (bf16_bits_to_f32(x[n][0, h]) for n in "qkv")
        ref = profile.sta_window_search(qf, kf, vf, rows[h], wl.T, wl.H, wl.W, wl.tile, cands)
        for c in range(len(cands)):
            assert abs(mse[h, c] - ref["mse"][c]) <= 0.05 * ref["mse"][c] + 1e-7, (h, c, mse[h], ref["mse"])
            re = ((ref["o"][c] - ref["o_full"]) ** 2).sum(axis=1)
            np.testing.assert_allclose(row_err[h, :, c], re, rtol=0.1, atol=0.02 * re.max() + 1e-6)
        srt = sorted(ref["mse"])
        if srt[1] - srt[0] > 0.1 * srt[1]:
            assert choice[h] == ref["choice"], (h, mse[h], ref["mse"])


def test_sta_window_search_full_grid_candidate_wins():
    # a window that spans the tile grid (3 x 3 x 3 tiles) keeps every key; it
    # visits them in tile order, so its bf16 P rounds differently from the
    # full pass (order of the online softmax), not to zero error
    wl = C.SMALL["sta_ragged"]
    cands = [(3, 3, 3), (5, 5, 5), (1, 1, 1)]
    rows = sample_rows(wl.N, wl.heads, fraction=0.1, seed=14)
    _, choice, mse, _ = _run_search(wl, rows, cands)
    assert np.all(mse[:, 1] < 1e-5 * np.minimum(mse[:, 0], mse[:, 2]))
    assert np.all(choice == 1)
