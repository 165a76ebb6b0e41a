"""Host-side logic that needs no GPU: which attention kernel the bench names
for each policy (it must be the one the library launches for it), the
launch count taken from a profiler result, and the argument checks of the
host-buffer call (they run before the library is reached)."""
import pytest
import torch

import bench
from synthetic import CONFIGS


def test_bench_names_the_kernel_each_policy_launches():
    # the library runs Top-K, tile-window and frame-window policies on the
    # one-warpgroup kernel, Top-P and explicit masks on the two-group kernel,
    # FG slices on its gather mode
    expect = {"topk": "attn_solo_kernel", "sta": "attn_solo_kernel",
              "spatiotemporal": "attn_solo_kernel", "spade": "attn_fwd_kernel",
              "fg": "attn_fwd_kernel"}
    for wl in CONFIGS.values():
        name = bench.attn_kernel_name(wl)
        assert name.startswith(expect[wl.kind] + "<%d,%d" % (wl.head_dim, wl.block)), (wl.name, name)
        assert ("gather" in name) == (wl.kind == "fg")


def test_launch_count_skips_copies_and_memsets():
    times = {"sa::attn_solo_kernel<128, 128>": (3, 1.0), "Memset (Device)": (2, 0.1),
             "Memcpy HtoD (Pinned -> Device)": (3, 2.0), "sa::select_kernel": (3, 0.2)}
    assert bench.launches_in(times) == 6
    assert bench.launches_in({}) == 0


def test_host_buffer_checks():
    from sparse_attention_video_b200.api import _check_host
    shape = (1, 2, 256, 64)
    _check_host(torch.empty(shape, dtype=torch.bfloat16), shape, torch.bfloat16, "q")
    with pytest.raises(ValueError):
        _check_host(torch.empty(shape, dtype=torch.float32), shape, torch.bfloat16, "q")
    with pytest.raises(ValueError):
        _check_host(torch.empty((1, 2, 255, 64), dtype=torch.bfloat16), shape, torch.bfloat16, "q")
    with pytest.raises(ValueError):
        _check_host(torch.empty((1, 2, 64, 256), dtype=torch.bfloat16).transpose(2, 3), shape,
                    torch.bfloat16, "q")
    with pytest.raises(ValueError):
        _check_host(None, shape, torch.bfloat16, "q")
