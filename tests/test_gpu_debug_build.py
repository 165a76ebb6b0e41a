"""The index-checking debug build (libsparse_attn_debug.so) on a B200.

The debug library is the same sources compiled with SA_DEBUG_CHECKS: indices
that come from data (the mask's key-block lists as the select kernel writes
them, the attention's output rows from the slot maps, the FG union lists'
keys before their K/V rows are copied) are tested against their buffers
before use, and a failure sets the bounds flag of the status word. On every
policy kind, ragged grids and both head dims, the debug library must report
a clean status word and give exactly the release library's mask and outputs.
"""
import os

import numpy as np
import pytest
import torch

from synthetic import Workload, make_qkv
from tests import _cases as C

pytestmark = pytest.mark.gpu

FG_CASE = Workload(name="fg_debug", config_id=116, T=6, H=12, W=20, heads=2, head_dim=128,
                   kind="fg", fg_group=64, fg_keep_fraction=0.15)
CASES = ["topk_ragged_d128", "sta_d64", "spatiotemporal_ragged", "spade_ragged",
         "tiny_topk", "sta_head_windows"]


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _run(wl):
    from sparse_attention_video_b200 import (SA_EXPORT_BLOCK_BITS, SA_EXPORT_FG_BITS,
                                             SparseAttention, make_policy)
    x = make_qkv(wl)
    q, k, v = (_dev(x[n]) for n in "qkv")
    sa = SparseAttention(wl.batch, wl.heads, wl.T, wl.H, wl.W, wl.head_dim,
                         make_policy(**C.policy_kwargs(wl)))
    o, lse = sa(q, k, v)
    torch.cuda.synchronize()
    bits = sa.export(SA_EXPORT_FG_BITS if wl.kind == "fg" else SA_EXPORT_BLOCK_BITS)
    return sa.status(), o.cpu(), lse.cpu(), bits


@pytest.fixture(scope="module")
def debug_lib():
    import sparse_attention_video_b200._native as N
    from sparse_attention_video_b200 import build as B
    if not os.path.exists(B.LIB_DEBUG):
        B.build(debug=True)                 # nvcc is on every machine the suite runs on
    release = (N.lib(), N.LIB_PATH)
    yield N, B.LIB_DEBUG
    N._LIB, N.LIB_PATH = release


@pytest.mark.parametrize("name", CASES + ["fg"])
def test_debug_build_matches_release_with_clean_status(debug_lib, name):
    N, debug_path = debug_lib
    wl = FG_CASE if name == "fg" else C.SMALL[name]
    release_lib, release_path = N.lib(), N.LIB_PATH
    st_r, o_r, lse_r, bits_r = _run(wl)
    try:
        N._LIB, N.LIB_PATH = None, debug_path
        N.lib()
        st_d, o_d, lse_d, bits_d = _run(wl)
    finally:
        N._LIB, N.LIB_PATH = release_lib, release_path
    assert st_r == 0 and st_d == 0, (st_r, st_d)
    np.testing.assert_array_equal(bits_d, bits_r)
    assert torch.equal(o_d.view(torch.int16), o_r.view(torch.int16))
    assert torch.equal(lse_d, lse_r)
