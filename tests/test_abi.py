"""The C ABI on a machine without a GPU: the library loads, exports every
symbol include/sparse_attn.h declares, sizes workspaces and rejects bad
arguments on the host before touching the device."""
import ctypes
import math
import os
import re

import numpy as np
import pytest

from sparse_attention_video_b200 import _native as N
from sparse_attention_video_b200 import make_policy
from synthetic import CONFIGS
from tests import _cases as C

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "sparse_attn.h")


def _declared():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"SA_API\s+(?:const\s+)?\w+\*?\s+\**(sparse_attn_\w+)\s*\(", txt)))


def test_header_declares_the_exported_api():
    assert _declared() == sorted(N.EXPORTED)


def test_library_exports_every_declared_symbol():
    L = N.lib()
    for name in _declared():
        assert hasattr(L, name), name


def test_struct_sizes_match_header_layout():
    # sa_problem: 6 ints; sa_head_info: 10 int32 + 4 float + 2 int32
    assert ctypes.sizeof(N.Problem) == 24
    assert ctypes.sizeof(N.HeadInfo) == 64


@pytest.mark.parametrize("name", list(CONFIGS))
def test_workspace_sizes_for_every_workload(name):
    wl = CONFIGS[name]
    pol = make_policy(**C.policy_kwargs(wl))
    m, s = N.workspace_size(N.Problem(wl.batch, wl.heads, wl.T, wl.H, wl.W, wl.head_dim), pol)
    assert m > 0 and s >= 256
    assert m % 256 == 0 and s % 256 == 0


def test_mask_workspace_holds_bits_and_lists():
    wl = CONFIGS["sta_wan21_1p3b_480p"]
    pol = make_policy(**C.policy_kwargs(wl))
    pr = N.Problem(1, wl.heads, wl.T, wl.H, wl.W, wl.head_dim)
    m, _ = N.workspace_size(pr, pol)
    nb = 336
    assert m >= wl.heads * nb * nb * 4                   # ascending key-block lists
    assert N.export_bytes(pr, pol, N.SA_EXPORT_BLOCK_BITS) == wl.heads * nb * ((nb + 31) // 32) * 4
    assert N.export_bytes(pr, pol, N.SA_EXPORT_HEAD_INFO) == wl.heads * 64


def test_invalid_arguments_are_rejected_on_the_host():
    L = N.lib()
    wl = CONFIGS["sta_wan21_1p3b_480p"]
    pol = make_policy(**C.policy_kwargs(wl))
    m, s = ctypes.c_size_t(), ctypes.c_size_t()
    bad_dim = N.Problem(1, 12, 21, 30, 52, 96)
    assert L.sparse_attn_workspace_size(ctypes.byref(bad_dim), ctypes.byref(pol), ctypes.byref(m),
                                        ctypes.byref(s)) == N.SA_ERR_UNSUPPORTED
    zero = N.Problem(1, 0, 21, 30, 52, 128)
    assert L.sparse_attn_workspace_size(ctypes.byref(zero), ctypes.byref(pol), ctypes.byref(m),
                                        ctypes.byref(s)) == N.SA_ERR_INVALID_ARG
    pr = N.Problem(1, 12, 21, 30, 52, 128)
    even = make_policy("sta", tile=(4, 4, 8), window=(3, 2, 3))
    assert L.sparse_attn_workspace_size(ctypes.byref(pr), ctypes.byref(even), ctypes.byref(m),
                                        ctypes.byref(s)) == N.SA_ERR_INVALID_ARG
    wrong_tile = make_policy("sta", tile=(4, 4, 4), window=(3, 3, 3))  # 64 tokens != block 128
    assert L.sparse_attn_workspace_size(ctypes.byref(pr), ctypes.byref(wrong_tile), ctypes.byref(m),
                                        ctypes.byref(s)) == N.SA_ERR_INVALID_ARG
    # extents whose product overflows 32 bits are refused, not wrapped around
    for t in ((1 << 16, 1 << 16, 1), (1 << 11, 1 << 11, 1 << 11), (1, 1 << 30, 1 << 30)):
        huge = make_policy("sta", tile=t, window=(3, 3, 3))
        assert L.sparse_attn_workspace_size(ctypes.byref(pr), ctypes.byref(huge), ctypes.byref(m),
                                            ctypes.byref(s)) == N.SA_ERR_INVALID_ARG, t
    # null / misaligned device pointers never reach the device
    assert L.sparse_attn_forward(ctypes.byref(pr), ctypes.byref(pol), None, None, None, None, None,
                                 None, None, None) == N.SA_ERR_INVALID_ARG
    assert L.sparse_attn_build_mask(ctypes.byref(pr), ctypes.byref(pol), None, None, 0x1001, 0x2000,
                                    None) == N.SA_ERR_WORKSPACE
    # the host-buffer call: missing host or device buffers, an LSE on one
    # side only, a misaligned device buffer; nothing is copied or launched
    hb = (ctypes.c_char * 64)()
    h = ctypes.addressof(hb)
    fh = L.sparse_attn_forward_host
    assert fh(ctypes.byref(pr), ctypes.byref(pol), None, h, h, h, None, 0x1000, 0x2000, None,
              0x3000, 0x4000, None) == N.SA_ERR_INVALID_ARG
    assert fh(ctypes.byref(pr), ctypes.byref(pol), h, h, h, h, None, None, 0x2000, None,
              0x3000, 0x4000, None) == N.SA_ERR_INVALID_ARG
    assert fh(ctypes.byref(pr), ctypes.byref(pol), h, h, h, h, h, 0x1000, 0x2000, None,
              0x3000, 0x4000, None) == N.SA_ERR_INVALID_ARG
    assert fh(ctypes.byref(pr), ctypes.byref(pol), h, h, h, h, None, 0x1008, 0x2000, None,
              0x3000, 0x4000, None) == N.SA_ERR_INVALID_ARG
    st = make_policy("spatiotemporal", block=128)                     # head types missing
    assert L.sparse_attn_workspace_size(ctypes.byref(pr), ctypes.byref(st), ctypes.byref(m),
                                        ctypes.byref(s)) == N.SA_ERR_INVALID_ARG


def test_summarizer_and_profiler_arguments_are_checked_on_the_host():
    L = N.lib()
    m, s = ctypes.c_size_t(), ctypes.c_size_t()
    wl = CONFIGS["spade_wan21_14b_720p"]
    pr = N.Problem(1, wl.heads, wl.T, wl.H, wl.W, wl.head_dim)
    for good in ("mean", "max", "min"):
        pol = make_policy(**{**C.policy_kwargs(wl), "summarizer": good})
        assert L.sparse_attn_workspace_size(ctypes.byref(pr), ctypes.byref(pol), ctypes.byref(m),
                                            ctypes.byref(s)) == N.SA_OK
    bad = make_policy(**{**C.policy_kwargs(wl), "summarizer": 3})
    assert L.sparse_attn_workspace_size(ctypes.byref(pr), ctypes.byref(bad), ctypes.byref(m),
                                        ctypes.byref(s)) == N.SA_ERR_INVALID_ARG
    # the profiler: spatial/temporal policy only, 1 <= n_rows <= N, aligned device buffers
    st = CONFIGS["spatiotemporal_hunyuan_720p"]
    pr = N.Problem(1, st.heads, st.T, st.H, st.W, st.head_dim)
    ok_pol = make_policy("spatiotemporal", block=128, sink_tokens=226)
    args = (0x1000, 0x1000, 0x1000, 0x1000, 16, 0x1000, 0x1000, 0x1000, None, None)
    sta = make_policy("sta", tile=(4, 4, 8), window=(3, 3, 3))
    assert L.sparse_attn_profile_heads(ctypes.byref(pr), ctypes.byref(sta), *args) == N.SA_ERR_INVALID_ARG
    for n_rows in (0, st.T * st.H * st.W + 1):
        a = list(args)
        a[4] = n_rows
        assert L.sparse_attn_profile_heads(ctypes.byref(pr), ctypes.byref(ok_pol), *a) == N.SA_ERR_INVALID_ARG
    a = list(args)
    a[0] = 0x1008                                                     # q not 16-byte aligned
    assert L.sparse_attn_profile_heads(ctypes.byref(pr), ctypes.byref(ok_pol), *a) == N.SA_ERR_INVALID_ARG
    a = list(args)
    a[7] = None                                                       # no decision buffer
    assert L.sparse_attn_profile_heads(ctypes.byref(pr), ctypes.byref(ok_pol), *a) == N.SA_ERR_INVALID_ARG
    a = list(args)
    a[8] = 0x1010                                                     # scratch not 256-byte aligned
    assert L.sparse_attn_profile_heads(ctypes.byref(pr), ctypes.byref(ok_pol), *a) == N.SA_ERR_WORKSPACE
    # the scratch workspace is required (gathered rows and the full pass's O)
    assert L.sparse_attn_profile_heads(ctypes.byref(pr), ctypes.byref(ok_pol), *args) == N.SA_ERR_WORKSPACE
    n_rows = 1152
    bytes_ = N.profile_workspace_size(pr, n_rows)
    BH, d = st.heads, st.head_dim
    n_pad = (n_rows + 127) // 128 * 128
    up = lambda x: (x + 255) // 256 * 256
    assert bytes_ == up(up(256 + BH * n_pad * d * 2) + BH * n_rows * d * 4)
    for bad in (0, st.T * st.H * st.W + 1):
        with pytest.raises(N.SparseAttnError):
            N.profile_workspace_size(pr, bad)


def test_window_search_and_head_windows_are_checked_on_the_host():
    L = N.lib()
    m, s = ctypes.c_size_t(), ctypes.c_size_t()
    wl = CONFIGS["sta_wan21_1p3b_480p"]
    pr = N.Problem(1, wl.heads, wl.T, wl.H, wl.W, wl.head_dim)
    ok = make_policy(**{**C.policy_kwargs(wl), "head_windows": [(3, 3, 3)] * wl.heads})
    assert L.sparse_attn_workspace_size(ctypes.byref(pr), ctypes.byref(ok), ctypes.byref(m),
                                        ctypes.byref(s)) == N.SA_OK
    for bad_w in ((2, 3, 3), (3, 3, 0), (257, 1, 1)):
        bad = make_policy(**{**C.policy_kwargs(wl), "head_windows": [(3, 3, 3)] * (wl.heads - 1) + [bad_w]})
        assert L.sparse_attn_workspace_size(ctypes.byref(pr), ctypes.byref(bad), ctypes.byref(m),
                                            ctypes.byref(s)) == N.SA_ERR_INVALID_ARG, bad_w
    sta = make_policy("sta", tile=wl.tile, window=(1, 1, 1))
    cand = (ctypes.c_int * 6)(3, 3, 3, 1, 3, 5)
    args = [0x1000, 0x1000, 0x1000, 0x1000, 16, cand, 2, 0x1000, 0x1000, 0x1000, None, None]
    call = lambda pol, a: L.sparse_attn_sta_window_search(ctypes.byref(pr), ctypes.byref(pol), *a)
    st = make_policy("spatiotemporal", block=128)
    assert call(st, args) == N.SA_ERR_INVALID_ARG                  # STA policies only
    for i, val in ((6, 0), (6, 9), (4, 0), (5, None)):               # candidate count, rows, list
        a = list(args)
        a[i] = val
        assert call(sta, a) == N.SA_ERR_INVALID_ARG, (i, val)
    even = (ctypes.c_int * 6)(3, 3, 3, 1, 2, 5)
    a = list(args)
    a[5] = even
    assert call(sta, a) == N.SA_ERR_INVALID_ARG
    wrong_tile = make_policy("sta", tile=(4, 4, 4), window=(1, 1, 1))   # 64 tokens != block 128
    assert call(wrong_tile, args) == N.SA_ERR_INVALID_ARG


def test_strerror_covers_every_code():
    for code in range(7):
        assert N.strerror(code) and N.strerror(code) != "unknown status"
    assert N.strerror(99) == "unknown status"


def test_python_api_checks_tensors_before_any_native_call():
    # The kernels see bare pointers, so the Python layer must refuse a tensor
    # of the wrong kind, shape, dtype or device before anything is launched.
    # CPU tensors stand in for the misplaced ones: every call must raise here.
    import torch
    from sparse_attention_video_b200 import api, profile_heads, sta_window_search
    pr = N.Problem(1, 2, 3, 4, 8, 64)
    good = (1, 2, 96, 64)
    with pytest.raises(ValueError, match="CUDA"):
        api._check_qkv(torch.zeros(good, dtype=torch.bfloat16), pr, "q")
    with pytest.raises(ValueError, match="shape"):
        api._check_qkv(torch.zeros((1, 2, 95, 64), dtype=torch.bfloat16), pr, "out")
    with pytest.raises(ValueError, match="float32"):
        api._check_lse(torch.zeros((1, 2, 96), dtype=torch.float16), pr, None)
    with pytest.raises(ValueError, match="got list"):
        api._check_qkv([0.0], pr, "v")
    with pytest.raises(ValueError, match="scratch_ws"):
        api._check_scratch(torch.zeros(256, dtype=torch.uint8), torch.device("cpu"))
    q = torch.zeros(good, dtype=torch.bfloat16)
    rows = torch.zeros((2, 4), dtype=torch.int32)
    for fn, extra in ((profile_heads, ()), (sta_window_search, ((1, 1, 64), [(1, 1, 1)]))):
        with pytest.raises(ValueError):
            fn(q, q, q, rows, 3, 4, 8, *extra, block=64)
        with pytest.raises(ValueError, match="rows"):
            fn(q, q, q, rows[:1], 3, 4, 8, *extra, block=64)
        with pytest.raises(ValueError, match="q must be"):
            fn(q[0], q, q, rows, 3, 4, 8, *extra, block=64)


def test_explicit_bits_are_checked_against_the_mask_size():
    import torch
    from sparse_attention_video_b200 import SparseAttention, make_policy
    sa = SparseAttention.__new__(SparseAttention)      # no device workspaces on this host
    sa.problem = N.Problem(1, 2, 3, 4, 128, 64)
    sa.device = torch.device("cuda", 0)
    sa.policy = make_policy("explicit", block=128, explicit_layout=N.SA_LAYOUT_IDENTITY)
    with pytest.raises(ValueError, match="needs explicit_bits"):
        sa._check_explicit_bits()
    need = 2 * 12 * 1                                  # [heads][nb = 12 blocks][1 word]
    for bad in (torch.zeros(need, dtype=torch.int32),           # host memory
                torch.zeros(need, dtype=torch.float32)):        # not words
        sa.policy = make_policy("explicit", block=128, explicit_layout=N.SA_LAYOUT_IDENTITY,
                                explicit_bits=bad)
        assert N.export_bytes(sa.problem, sa.policy, N.SA_EXPORT_BLOCK_BITS) == 4 * need
        with pytest.raises(ValueError, match="explicit_bits must be"):
            sa._check_explicit_bits()


def test_quantize_and_cached_mask_arguments_are_checked_on_the_host():
    L = N.lib()
    vp = 0x1000                                        # aligned, never dereferenced
    for n_elems, n_tensors in ((12, 1), (0, 1), (64, 0), (64, 70000)):
        assert L.sparse_attn_quantize_e4m3(vp, n_elems, n_tensors, vp, vp, None) \
            == N.SA_ERR_INVALID_ARG, (n_elems, n_tensors)
    assert L.sparse_attn_quantize_e4m3(vp + 8, 64, 1, vp, vp, None) == N.SA_ERR_INVALID_ARG
    assert L.sparse_attn_quantize_e4m3(vp, 64, 1, None, vp, None) == N.SA_ERR_INVALID_ARG
    pr = N.Problem(1, 2, 3, 4, 64, 128)
    fg = make_policy("fg", fg_group=64, fg_keep_fraction=1.0)
    sta = make_policy("sta", tile=(1, 2, 64), window=(1, 1, 1))
    call = lambda pol, tau, lse=vp, ws=vp: L.sparse_attn_build_mask_fg_cached(
        ctypes.byref(pr), ctypes.byref(pol), vp, vp, lse, tau, ws, ws, None)
    assert call(sta, 0.0) == N.SA_ERR_INVALID_ARG             # FG policies only
    for tau in (-0.1, 1.0, float("nan")):
        assert call(fg, tau) == N.SA_ERR_INVALID_ARG, tau
    assert call(fg, 0.0, lse=None) == N.SA_ERR_INVALID_ARG
    assert call(fg, 0.0, ws=vp + 16) == N.SA_ERR_WORKSPACE


def test_policy_head_arrays_must_cover_the_problem():
    # the library reads one temporal flag and one window per head of the
    # problem from the policy's host arrays
    from sparse_attention_video_b200 import api, make_policy
    st = make_policy("spatiotemporal", temporal_heads=(1,), heads=2)
    api._check_head_arrays(st, 2)
    with pytest.raises(ValueError, match="temporal-head flags cover 2 heads"):
        api._check_head_arrays(st, 4)
    with pytest.raises(ValueError, match="outside"):
        make_policy("spatiotemporal", temporal_heads=(2,), heads=2)
    sta = make_policy("sta", tile=(4, 4, 8), window=(3, 3, 3), head_windows=[(1, 1, 1), (3, 3, 3)])
    api._check_head_arrays(sta, 2)
    with pytest.raises(ValueError, match="head_windows cover 2 heads"):
        api._check_head_arrays(sta, 3)
    with pytest.raises(ValueError, match="head_windows cover 0 heads"):
        api._check_head_arrays(make_policy("sta", tile=(4, 4, 8), head_windows=[]), 1)
    with pytest.raises(ValueError, match="each head window"):
        make_policy("sta", tile=(4, 4, 8), head_windows=[(3, 3)])
    api._check_head_arrays(make_policy("topk", tile=(4, 4, 8), topk=2), 8)   # no head arrays


def _layout_bytes(wl):
    """Mask and scratch bytes from the documented layout: regions in order,
    each padded to 256 bytes (the mask workspace is at least 256 bytes)."""
    up = lambda n: (n + 255) // 256 * 256
    BH, N_, d = wl.batch * wl.heads, wl.N, wl.head_dim
    cdiv = lambda a, b: -(-a // b)
    tiles = lambda t: cdiv(wl.T, t[0]) * cdiv(wl.H, t[1]) * cdiv(wl.W, t[2])
    if wl.kind in ("topk", "sta"):
        NB = tiles(wl.tile)
    elif wl.kind == "spade":
        NB = max(tiles(t) for t in wl.candidates)
    elif wl.kind == "fg":
        NB = 0
    else:
        NB = cdiv(N_, wl.block)
    W32 = cdiv(NB, 32)
    mask = [64 * BH, 4 * BH * NB, 4 * BH * NB * NB, 4 * BH * NB * W32]
    scratch = [256]
    if wl.kind == "spatiotemporal" and wl.temporal_heads:
        scratch.append(3 * up(BH * cdiv(N_, wl.block) * wl.block * d * 2))
    C = len(wl.candidates) if wl.kind == "spade" else (1 if wl.kind == "topk" else 0)
    if C:
        scratch += [4 * BH * C * NB * d, 4 * BH * C * NB * d, 4 * BH * C * NB, 4 * BH * NB * NB]
    if wl.kind == "fg":
        G, WN, P = cdiv(N_, wl.fg_group), cdiv(N_, 32), cdiv(N_, 128)
        cap = math.ceil(float(np.float32(wl.fg_keep_fraction)) * G * N_) + N_ + 32
        mask += [4 * BH * G * WN, 4 * BH, 4 * BH * P, 4 * BH * (P + 1), 4 * BH * cap]
        scratch += [3 * BH * cdiv(G, 128) * 128 * d * 2, 4 * BH * 4096, 4 * BH * 4,
                    8 * BH * 65536 + 24 * BH]
    return max(sum(up(b) for b in mask), 256), sum(up(b) for b in scratch)


@pytest.mark.parametrize("name", list(CONFIGS) + list(C.SMALL))
def test_workspace_sizes_equal_the_documented_layout(name):
    wl = CONFIGS[name] if name in CONFIGS else C.SMALL[name]
    pol = make_policy(**C.policy_kwargs(wl))
    got = N.workspace_size(N.Problem(wl.batch, wl.heads, wl.T, wl.H, wl.W, wl.head_dim), pol)
    assert got == _layout_bytes(wl), (name, got, _layout_bytes(wl))
