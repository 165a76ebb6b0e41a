"""The no-allocation mask build (sparse_attn_build_mask_static) on a B200.

Some callers cannot allocate device memory when they build a mask (framework
execute callbacks, latency paths where cudaMalloc may synchronize, processes
with a fixed memory reservation). For them the library takes its scratch from
a static device array. This test calls that entry point through the C ABI and
checks, on two calls in a row with different inputs, that its mask equals the
one sparse_attn_build_mask writes with a caller-owned scratch workspace
(bit-exact bit rows, identical per-head geometry and SICS totals) and that
attention over either mask gives the same output within the parity
tolerances. It also checks that a problem too large for the static array is
rejected before anything runs, and that the device status word of the
static build (sparse_attn_status_static) reports no error after each call.
A fine-grained key-slice case runs the same comparison on the slice bits,
the per-head threshold and the union key lists.

This file is collected last so that a run stopping at the first failure has
already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from synthetic import bf16_bits_to_f32, make_qkv
from tests import _cases as C

pytestmark = pytest.mark.gpu


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _export(N, problem, policy, mask_ws, what):
    nbytes = N.export_bytes(problem, policy, what)
    if what == N.SA_EXPORT_HEAD_INFO:
        buf = (N.HeadInfo * (nbytes // ctypes.sizeof(N.HeadInfo)))()
        N.mask_export(problem, policy, mask_ws.data_ptr(), what, ctypes.addressof(buf), nbytes)
        return [bytes(h) for h in buf]
    arr = np.empty(nbytes // 4, dtype=np.uint32)
    N.mask_export(problem, policy, mask_ws.data_ptr(), what, arr.ctypes.data, nbytes)
    return arr


@pytest.mark.parametrize("name", ["tiny_topk", "spade_ragged"])
def test_static_scratch_mask_matches_caller_scratch_mask(name):
    from sparse_attention_video_b200 import SparseAttention, _native as N, make_policy
    base = C.SMALL[name]
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):                      # two calls in a row, different inputs
        wl = base.with_(config_id=base.config_id + 500 + call)
        x = make_qkv(wl)
        q, k, v = (_dev(x[n]) for n in "qkv")
        policy = make_policy(**C.policy_kwargs(wl))
        sa = SparseAttention(wl.batch, wl.heads, wl.T, wl.H, wl.W, wl.head_dim, policy)
        assert sa.scratch_bytes <= N.SA_STATIC_SCRATCH_BYTES
        sa.build_mask(q, k)                    # existing entry point, caller scratch
        mask_static = torch.empty(sa.mask_bytes, dtype=torch.uint8, device="cuda")
        N.build_mask_static(sa.problem, policy, q.data_ptr(), k.data_ptr(),
                            mask_static.data_ptr(), stream)
        torch.cuda.synchronize()
        assert N.status_static(stream) == N.SA_OK, f"call {call}: static build status"
        assert sa.status() == N.SA_OK, f"call {call}: caller-scratch build status"
        info_a = _export(N, sa.problem, policy, sa.mask_ws, N.SA_EXPORT_HEAD_INFO)
        info_b = _export(N, sa.problem, policy, mask_static, N.SA_EXPORT_HEAD_INFO)
        assert info_a == info_b, f"call {call}: per-head info differs"
        # bit rows a head actually has (rows past its block count are not written)
        nbs = [N.HeadInfo.from_buffer_copy(h).nb for h in info_a]
        NB = max(C.n_blocks(wl, t) for t in (wl.candidates or [None]))
        bits_a = _export(N, sa.problem, policy, sa.mask_ws, N.SA_EXPORT_BLOCK_BITS)
        bits_b = _export(N, sa.problem, policy, mask_static, N.SA_EXPORT_BLOCK_BITS)
        bits_a = bits_a.reshape(len(nbs), NB, -1)
        bits_b = bits_b.reshape(len(nbs), NB, -1)
        for bh, nb in enumerate(nbs):
            np.testing.assert_array_equal(bits_a[bh, :nb], bits_b[bh, :nb],
                                          err_msg=f"call {call}, head {bh}: bit rows differ")
        o1, l1 = sa.forward(q, k, v)
        o2 = torch.empty_like(q)
        l2 = torch.empty_like(l1)
        N.forward(sa.problem, policy, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                  mask_static.data_ptr(), sa.scratch_ws.data_ptr(), o2.data_ptr(),
                  l2.data_ptr(), stream)
        torch.cuda.synchronize()
        to_np = lambda t: bf16_bits_to_f32(t.view(torch.int16).cpu().numpy().view(np.uint16))
        e = C.attention_errors(to_np(o2), l2.cpu().numpy(), to_np(o1).astype(np.float64),
                               l1.cpu().numpy().astype(np.float64))
        C.check_errors(*e, where=f"{name} call {call}")


def test_static_scratch_rejects_problems_beyond_its_size():
    from sparse_attention_video_b200 import _native as N, make_policy
    from synthetic import CONFIGS
    wl = CONFIGS["spade_wan21_14b_720p"]       # needs far more than the static array
    policy = make_policy(**C.policy_kwargs(wl))
    problem = N.Problem(1, wl.heads, wl.T, wl.H, wl.W, wl.head_dim)
    _, scratch = N.workspace_size(problem, policy)
    assert scratch > N.SA_STATIC_SCRATCH_BYTES
    mask = torch.empty(256, dtype=torch.uint8, device="cuda")
    rc = N.lib().sparse_attn_build_mask_static(ctypes.byref(problem), ctypes.byref(policy),
                                               None, None, mask.data_ptr(), None)
    assert rc == N.SA_ERR_UNSUPPORTED


def test_static_scratch_fg_slices_match_caller_scratch():
    """The FG slice build through the static array: its scratch holds the
    split group-mean operands behind the scoring tensor maps, the threshold
    histograms and candidate lists; bits, tau and the union lists must equal
    the caller-scratch build's, and attention over either mask must agree."""
    from sparse_attention_video_b200 import SparseAttention, _native as N, make_policy
    from synthetic import Workload
    base = Workload(name="fg_ragged_g64", config_id=611, T=6, H=12, W=20, heads=2,
                    head_dim=128, kind="fg", fg_group=64, fg_keep_fraction=0.15)
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        wl = base.with_(config_id=base.config_id + call)
        x = make_qkv(wl)
        q, k, v = (_dev(x[n]) for n in "qkv")
        policy = make_policy(**C.policy_kwargs(wl))
        sa = SparseAttention(wl.batch, wl.heads, wl.T, wl.H, wl.W, wl.head_dim, policy)
        assert sa.scratch_bytes <= N.SA_STATIC_SCRATCH_BYTES
        sa.build_mask(q, k)
        mask_static = torch.empty(sa.mask_bytes, dtype=torch.uint8, device="cuda")
        N.build_mask_static(sa.problem, policy, q.data_ptr(), k.data_ptr(),
                            mask_static.data_ptr(), stream)
        torch.cuda.synchronize()
        assert N.status_static(stream) == N.SA_OK, f"call {call}: static build status"
        assert sa.status() == N.SA_OK, f"call {call}: caller-scratch build status"
        for what in (N.SA_EXPORT_FG_BITS, N.SA_EXPORT_FG_TAU, N.SA_EXPORT_FG_TILE_KEYS):
            a = _export(N, sa.problem, policy, sa.mask_ws, what)
            b = _export(N, sa.problem, policy, mask_static, what)
            np.testing.assert_array_equal(a, b, err_msg=f"call {call}: export {what} differs")
        o1, l1 = sa.forward(q, k, v)
        o2 = torch.empty_like(q)
        l2 = torch.empty_like(l1)
        N.forward(sa.problem, policy, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                  mask_static.data_ptr(), sa.scratch_ws.data_ptr(), o2.data_ptr(),
                  l2.data_ptr(), stream)
        torch.cuda.synchronize()
        to_np = lambda t: bf16_bits_to_f32(t.view(torch.int16).cpu().numpy().view(np.uint16))
        e = C.attention_errors(to_np(o2), l2.cpu().numpy(), to_np(o1).astype(np.float64),
                               l1.cpu().numpy().astype(np.float64))
        C.check_errors(*e, where=f"fg call {call}")
