"""Guard regions around every device buffer of a call (B200 only).

In place of a memory checker: each workspace, input and output of
sparse_attn_build_mask + sparse_attn_forward sits between two 4 KiB guards
filled with a byte pattern, and the call gets the interior pointers through
the C ABI. Afterwards every guard byte (and the padding up to the next 256
bytes) must be unchanged, the inputs must be unmodified, and O and LSE must
equal, bit for bit, those of the same call on ordinary allocations: every
reduction in these kernels is in a fixed order or on integers, so the
result may not depend on where the buffers are.
"""
import math

import numpy as np
import pytest
import torch

from synthetic import Workload, make_qkv
from tests import _cases as C

pytestmark = pytest.mark.gpu

GUARD = 4096
PATTERN = 0xA5

CASES = ["tiny_topk", "topk_ragged_d128", "sta_ragged", "sta_d64", "spatiotemporal_ragged",
         "spade_ragged", "spade_pool_fallback", "sta_head_windows", "fg"]
FG = Workload(name="guard_fg", config_id=151, T=6, H=12, W=20, heads=2, head_dim=128, kind="fg",
              fg_group=64, fg_keep_fraction=0.15)


class Guarded:
    """``nbytes`` of device memory between two guards of the pattern."""

    def __init__(self, nbytes):
        self.nbytes = nbytes
        span = (nbytes + 255) // 256 * 256
        self.buf = torch.full((GUARD + span + GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
        assert self.buf.data_ptr() % 256 == 0
        self.ptr = self.buf.data_ptr() + GUARD

    def payload(self):
        return self.buf[GUARD:GUARD + self.nbytes]

    def intact(self):
        return bool((self.buf[:GUARD] == PATTERN).all()) and \
            bool((self.buf[GUARD + self.nbytes:] == PATTERN).all())


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


@pytest.mark.parametrize("name", CASES)
def test_no_write_outside_any_buffer(name):
    from sparse_attention_video_b200 import SparseAttention, _native as N, make_policy
    wl = FG if name == "fg" else C.SMALL[name]
    x = make_qkv(wl)
    q, k, v = (_dev(x[n]) for n in "qkv")
    policy = make_policy(**C.policy_kwargs(wl))
    sa = SparseAttention(wl.batch, wl.heads, wl.T, wl.H, wl.W, wl.head_dim, policy)
    o_ref, lse_ref = sa(q, k, v)

    problem = sa.problem
    mask_bytes, scratch_bytes = N.workspace_size(problem, policy)
    qkv_bytes = q.numel() * 2
    g = {"q": Guarded(qkv_bytes), "k": Guarded(qkv_bytes), "v": Guarded(qkv_bytes),
         "mask": Guarded(mask_bytes), "scratch": Guarded(max(scratch_bytes, 256)),
         "o": Guarded(qkv_bytes), "lse": Guarded(lse_ref.numel() * 4)}
    for n, t in (("q", q), ("k", k), ("v", v)):
        g[n].payload().copy_(t.contiguous().view(torch.uint8).reshape(-1))
    stream = torch.cuda.current_stream().cuda_stream
    N.build_mask(problem, policy, g["q"].ptr, g["k"].ptr, g["mask"].ptr, g["scratch"].ptr, stream)
    N.forward(problem, policy, g["q"].ptr, g["k"].ptr, g["v"].ptr, g["mask"].ptr,
              g["scratch"].ptr, g["o"].ptr, g["lse"].ptr, stream)
    torch.cuda.synchronize()
    assert N.status(g["scratch"].ptr, stream) == N.SA_OK

    bad = [n for n, b in g.items() if not b.intact()]
    assert not bad, f"{wl.name}: written outside {bad}"
    for n, t in (("q", q), ("k", k), ("v", v)):
        assert torch.equal(g[n].payload(), t.contiguous().view(torch.uint8).reshape(-1)), n
    assert torch.equal(g["o"].payload(), o_ref.contiguous().view(torch.uint8).reshape(-1))
    assert torch.equal(g["lse"].payload(), lse_ref.contiguous().view(torch.uint8).reshape(-1))
    assert math.isfinite(float(o_ref.float().abs().max()))


def test_cached_mask_and_quantizer_write_inside_their_buffers():
    # the FG cached mask (LSE in, bits and union lists out) and the E4M3
    # quantizer (codes and scales out), each between guards
    from sparse_attention_video_b200 import SparseAttention, _native as N, make_policy
    wl = FG
    x = make_qkv(wl)
    q, k, v = (_dev(x[n]) for n in "qkv")
    policy = make_policy("fg", block=128, fg_group=64, fg_keep_fraction=1.0)
    sa = SparseAttention(wl.batch, wl.heads, wl.T, wl.H, wl.W, wl.head_dim, policy)
    lse = torch.zeros((wl.batch, wl.heads, wl.N), dtype=torch.float32, device="cuda")
    sa.build_mask_fg_cached(q, k, lse + float(np.log(wl.N)))     # a uniform-attention LSE
    problem = sa.problem
    mask_bytes, scratch_bytes = N.workspace_size(problem, policy)
    qkv_bytes = q.numel() * 2
    g = {"q": Guarded(qkv_bytes), "k": Guarded(qkv_bytes), "lse": Guarded(lse.numel() * 4),
         "mask": Guarded(mask_bytes), "scratch": Guarded(max(scratch_bytes, 256))}
    g["q"].payload().copy_(q.view(torch.uint8).reshape(-1))
    g["k"].payload().copy_(k.view(torch.uint8).reshape(-1))
    g["lse"].payload().copy_((lse + float(np.log(wl.N))).view(torch.uint8).reshape(-1))
    stream = torch.cuda.current_stream().cuda_stream
    N.build_mask_fg_cached(problem, policy, g["q"].ptr, g["k"].ptr, g["lse"].ptr, 0.0,
                           g["mask"].ptr, g["scratch"].ptr, stream)
    n_el, n_t = wl.N * wl.head_dim, wl.batch * wl.heads
    gc, gi = Guarded(n_el * n_t), Guarded(4 * n_t)
    N.quantize_e4m3(g["q"].ptr, n_el, n_t, gc.ptr, gi.ptr, stream)
    torch.cuda.synchronize()
    assert N.status(g["scratch"].ptr, stream) == N.SA_OK
    bad = [n for n, b in list(g.items()) + [("codes", gc), ("inv", gi)] if not b.intact()]
    assert not bad, f"written outside {bad}"
    # the bitmask, tau and union lists match the ordinary run's; the rest of
    # the mask workspace is not written by this call
    lay = [(N.SA_EXPORT_FG_BITS, "bits"), (N.SA_EXPORT_FG_TAU, "tau"),
           (N.SA_EXPORT_FG_TILE_KEYS, "tile keys")]
    for what, label in lay:
        nb = N.export_bytes(problem, policy, what)
        a = np.empty(nb, np.uint8)
        b = np.empty(nb, np.uint8)
        N.mask_export(problem, policy, sa.mask_ws.data_ptr(), what, a.ctypes.data, nb, stream)
        N.mask_export(problem, policy, g["mask"].ptr, what, b.ctypes.data, nb, stream)
        assert np.array_equal(a, b), label
