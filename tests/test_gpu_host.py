"""The host-buffer entry point (sparse_attn_forward_host) on a B200.

One call copies Q, K and V in from host memory, builds the mask, runs the
forward pass and copies O and LSE back. Its outputs must equal, bit for bit,
the device path (build_mask + forward on device tensors) on the same inputs,
whose parity with the oracle the other GPU tests establish; and steps that
alternate between two objects on two streams, each step with its own
inputs, must each give its own device-path result.
"""
import numpy as np
import pytest
import torch

from synthetic import make_qkv
from tests import _cases as C

pytestmark = pytest.mark.gpu


def _host(bits):
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.pin_memory()


def _device_path(wl, policy, x):
    from sparse_attention_video_b200 import SparseAttention
    q, k, v = (_host(x[n]).cuda() for n in "qkv")
    sa = SparseAttention(wl.batch, wl.heads, wl.T, wl.H, wl.W, wl.head_dim, policy)
    o, lse = sa(q, k, v)
    torch.cuda.synchronize()
    assert sa.status() == 0
    return o.cpu(), lse.cpu()


@pytest.mark.parametrize("name", ["spatiotemporal_ragged", "spade_ragged", "sta_d64"])
def test_forward_host_equals_device_path(name):
    from sparse_attention_video_b200 import SparseAttention, make_policy
    wl = C.SMALL[name]
    policy = make_policy(**C.policy_kwargs(wl))
    x = make_qkv(wl)
    o_ref, lse_ref = _device_path(wl, policy, x)
    sa = SparseAttention(wl.batch, wl.heads, wl.T, wl.H, wl.W, wl.head_dim, policy)
    qh, kh, vh = (_host(x[n]) for n in "qkv")
    oh = torch.empty(qh.shape, dtype=torch.bfloat16).pin_memory()
    lh = torch.empty(qh.shape[:3], dtype=torch.float32).pin_memory()
    sa.forward_host(qh, kh, vh, oh, lh)
    torch.cuda.synchronize()
    assert sa.status() == 0
    assert torch.equal(oh.view(torch.int16), o_ref.view(torch.int16))
    assert torch.equal(lh, lse_ref)


def test_forward_host_two_streams_alternating():
    from sparse_attention_video_b200 import SparseAttention, make_policy
    base = C.SMALL["topk_ragged_d128"]
    policy = make_policy(**C.policy_kwargs(base))
    lanes = [(SparseAttention(base.batch, base.heads, base.T, base.H, base.W, base.head_dim,
                              policy), torch.cuda.Stream()) for _ in range(2)]
    steps = []
    for i in range(4):                              # different inputs every step
        wl = base.with_(config_id=base.config_id + 700 + i)
        x = make_qkv(wl)
        hq, hk, hv = (_host(x[n]) for n in "qkv")
        oh = torch.empty(hq.shape, dtype=torch.bfloat16).pin_memory()
        lh = torch.empty(hq.shape[:3], dtype=torch.float32).pin_memory()
        steps.append((wl, x, (hq, hk, hv), oh, lh))
    for i, (_, _, (hq, hk, hv), oh, lh) in enumerate(steps):
        sa, st = lanes[i % 2]
        sa.forward_host(hq, hk, hv, oh, lh, st)
    torch.cuda.synchronize()
    for sa, _ in lanes:
        assert sa.status() == 0
    for wl, x, _, oh, lh in steps:
        o_ref, lse_ref = _device_path(wl, policy, x)
        assert torch.equal(oh.view(torch.int16), o_ref.view(torch.int16)), wl.config_id
        assert torch.equal(lh, lse_ref), wl.config_id
