"""Device-side failure detection without a GPU fault (B200 only).

A kernel waits, with the library's bounded wait, on a barrier that nothing
completes. The wait must give up after about a second, record a timeout and
the wait's site in the status word, and return; while the status is set,
attention kernels that share the status word stop at once; once it is
cleared, the same context computes correct results again.
"""
import time

import numpy as np
import pytest
import torch

from oracle import attention, pipeline
from synthetic import bf16_bits_to_f32, make_qkv
from tests import _cases as C

pytestmark = pytest.mark.gpu


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def test_bounded_wait_times_out_reports_and_context_recovers():
    from sparse_attention_video_b200 import SparseAttention, _native as N, make_policy
    wl = C.SMALL["sta_ragged"]
    x = make_qkv(wl)
    q, k, v = (_dev(x[n]) for n in "qkv")
    sa = SparseAttention(1, wl.heads, wl.T, wl.H, wl.W, wl.head_dim, make_policy(**C.policy_kwargs(wl)))
    stream = torch.cuda.current_stream()
    sa.build_mask(q, k)                              # clears the status word
    torch.cuda.synchronize()
    assert sa.status() == N.SA_OK

    t0 = time.perf_counter()
    assert N.lib().sparse_attn_selftest_wait_timeout(sa.scratch_ws.data_ptr(), stream.cuda_stream) == 0
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert 0.5 < dt < 30.0, dt                       # gave up after about one second
    words = sa.scratch_ws[:12].cpu().view(torch.int32).numpy().view(np.uint32)
    assert words[0] & 1                              # timeout flag
    assert words[1] >> 16 == 0x7E57                  # the self-test's wait site
    assert words[2] == 1                             # the kernel saw its own wait give up

    # a timeout recorded in the status word stops later kernels that share it
    o = torch.full_like(q, 7.0)
    lse = torch.full(q.shape[:3], 7.0, dtype=torch.float32, device="cuda")
    sa.attend(q, k, v, o, lse)
    torch.cuda.synchronize()
    assert torch.all(o == 7.0) and torch.all(lse == 7.0)
    assert sa.status(clear=True) == N.SA_ERR_DEVICE_TIMEOUT
    assert sa.status() == N.SA_OK

    # the context is still usable: a normal call matches the oracle
    o, lse = sa.forward(q, k, v)
    torch.cuda.synchronize()
    assert sa.status() == N.SA_OK
    o_np = bf16_bits_to_f32(o.view(torch.int16).cpu().numpy().view(np.uint16))
    for h in range(wl.heads):
        qf, kf, vf = (bf16_bits_to_f32(x[n][0, h]) for n in "qkv")
        ref = pipeline.head_mask(wl, qf, kf, h)
        o_ref, lse_ref = attention.block_sparse_attention(qf, kf, vf, ref["order_blocks"], ref["bmask"])
        C.check_errors(*C.attention_errors(o_np[0, h], lse.cpu().numpy()[0, h], o_ref, lse_ref),
                       where=f"after recovery, head {h}")
