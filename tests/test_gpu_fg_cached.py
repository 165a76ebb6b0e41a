"""GPU parity of the FG cached mask (FG-Attn review: the cached strategy,
threshold 0.5/N on the full attention map), through the C ABI.

The mask kernel takes the LSE of full attention as an input. Two sources:
  - the oracle's float64 LSE, which isolates the mask kernel: a slice's
    decision may differ from the oracle's only where its largest probability
    lies within 1e-4 relative of tau;
  - the library's own dense attention (an explicit policy keeping every
    block), the whole path a caller runs: its LSE parity bound is 1e-3
    absolute, which moves a probability by up to e^1e-3 - 1 relative, so the
    band there is 2e-3.
Then the gather attention over the validated mask against the oracle's slice
attention, with the usual O and LSE tolerances, and a threshold so small that
every slice is kept, where the cached path must reproduce dense attention.
"""
import math

import numpy as np
import pytest
import torch

from oracle import attention, masks
from synthetic import Workload, bf16_bits_to_f32, f32_to_bf16_bits, make_qkv
from tests import _cases as C

pytestmark = pytest.mark.gpu

CASES = {
    "cached_ragged_g64": Workload(name="cached_ragged_g64", config_id=131, T=6, H=12, W=20, heads=2,
                                  head_dim=128, kind="fg", fg_group=64, fg_rule="cached"),
    "cached_g128_d64": Workload(name="cached_g128_d64", config_id=132, T=5, H=9, W=16, heads=2,
                                head_dim=64, kind="fg", fg_group=128, fg_rule="cached"),
}


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _dense_lse(wl, q, k, v):
    from sparse_attention_video_b200 import SA_LAYOUT_IDENTITY, SparseAttention, make_policy
    nb = math.ceil(wl.N / 128)
    words = torch.full((wl.batch * wl.heads, nb, math.ceil(nb / 32)), -1, dtype=torch.int32,
                       device="cuda")
    pol = make_policy("explicit", block=128, explicit_layout=SA_LAYOUT_IDENTITY, explicit_bits=words)
    dsa = SparseAttention(wl.batch, wl.heads, wl.T, wl.H, wl.W, wl.head_dim, pol)
    _, lse = dsa(q, k, v)
    return lse


def _oracle_lse(wl, x):
    out = np.zeros((wl.batch, wl.heads, wl.N), dtype=np.float32)
    rows = np.arange(wl.N)
    keep = np.ones((wl.N, wl.N), dtype=bool)
    for b in range(wl.batch):
        for h in range(wl.heads):
            qf, kf, vf = (bf16_bits_to_f32(x[n][b, h]) for n in "qkv")
            out[b, h] = attention.masked_attention_rows(qf, kf, vf, rows, keep)[1]
    return out


def _run(wl, lse_source, band, tau=0.0, q_scale=8.0):
    from sparse_attention_video_b200 import (SA_EXPORT_FG_BITS, SA_EXPORT_FG_TAU,
                                             SparseAttention, make_policy)
    x = make_qkv(wl)
    # The smooth synthetic fields give near-uniform attention (every slice
    # passes 0.5/N); queries scaled by 8 sharpen it so that the cut keeps
    # about a third (d 128, groups of 64) to two thirds (d 64, groups of 128)
    # of the slices, with a few slices near tau.
    x["q"] = f32_to_bf16_bits(np.float32(q_scale) * bf16_bits_to_f32(x["q"]))
    q, k, v = (_dev(x[n]) for n in "qkv")
    if lse_source == "oracle":
        lse_in = torch.from_numpy(_oracle_lse(wl, x)).cuda()
    else:
        lse_in = _dense_lse(wl, q, k, v)
    # keep fraction 1: the union lists may hold every slice
    sa = SparseAttention(wl.batch, wl.heads, wl.T, wl.H, wl.W, wl.head_dim,
                         make_policy("fg", block=128, fg_group=wl.fg_group, fg_keep_fraction=1.0))
    sa.build_mask_fg_cached(q, k, lse_in, tau=tau)
    o, lse = sa.forward(q, k, v)
    torch.cuda.synchronize()
    assert sa.status() == 0
    N, M = wl.N, wl.fg_group
    G, WN = math.ceil(N / M), math.ceil(N / 32)
    tau_ref = tau if tau > 0 else 0.5 / N
    assert np.all(sa.export(SA_EXPORT_FG_TAU) == np.float32(tau_ref))
    words = sa.export(SA_EXPORT_FG_BITS).reshape(wl.batch * wl.heads, G, WN)
    o_np = bf16_bits_to_f32(o.view(torch.int16).cpu().numpy().view(np.uint16))
    lse_np = lse.cpu().numpy()
    kept = []
    for b in range(wl.batch):
        for h in range(wl.heads):
            bh = b * wl.heads + h
            qf, kf, vf = (bf16_bits_to_f32(x[n][b, h]) for n in "qkv")
            pmax = masks.fg_cached_pmax(qf, kf, M)
            keep_ref = pmax > np.float32(tau_ref)
            bits = np.unpackbits(words[bh].view(np.uint8), bitorder="little").reshape(G, -1)
            assert not bits[:, N:].any(), "bits past the last key"
            keep_gpu = bits[:, :N].astype(bool)
            bad = (keep_gpu != keep_ref) & (np.abs(pmax - tau_ref) > band * tau_ref)
            assert not bad.any(), (f"{wl.name} head {h}: {int(bad.sum())} slices differ outside "
                                   f"the band; first {np.argwhere(bad)[:5].tolist()}")
            o_ref, lse_ref = attention.slice_attention(qf, kf, vf, keep_gpu, M)
            e = C.attention_errors(o_np[b, h], lse_np[b, h], o_ref, lse_ref)
            C.check_errors(*e, where=f"{wl.name} head {h}")
            kept.append(keep_gpu.mean())
    return kept


@pytest.mark.parametrize("name", list(CASES))
def test_cached_mask_kernel_with_oracle_lse(name):
    kept = _run(CASES[name], "oracle", C.REL_TIE)
    assert all(0.0 < f < 1.0 for f in kept)          # a real cut, not all or nothing


@pytest.mark.parametrize("name", list(CASES))
def test_cached_mask_whole_path_with_library_lse(name):
    _run(CASES[name], "library", 2e-3)


def test_cached_mask_tiny_threshold_keeps_every_slice():
    # tau = 1e-30: every probability of these inputs is far above it, so every
    # slice is kept and the gather attention is dense attention
    kept = _run(CASES["cached_ragged_g64"], "oracle", C.REL_TIE, tau=1e-30, q_scale=1.0)
    assert all(f == 1.0 for f in kept)
