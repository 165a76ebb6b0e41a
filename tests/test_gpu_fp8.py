"""GPU parity of FP8 attention (B200 only): E4M3 operands on kind::f8f6f4.

Through the C ABI: build the block mask (bf16 inputs), quantize Q, K and V to
E4M3 with one scale per (batch, head) tensor (sparse_attn_quantize_e4m3),
permute the codes of frame-major heads, run sparse_attn_attend_fp8. The
oracle is the exact attention of the dequantized operands
(oracle.quant.fp8_attention_rows) over the GPU's block mask.

Tolerance, derived from the kernel's arithmetic (the probabilities of the
second product are E4M3 codes of 2^4 P, P relative to the running maximum,
so an error of at most 2^-4 P above the normal range and 2^-14 below it; the
row sum uses the unrounded P):
    |O_gpu - O_ref|_c <= sum_j max(2^-4 p_j, 2^-14 / l) |v_jc|
                         + 2^-8 |O_ref|_c + 1e-4
with p_j the exact probabilities and l the row sum relative to the row
maximum (the running rescale by 2^(m_old - m_new) <= 1 only shrinks it), the
second term the bf16 rounding of the output. LSE within 1e-3.
"""
import math

import numpy as np
import pytest
import torch

from oracle import attention, pipeline, quant
from synthetic import CONFIGS, bf16_bits_to_f32, make_qkv
from tests import _cases as C

pytestmark = pytest.mark.gpu


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _bf16_to_np(t):
    return bf16_bits_to_f32(t.view(torch.int16).cpu().numpy().view(np.uint16))


def fp8_bound(qh, kh, vh, rows, keep):
    """Per-element bound on |O_gpu - O_ref| for the rows (see the module doc)."""
    d = qh.shape[1]
    s = (qh[rows] @ kh.T) / math.sqrt(d)
    s = np.where(keep, s, -np.inf)
    m = s.max(axis=1)
    p = np.exp(s - np.where(np.isfinite(m), m, 0.0)[:, None])
    l = p.sum(axis=1)
    pt = p / np.where(l > 0, l, 1.0)[:, None]
    e = np.maximum(2.0 ** -4 * pt, (2.0 ** -14 / np.where(l > 0, l, 1.0))[:, None])
    e = np.where(keep, e, 0.0)
    return e @ np.abs(vh)


def run_fp8_case(wl, heads_check=None, qblocks_per_head=None, seed=0):
    from sparse_attention_video_b200 import (SA_EXPORT_BLOCK_BITS, SA_EXPORT_HEAD_INFO,
                                             SparseAttention, make_policy)
    x = make_qkv(wl)
    q, k, v = (_dev(x[n]) for n in "qkv")
    sa = SparseAttention(wl.batch, wl.heads, wl.T, wl.H, wl.W, wl.head_dim,
                         make_policy(**C.policy_kwargs(wl)))
    sa.build_mask(q, k)
    o, lse, quantized = sa.forward_fp8(q, k, v)
    torch.cuda.synchronize()
    assert sa.status() == 0
    info = sa.export(SA_EXPORT_HEAD_INFO)
    BH = wl.batch * wl.heads
    NB = max(C.n_blocks(wl, t) for t in (wl.candidates or [None]))
    words = sa.export(SA_EXPORT_BLOCK_BITS).reshape(BH, NB, (NB + 31) // 32)
    o_np, lse_np = _bf16_to_np(o), lse.cpu().numpy()
    codes = [c.cpu().numpy() for c, _ in quantized]
    invs = [i.cpu().numpy() for _, i in quantized]
    rng = np.random.default_rng(seed)
    heads_check = range(wl.heads) if heads_check is None else heads_check
    for b in range(wl.batch):
        for h in heads_check:
            bh = b * wl.heads + h
            qf, kf, vf = (bf16_bits_to_f32(x[n][b, h]) for n in "qkv")
            # the codes the GPU attended over are the oracle's codes
            for t, (xf, name) in enumerate(((qf, "q"), (kf, "k"), (vf, "v"))):
                c_ref, inv_ref = quant.quantize_tensor(xf)
                np.testing.assert_array_equal(codes[t][b, h].reshape(-1), c_ref.reshape(-1),
                                              err_msg=f"{name} codes, head {h}")
                assert np.float32(invs[t][bh]) == inv_ref, (name, h)
            gi = info[bh]
            force = gi.candidate if wl.kind == "spade" else None
            ref = pipeline.head_mask(wl, qf, kf, h, force_choice=force)
            nb = ref["bmask"].shape[0]
            gm = C.bits_to_bool(words[bh], NB)[:nb, :nb]
            blk = ref["order_blocks"]
            from oracle import masks
            vq = np.nonzero(masks.valid_blocks(blk))[0]
            sample = vq if qblocks_per_head is None else rng.choice(
                vq, size=min(qblocks_per_head, len(vq)), replace=False)
            qh, kh, vh = quant.fp8_operands(qf, kf, vf)
            for qb in sample:
                rows, keep = attention.block_keep_rows(blk, gm, qb, wl.N)
                if len(rows) == 0:
                    continue
                o_ref, lse_ref = quant.fp8_attention_rows(qf, kf, vf, rows, keep)
                bound = fp8_bound(qh, kh, vh, rows, keep)
                err = np.abs(o_np[b, h, rows].astype(np.float64) - o_ref)
                lim = bound + 2.0 ** -8 * np.abs(o_ref) + 1e-4
                worst = float((err / lim).max())
                assert worst <= 1.0, (f"{wl.name} head {h} block {qb}: O error {err.max():.3e} "
                                      f"exceeds the FP8 bound ({worst:.2f} of it)")
                fin = np.isfinite(lse_ref)
                assert np.all(np.isneginf(lse_np[b, h, rows][~fin]))
                if fin.any():
                    lerr = np.abs(lse_np[b, h, rows][fin].astype(np.float64) - lse_ref[fin]).max()
                    assert lerr <= 1e-3, f"{wl.name} head {h} block {qb}: LSE error {lerr:.3e}"


@pytest.mark.parametrize("name", ["topk_ragged_d128", "sta_ragged", "spatiotemporal_ragged",
                                  "spade_ragged", "sta_head_windows"])
def test_fp8_small_cases(name):
    run_fp8_case(C.SMALL[name])


@pytest.mark.parametrize("name,heads,qbs", [
    ("spatiotemporal_hunyuan_720p", [0, 12, 23], 4),
    ("sta_wan21_1p3b_480p", [0, 11], 6),
])
def test_fp8_full_size_sampled(name, heads, qbs):
    run_fp8_case(CONFIGS[name], heads_check=heads, qblocks_per_head=qbs)


def test_fp8_rejects_unsupported():
    """FG slices and head_dim 64 have no FP8 kernel: rejected before any launch."""
    from sparse_attention_video_b200 import SparseAttention, _native as N, make_policy
    wl = C.SMALL["sta_d64"]
    sa = SparseAttention(1, wl.heads, wl.T, wl.H, wl.W, wl.head_dim,
                         make_policy(**C.policy_kwargs(wl)))
    z8 = torch.zeros((1, wl.heads, wl.N, wl.head_dim), dtype=torch.uint8, device="cuda")
    inv = torch.ones(wl.heads, dtype=torch.float32, device="cuda")
    o = torch.empty((1, wl.heads, wl.N, wl.head_dim), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((1, wl.heads, wl.N), dtype=torch.float32, device="cuda")
    with pytest.raises(N.SparseAttnError) as ei:
        sa.attend_fp8(z8, z8, z8, inv, inv, inv, o, lse)
    assert ei.value.code == N.SA_ERR_UNSUPPORTED
