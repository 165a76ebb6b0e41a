"""GPU parity of the block-sparse path against the CPU oracle (B200 only).

Every case goes through the C ABI (libsparse_attn.so via the ctypes binding):
build the mask, run attention, then compare
  - the block mask bit by bit with the oracle's (a block whose deciding value
    lies within 1e-4 relative of the cut may differ; nothing else may),
  - the SPADE blocking choice (may differ only on a SICS near-tie),
  - O and LSE with the oracle's masked attention over the GPU's validated
    mask: O max-abs <= 2e-2, mean-abs <= 2e-3, LSE max-abs <= 1e-3.
"""
import numpy as np
import pytest
import torch

from oracle import attention, masks, pipeline
from synthetic import CONFIGS, bf16_bits_to_f32, make_qkv
from tests import _cases as C

pytestmark = pytest.mark.gpu


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _bf16_to_np(t):
    return bf16_bits_to_f32(t.view(torch.int16).cpu().numpy().view(np.uint16))


def run_block_case(wl, heads_check=None, qblocks_per_head=None, seed=0):
    from sparse_attention_video_b200 import (SA_EXPORT_BLOCK_BITS, SA_EXPORT_HEAD_INFO,
                                             SparseAttention, make_policy)
    x = make_qkv(wl)
    q, k, v = (_dev(x[n]) for n in "qkv")
    sa = SparseAttention(wl.batch, wl.heads, wl.T, wl.H, wl.W, wl.head_dim,
                         make_policy(**C.policy_kwargs(wl)))
    o, lse = sa(q, k, v)
    torch.cuda.synchronize()
    assert sa.status() == 0
    info = sa.export(SA_EXPORT_HEAD_INFO)
    BH = wl.batch * wl.heads
    words = sa.export(SA_EXPORT_BLOCK_BITS)
    NB = max(C.n_blocks(wl, t) for t in (wl.candidates or [None]))
    words = words.reshape(BH, NB, (NB + 31) // 32)
    o_np = _bf16_to_np(o)
    lse_np = lse.cpu().numpy()
    rng = np.random.default_rng(seed)
    heads_check = range(wl.heads) if heads_check is None else heads_check
    worst = [0.0, 0.0, 0.0]
    for b in range(wl.batch):
        for h in heads_check:
            bh = b * wl.heads + h
            qf, kf, vf = (bf16_bits_to_f32(x[n][b, h]) for n in "qkv")
            gi = info[bh]
            ref = pipeline.head_mask(wl, qf, kf, h)
            if wl.kind == "spade":
                tot = ref["info"]["sics_totals"]
                np.testing.assert_allclose(list(gi.sics_total)[:len(tot)], tot, rtol=2e-4, atol=1e-2)
                if gi.candidate != ref["info"]["choice"]:
                    a, c = tot[gi.candidate], tot[ref["info"]["choice"]]
                    assert abs(a - c) <= C.REL_TIE * max(abs(a), abs(c)), (h, tot, gi.candidate)
                    ref = pipeline.head_mask(wl, qf, kf, h, force_choice=gi.candidate)
            nb = ref["bmask"].shape[0]
            assert gi.nb == nb
            gm = C.bits_to_bool(words[bh], NB)[:nb, :nb]
            om = ref["bmask"]
            diff = np.argwhere(gm != om)
            if len(diff):
                valid = masks.valid_blocks(ref["order_blocks"])
                for i in np.unique(diff[:, 0]):
                    row_diff = gm[i] != om[i]
                    if wl.kind == "topk":
                        amb = C.ambiguous_topk(ref["info"]["scores"][i], wl.topk, valid)
                        amb[i] = False if wl.keep_diagonal else amb[i]
                    elif wl.kind == "spade":
                        amb = C.ambiguous_top_p(ref["info"]["scores"][i], valid, wl.top_p)
                    else:
                        amb = np.zeros(nb, bool)
                    bad = row_diff & ~amb
                    assert not bad.any(), (f"head {h} query block {i}: blocks "
                                           f"{np.nonzero(bad)[0].tolist()} differ")
            assert gi.kept == int(gm.sum())
            blk = ref["order_blocks"]
            vq = np.nonzero(masks.valid_blocks(blk))[0]
            sample = vq if qblocks_per_head is None else rng.choice(
                vq, size=min(qblocks_per_head, len(vq)), replace=False)
            o_ref, lse_ref = attention.block_sparse_attention(qf, kf, vf, blk, gm, sample)
            rows = np.concatenate([blk[i][blk[i] >= 0] for i in sample])
            e = C.attention_errors(o_np[b, h, rows], lse_np[b, h, rows], o_ref[rows], lse_ref[rows])
            C.check_errors(*e, where=f"{wl.name} head {h}")
            worst = [max(a, c) for a, c in zip(worst, e)]
    return worst


@pytest.mark.parametrize("name", list(C.SMALL))
def test_small_cases(name):
    run_block_case(C.SMALL[name])


@pytest.mark.parametrize("name,heads,qbs", [
    ("tiny_topk", None, None),
    ("sta_wan21_1p3b_480p", [0, 5, 11], 12),
    ("spatiotemporal_hunyuan_720p", [0, 11, 12, 23], 8),
    ("spade_wan21_14b_720p", [0, 17, 39], 8),
])
def test_full_size_sampled(name, heads, qbs):
    run_block_case(CONFIGS[name], heads_check=heads, qblocks_per_head=qbs)


@pytest.mark.parametrize("name", ["sta_wan21_1p3b_480p", "spatiotemporal_hunyuan_720p",
                                  "spade_wan21_14b_720p"])
def test_full_size_every_head(name):
    """Every head's whole block mask at full size against the oracle
    (bit-exact outside the 1e-4 tie band; SPADE's blocking choice and SICS
    totals), attention on one sampled query block per head."""
    run_block_case(CONFIGS[name], heads_check=None, qblocks_per_head=1, seed=11)


def test_explicit_random_masks_with_empty_rows():
    """Attention alone on random block masks in every layout; rows with no kept
    block must give O = 0 and LSE = -inf."""
    from sparse_attention_video_b200 import (SA_LAYOUT_FRAME_MAJOR, SA_LAYOUT_IDENTITY,
                                             SA_LAYOUT_TILE, SparseAttention, make_policy)
    from oracle import layout
    wl = C.SMALL["spatiotemporal_ragged"]
    x = make_qkv(wl)
    q, k, v = (_dev(x[n]) for n in "qkv")
    rng = np.random.default_rng(7)
    for lay, tile in ((SA_LAYOUT_IDENTITY, (1, 1, 128)), (SA_LAYOUT_FRAME_MAJOR, (1, 1, 128)),
                      (SA_LAYOUT_TILE, (2, 8, 8))):
        if lay == SA_LAYOUT_TILE:
            order = layout.tile_order(wl.T, wl.H, wl.W, *tile)
        elif lay == SA_LAYOUT_FRAME_MAJOR:
            order = layout.frame_major_order(wl.T, wl.H, wl.W, 128)
        else:
            order = layout.identity_order(wl.T, wl.H, wl.W, 128)
        blk = layout.blocks(order, 128)
        nb = blk.shape[0]
        dense = rng.random((wl.heads, nb, nb)) < 0.35
        dense[:, 1, :] = False                                  # an empty row
        dense[:, :, ~masks.valid_blocks(blk)] = False
        packed = C.pack_rows(dense)
        bits_dev = torch.from_numpy(packed.view(np.int32)).cuda()
        pol = make_policy("explicit", block=128, tile=tile, explicit_layout=lay, explicit_bits=bits_dev)
        sa = SparseAttention(1, wl.heads, wl.T, wl.H, wl.W, wl.head_dim, pol)
        o, lse = sa(q, k, v)
        torch.cuda.synchronize()
        assert sa.status() == 0
        o_np, lse_np = _bf16_to_np(o), lse.cpu().numpy()
        for h in range(wl.heads):
            qf, kf, vf = (bf16_bits_to_f32(x[n][0, h]) for n in "qkv")
            o_ref, lse_ref = attention.block_sparse_attention(qf, kf, vf, blk, dense[h])
            e = C.attention_errors(o_np[0, h], lse_np[0, h], o_ref, lse_ref)
            C.check_errors(*e, where=f"explicit layout {lay} head {h}")
            empty_rows = blk[1][blk[1] >= 0]
            assert np.all(o_np[0, h, empty_rows] == 0.0)


def test_explicit_head_dim_64_blocks_of_64():
    """Caller-supplied masks run the two-warpgroup kernel: head_dim 64 with
    64-token blocks in the identity and 3D tile layouts (the policies that
    bound their rows run the one-warpgroup kernel at these sizes)."""
    from sparse_attention_video_b200 import SA_LAYOUT_IDENTITY, SA_LAYOUT_TILE, SparseAttention, make_policy
    from oracle import layout
    wl = C.SMALL["sta_d64"]
    x = make_qkv(wl)
    q, k, v = (_dev(x[n]) for n in "qkv")
    rng = np.random.default_rng(9)
    for lay, tile in ((SA_LAYOUT_IDENTITY, (1, 1, 64)), (SA_LAYOUT_TILE, (2, 4, 8))):
        if lay == SA_LAYOUT_TILE:
            order = layout.tile_order(wl.T, wl.H, wl.W, *tile)
        else:
            order = layout.identity_order(wl.T, wl.H, wl.W, 64)
        blk = layout.blocks(order, 64)
        nb = blk.shape[0]
        dense = rng.random((wl.heads, nb, nb)) < 0.4
        dense[:, :, ~masks.valid_blocks(blk)] = False
        bits_dev = torch.from_numpy(C.pack_rows(dense).view(np.int32)).cuda()
        pol = make_policy("explicit", block=64, tile=tile, explicit_layout=lay, explicit_bits=bits_dev)
        sa = SparseAttention(1, wl.heads, wl.T, wl.H, wl.W, wl.head_dim, pol)
        o, lse = sa(q, k, v)
        torch.cuda.synchronize()
        assert sa.status() == 0
        o_np, lse_np = _bf16_to_np(o), lse.cpu().numpy()
        for h in range(wl.heads):
            qf, kf, vf = (bf16_bits_to_f32(x[n][0, h]) for n in "qkv")
            o_ref, lse_ref = attention.block_sparse_attention(qf, kf, vf, blk, dense[h])
            e = C.attention_errors(o_np[0, h], lse_np[0, h], o_ref, lse_ref)
            C.check_errors(*e, where=f"explicit d64 layout {lay} head {h}")
