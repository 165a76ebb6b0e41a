"""GPU parity of the E4M3 quantizer (Sparse VideoGen review: FP8
quantization) against the oracle, through the C ABI.

The codes are integers decided by the same correctly rounded float32 steps
on both sides (inv = 448 / amax, y = x * inv, then round to nearest even
with saturation), so codes and scales must match bit for bit.
"""
import numpy as np
import pytest
import torch

from oracle import quant
from synthetic import CONFIGS, Workload, bf16_bits_to_f32, f32_to_bf16_bits, make_qkv

pytestmark = pytest.mark.gpu


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _check(x_bits):
    from sparse_attention_video_b200 import quantize_e4m3
    codes, inv = quantize_e4m3(_dev(x_bits))
    torch.cuda.synchronize()
    codes, inv = codes.cpu().numpy(), inv.cpu().numpy()
    B, H = x_bits.shape[:2]
    for b in range(B):
        for h in range(H):
            ref_codes, ref_inv = quant.quantize_tensor(bf16_bits_to_f32(x_bits[b, h]))
            assert inv[b * H + h] == ref_inv, (b, h, inv[b * H + h], ref_inv)
            diff = codes[b, h] != ref_codes
            assert not diff.any(), (b, h, int(diff.sum()), np.argwhere(diff)[:5].tolist())


@pytest.mark.parametrize("tensor", ["q", "k", "v"])
def test_quantize_small_workload_bit_exact(tensor):
    wl = Workload(name="quant_small", config_id=141, T=5, H=9, W=16, heads=3, head_dim=64)
    _check(make_qkv(wl)[tensor])


def test_quantize_wide_range_subnormals_and_zero_head():
    # per-row magnitudes over 2^-20 .. 2^4, so many codes are subnormal; one
    # head is all zeros (inv = 1, every code 0) and one holds a single value
    g = np.random.default_rng(5)
    x = g.standard_normal((1, 3, 1000, 64)) * np.exp2(g.uniform(-20, 4, (1, 3, 1000, 1)))
    x[0, 1] = 0.0
    x[0, 2] = 0.0
    x[0, 2, 17, 5] = -3.0
    _check(f32_to_bf16_bits(x.astype(np.float32)))


def test_quantize_full_size_heads():
    # two heads of the 115,200-token grid: 14.7 M elements per head
    wl = CONFIGS["fg_slices_hunyuan_720p"].with_(heads=2)
    _check(make_qkv(wl)["k"])
