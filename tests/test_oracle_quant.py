"""Pins for the oracle's FP8 (E4M3) operands (CPU only).

The E4M3 codec is checked against torch's float8_e4m3fn type (its byte
decoding and its round-to-nearest-even cast), and every code's round trip.
The per-tensor scale is checked by its defining properties: the largest
element lands on 448, a power-of-two rescale of the tensor leaves the codes
unchanged, and each element's error stays within half a step of the grid.
"""
import numpy as np
import pytest
import torch

from oracle import attention, quant


def _torch_codes(y):
    t = torch.from_numpy(np.asarray(y, dtype=np.float32))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def _finite_values():
    vals = quant.e4m3_decode(np.arange(256, dtype=np.uint8))
    return np.unique(vals[np.isfinite(vals)])


def test_decode_matches_torch_float8_e4m3fn():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = quant.e4m3_decode(codes.numpy())
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.nonzero(nan)[0].tolist() == [0x7F, 0xFF]
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.nanmax(got) == 448.0 and got[1] == 2.0 ** -9


def test_every_finite_code_round_trips():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    assert np.array_equal(quant.e4m3_encode(quant.e4m3_decode(codes)), codes)


def test_round_matches_torch_cast_including_ties():
    g = np.random.default_rng(0)
    mags = np.exp2(g.uniform(-14.0, np.log2(448.0), 20000))
    y = (mags * g.choice([-1.0, 1.0], mags.size)).astype(np.float32)
    grid = _finite_values()
    pos = grid[grid > 0]
    mids = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)          # exact in float32: ties
    near = np.concatenate([np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(1e9))])
    tiny = (np.arange(0, 40, dtype=np.float32) * np.float32(2.0 ** -11))   # around the subnormals
    for arr in (y, mids, -mids, near, tiny, -tiny):
        arr = np.asarray(arr, dtype=np.float32)
        assert np.array_equal(quant.e4m3_encode(arr), _torch_codes(arr)), arr[:8]


def test_ties_go_to_the_even_mantissa():
    # between 1 (m=0) and 1.125 (m=1): 1.0625 goes down; between 1.125 and
    # 1.25 (m=2): 1.1875 goes up; subnormal 1.5 * 2^-9 goes to 2 * 2^-9
    assert quant.e4m3_round(1.0625) == 1.0
    assert quant.e4m3_round(1.1875) == 1.25
    assert quant.e4m3_round(1.5 * 2.0 ** -9) == 2.0 * 2.0 ** -9
    assert quant.e4m3_round(0.5 * 2.0 ** -9) == 0.0


def test_saturates_at_448():
    for v in (448.0, 449.0, 463.9, 464.0, 480.0, 1e6):
        assert quant.e4m3_round(v) == 448.0 and quant.e4m3_round(-v) == -448.0
    assert quant.e4m3_encode(np.array([1e6], np.float32))[0] == 0x7E


def test_quantize_tensor_scale_and_extreme_element():
    g = np.random.default_rng(1)
    x = g.standard_normal((64, 32)).astype(np.float32)
    codes, inv = quant.quantize_tensor(x)
    i = np.unravel_index(np.argmax(np.abs(x)), x.shape)
    assert abs(quant.e4m3_decode(codes[i])) == 448.0
    assert inv == np.float32(np.float32(448.0) / np.float32(np.abs(x).max()))
    z_codes, z_inv = quant.quantize_tensor(np.zeros((4, 4), np.float32))
    assert z_inv == 1.0 and not z_codes.any()


@pytest.mark.parametrize("k", [-7, -1, 3, 10])
def test_power_of_two_rescale_keeps_codes(k):
    g = np.random.default_rng(2)
    x = (g.standard_normal((50, 16)) * np.exp2(g.uniform(-6, 2, (50, 1)))).astype(np.float32)
    c0, inv0 = quant.quantize_tensor(x)
    c1, inv1 = quant.quantize_tensor((x * np.float32(2.0 ** k)).astype(np.float32))
    assert np.array_equal(c0, c1)
    assert inv1 == np.float32(inv0 * np.float32(2.0 ** -k))


def test_dequantized_error_within_half_a_grid_step():
    g = np.random.default_rng(3)
    x = (g.standard_normal((200, 64)) * np.exp2(g.uniform(-12, 0, (200, 1)))).astype(np.float32)
    codes, inv = quant.quantize_tensor(x)
    xh = quant.dequantize(codes, inv)
    y = x.astype(np.float64) * np.float64(inv)
    normal = np.abs(y) >= 2.0 ** -6
    err = np.abs(xh - x.astype(np.float64)) * np.float64(inv)      # in grid units of y
    # one float32 rounding of x * inv plus half a step of the grid
    assert np.all(err[normal] <= (2.0 ** -4 + 2.0 ** -23) * np.abs(y[normal]))
    assert np.all(err[~normal] <= 2.0 ** -10 + 2.0 ** -23 * 2.0 ** -6)
    assert (~normal).any() and normal.any()


def test_representable_operands_are_unchanged():
    # values already on the E4M3 grid with 448 present: inv = 1, codes exact
    g = np.random.default_rng(4)
    grid = _finite_values()
    x = g.choice(grid, (30, 8)).astype(np.float32)
    x[0, 0] = 448.0
    for xh in quant.fp8_operands(x, -x, x):
        assert np.array_equal(np.abs(xh), np.abs(x.astype(np.float64)))


def test_fp8_attention_on_grid_operands_is_plain_attention():
    # operands on the E4M3 grid with 448 present in each: quantization is the
    # identity, so FP8 attention is the plain attention of the same values
    g = np.random.default_rng(6)
    grid = _finite_values()
    small = grid[np.abs(grid) <= 4.0]
    q, k, v = (g.choice(small, (40, 16)).astype(np.float32) for _ in range(3))
    for x in (q, k, v):
        x[0, 0] = 448.0
    rows = np.arange(40)
    keep = g.random((40, 40)) < 0.6
    keep[:, 0] = True
    o8, l8 = quant.fp8_attention_rows(q, k, v, rows, keep)
    o, l = attention.masked_attention_rows(q, k, v, rows, keep)
    assert np.array_equal(o8, o) and np.array_equal(l8, l)


def test_fp8_attention_error_is_bounded_by_the_operand_steps():
    # each operand moves by at most half a grid step (2^-4 relative for
    # normals): scores move by at most |dq||k| + |q||dk| + |dq||dk| per
    # pair (Cauchy-Schwarz), which bounds the LSE shift; O moves by at most
    # the V step plus the spread of V times the weight change
    g = np.random.default_rng(7)
    n, d = 64, 32
    q, k, v = (g.standard_normal((n, d)).astype(np.float32) for _ in range(3))
    rows = np.arange(n)
    keep = np.ones((n, n), bool)
    o8, l8 = quant.fp8_attention_rows(q, k, v, rows, keep)
    o, l = attention.masked_attention_rows(q, k, v, rows, keep)
    qh, kh, vh = quant.fp8_operands(q, k, v)
    dq = np.linalg.norm(qh - q, axis=1)
    dk = np.linalg.norm(kh - k, axis=1)
    nq, nk = np.linalg.norm(q, axis=1), np.linalg.norm(k, axis=1)
    ds = (np.outer(dq, nk) + np.outer(nq, dk) + np.outer(dq, dk)).max() / np.sqrt(d)
    assert np.all(np.abs(l8 - l) <= ds + 1e-12)
    w_change = np.expm1(2 * ds)                       # relative weight change bound
    spread = np.abs(v).max() + np.abs(vh).max()
    assert np.all(np.abs(o8 - o) <= np.abs(vh - v).max() + spread * w_change + 1e-12)
    assert 0 < np.abs(o8 - o).max() < 0.2              # a real, small difference
