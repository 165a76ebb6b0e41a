"""FP8 (E4M3) operands for attention, written out plainly (test infrastructure).

Sparse VideoGen review (summary and forward implications): attention may run
with FP8-quantized operands, which the pages credit with about 1.3x more on
HunyuanVideo at a small fidelity cost. The pages give no format, scale or
granularity. The reading here: Q, K and V are each quantized to E4M3, with one
scale per (batch, head) tensor, and the attention is the exact attention of
the dequantized operands. How a kernel rounds its softmax probabilities for
the second product is the kernel's arithmetic, bounded by the tests, not part
of this definition.

E4M3 is the format of "FP8 Formats for Deep Learning" (Micikevicius et al.,
arXiv 2209.05433): 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits;
exponent field 0 holds the subnormals m * 2^-9; the all-ones exponent with
mantissa 7 is NaN and there is no infinity, so the largest finite value is
1.75 * 2^8 = 448. Rounding is to nearest, ties to the even mantissa, and a
finite value beyond 448 saturates to 448.

The quantization codes are integers decided in float32: inv = 448 / amax and
y = x * inv are each one correctly rounded float32 operation, then y is
rounded to E4M3. A kernel takes the same steps in the same precision, so its
codes must match bit for bit.
"""
import numpy as np

from .attention import masked_attention_rows

F32 = np.float32
E4M3_MAX = 448.0
_MIN_NORMAL = 2.0 ** -6
_SUB_ULP = 2.0 ** -9


def e4m3_decode(codes):
    """Value of each byte code, float64; NaN for the two NaN codes."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c >> 7, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, m * _SUB_ULP, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return sign * mag


def e4m3_round(y):
    """Nearest E4M3 value to each finite y (ties to the even mantissa), float64.

    Below 2^-6 the grid is the subnormal spacing 2^-9. From 2^e to 2^(e+1)
    (e >= -6) it is 2^(e-3). Division by a power of two is exact in float64,
    so rounding the quotient half-to-even rounds y on that grid. A value that
    rounds up to the next power of two lands on that binade's first point,
    which is also on the finer grid, so the result is the same either way.
    """
    y = np.asarray(y, dtype=np.float64)
    a = np.abs(y)
    _, ex = np.frexp(a)                     # a = f * 2^ex, f in [0.5, 1)
    ulp = np.where(a < _MIN_NORMAL, _SUB_ULP, np.exp2(ex - 1 - 3.0))
    r = np.round(a / ulp) * ulp             # numpy rounds half to even
    r = np.minimum(r, E4M3_MAX)
    return np.copysign(r, y)


def e4m3_encode(y):
    """Byte code of e4m3_round(y), uint8."""
    r = e4m3_round(y)
    a = np.abs(r)
    _, ex = np.frexp(a)
    sub = a < _MIN_NORMAL
    e_field = np.where(sub, 0, ex - 1 + 7)
    m_field = np.where(sub, a / _SUB_ULP, (a / np.exp2(ex - 1.0) - 1.0) * 8.0)
    code = (e_field.astype(np.int64) << 3) | m_field.astype(np.int64)
    code = np.where(np.signbit(r), code | 0x80, code)
    return code.astype(np.uint8)


def quantize_tensor(x):
    """One (batch, head) tensor to E4M3 with one scale: (codes, inv).

    amax = max |x| over the tensor; inv = float32(448) / float32(amax) in
    float32 (inv = 1 for an all-zero tensor); codes = E4M3(float32(x) * inv),
    the product rounded to float32 first. The element of largest magnitude
    maps to +-448.
    """
    xf = np.asarray(x, dtype=F32)
    amax = F32(np.max(np.abs(xf))) if xf.size else F32(0.0)
    inv = F32(1.0) if amax == 0 else F32(F32(E4M3_MAX) / amax)
    y = (xf * inv).astype(F32)
    return e4m3_encode(y), inv


def dequantize(codes, inv):
    """codes / inv in float64: the operand the attention sees."""
    return e4m3_decode(codes) / np.float64(inv)


def fp8_operands(q, k, v):
    """Dequantized Q, K, V of one (batch, head), float64 [N, d] each."""
    return tuple(dequantize(*quantize_tensor(x)) for x in (q, k, v))


def fp8_attention_rows(q, k, v, rows, keep):
    """O [r, d] and LSE [r] of FP8 attention for query tokens ``rows``:
    the exact masked attention (float64) of the dequantized E4M3 operands of
    one (batch, head)."""
    qh, kh, vh = fp8_operands(q, k, v)
    return masked_attention_rows(qh, kh, vh, rows, keep)
