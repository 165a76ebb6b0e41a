"""Smooth-field-plus-noise Q/K/V in bf16, generated on the host.

Recipe, per tensor (Q, K, V), per batch item, per head and per channel c:

    field_c(t,h,w) = sum_{s=1..8} a_s * sin(2*pi*(f_t*t/T + f_h*h/H + f_w*w/W) + phi_s)

with a_s ~ N(0,1), each of f_t, f_h, f_w drawn uniformly from {0,1,2} with the
all-zero triple redrawn ("low frequency"), and phi_s ~ U[0, 2*pi). Each channel
is shifted and scaled to zero mean and unit variance over the grid, then
N(0, 0.3^2) noise is added and the value is rounded to bf16 with
round-to-nearest-even. Token order is the original raster order
n = (t*H + h)*W + w.

Random numbers come from numpy's Philox counter-based generator (Salmon et
al., "Parallel random numbers: as easy as 1, 2, 3", SC 2011), keyed by
(workload id, tensor, batch, head), so any head can be regenerated alone.

The sum of sinusoids is evaluated through the angle-addition identity
sin(x + phi) = sin(x)cos(phi) + cos(x)sin(phi): there are only 26 distinct
frequency triples, so every channel is a linear combination of 52 fixed grid
functions, which turns generation into one small matrix product per head.
"""
from concurrent.futures import ThreadPoolExecutor
import os

import numpy as np

N_SINUSOIDS = 8
NOISE_STD = 0.3
_TRIPLES = np.array([(a, b, c) for a in range(3) for b in range(3) for c in range(3)
                     if (a, b, c) != (0, 0, 0)], dtype=np.int64)   # 26 triples


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (round to nearest, ties to even); return the uint16 bits.

    Inputs are finite. The rounding bias is 0x7FFF plus the lowest kept bit.
    """
    b = np.array(x, dtype=np.float32, copy=True).view(np.uint32)
    r = b >> 16
    r &= 1
    r += np.uint32(0x7FFF)
    b += r
    b >>= 16
    return b.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32."""
    return (bits.astype(np.uint32) << 16).view(np.float32)


def _basis(T: int, H: int, W: int) -> np.ndarray:
    """[52, N] float64: sin and cos of the 26 frequency phases over the grid."""
    t = np.arange(T, dtype=np.float64)[:, None, None] / T
    h = np.arange(H, dtype=np.float64)[None, :, None] / H
    w = np.arange(W, dtype=np.float64)[None, None, :] / W
    out = np.empty((2 * len(_TRIPLES), T * H * W), dtype=np.float64)
    for i, (ft, fh, fw) in enumerate(_TRIPLES):
        x = 2.0 * np.pi * (ft * t + fh * h + fw * w)
        out[2 * i] = np.sin(x).reshape(-1)
        out[2 * i + 1] = np.cos(x).reshape(-1)
    return out


def _seed(config_id: int, tensor: int, batch: int, head: int) -> int:
    return (config_id << 40) | (tensor << 32) | (batch << 16) | head


class _Grid:
    """Grid functions of one (T, H, W), shared by every head generated on it."""

    def __init__(self, T: int, H: int, W: int):
        b = _basis(T, H, W)
        self.n_tok = b.shape[1]
        self.basis_t32 = np.ascontiguousarray(b.T, dtype=np.float32)   # [N, 52]
        self.colsum = b.sum(axis=1)                       # [52]
        self.gram = b @ b.T                               # [52, 52]


def _one_head(grid: "_Grid", d: int, key: int) -> np.ndarray:
    rng = np.random.Generator(np.random.Philox(key=key))
    n_trip = len(_TRIPLES)
    coeff = np.zeros((d, 2 * n_trip), dtype=np.float64)
    a = rng.standard_normal((d, N_SINUSOIDS))
    trip = rng.integers(0, n_trip, size=(d, N_SINUSOIDS))
    phi = rng.uniform(0.0, 2.0 * np.pi, size=(d, N_SINUSOIDS))
    rows = np.repeat(np.arange(d), N_SINUSOIDS)
    np.add.at(coeff, (rows, 2 * trip.reshape(-1)), (a * np.cos(phi)).reshape(-1))
    np.add.at(coeff, (rows, 2 * trip.reshape(-1) + 1), (a * np.sin(phi)).reshape(-1))
    # Per-channel mean and variance over the grid from the coefficients:
    # mean = c.(sum_n B[:, n]) / N and E[f^2] = c G c^T / N with G = B B^T.
    n_tok = grid.n_tok
    mean = coeff @ grid.colsum / n_tok
    second = np.einsum("ci,ij,cj->c", coeff, grid.gram, coeff) / n_tok
    std = np.sqrt(np.maximum(second - mean * mean, 0.0))
    std[std == 0] = 1.0
    scale = 1.0 / std
    w = np.ascontiguousarray((coeff * scale[:, None]).T, dtype=np.float32)  # [52, d]
    x = grid.basis_t32 @ w                                                   # [N, d] fp32
    x -= (mean * scale).astype(np.float32)[None, :]
    noise = rng.standard_normal(x.shape, dtype=np.float32)
    noise *= np.float32(NOISE_STD)
    x += noise
    del noise
    return f32_to_bf16_bits(x)                              # [N, d] uint16


def make_qkv(wl, heads=None, threads=None):
    """Return dict q, k, v of uint16 bf16 bits shaped [B, len(heads), N, d].

    ``heads`` selects a subset of heads (default: all); each head's values do
    not depend on which other heads are generated.
    """
    heads = list(range(wl.heads)) if heads is None else list(heads)
    grid = _Grid(wl.T, wl.H, wl.W)
    out = {}
    jobs = []
    for ti, name in enumerate(("q", "k", "v")):
        arr = np.empty((wl.batch, len(heads), wl.N, wl.head_dim), dtype=np.uint16)
        out[name] = arr
        for b in range(wl.batch):
            for j, h in enumerate(heads):
                jobs.append((arr, b, j, _seed(wl.config_id, ti, b, h)))
    nthreads = threads or min(16, os.cpu_count() or 1)

    def run(job):
        arr, b, j, key = job
        arr[b, j] = _one_head(grid, wl.head_dim, key)

    # Each worker runs single-threaded BLAS: nesting a threaded BLAS inside a
    # thread pool oversubscribes many-core hosts badly.
    try:
        from threadpoolctl import threadpool_limits
        limit = threadpool_limits(limits=1, user_api="blas")
    except Exception:
        limit = None
    try:
        if nthreads > 1 and len(jobs) > 1:
            with ThreadPoolExecutor(nthreads) as ex:
                list(ex.map(run, jobs))
        else:
            for job in jobs:
                run(job)
    finally:
        if limit is not None:
            limit.unregister()
    return out
