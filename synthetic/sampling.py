"""Seeded query-row samples (inputs of the head profiler).

The profiler of the Sparse VideoGen review (key machinery) decides each head's
pattern from a random 1 % of its query rows. The draw itself is an input here:
per head, ``ceil(fraction * N)`` distinct token indices from a numpy PCG64
stream seeded by (seed, head), returned in ascending order (the profiler's
result does not depend on the order; ascending token order keeps the rows of
one frame together).
"""
import math

import numpy as np


def sample_rows(n_tokens: int, heads: int, fraction: float = 0.01, seed: int = 0) -> np.ndarray:
    """int32 [heads, n_rows] ascending token indices, n_rows = ceil(fraction * n_tokens)."""
    n_rows = max(1, min(n_tokens, math.ceil(fraction * n_tokens)))
    out = np.empty((heads, n_rows), dtype=np.int32)
    for h in range(heads):
        g = np.random.default_rng([seed, h])
        out[h] = np.sort(g.choice(n_tokens, size=n_rows, replace=False)).astype(np.int32)
    return out
