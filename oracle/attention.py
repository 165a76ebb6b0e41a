"""Masked softmax attention by its definition (test infrastructure).

For query token i with kept key set K(i):
    O_i   = sum_{j in K(i)} softmax_j(q_i . k_j / sqrt(d)) v_j
    LSE_i = ln sum_{j in K(i)} exp(q_i . k_j / sqrt(d))
Evaluated in float64 from the bf16-rounded inputs, one full score row per
query: scores against every key, -inf where the mask is 0, max-subtracted
exponentials, their sum, and the division. A row with no kept key has O = 0
and LSE = -inf.

Block-sparse FlashAttention reaches this result exactly up to rounding, since
its online softmax is exact (SPADE review, axiom ledger: FlashAttention-style
online softmax is "standard math"); that is why the oracle needs no blocking.
"""
import math

import numpy as np


def masked_attention_rows(q, k, v, rows, keep):
    """O [r, d] and LSE [r] for query tokens ``rows`` given ``keep`` [r, N] bool."""
    d = q.shape[1]
    s = (q[rows].astype(np.float64) @ k.astype(np.float64).T) / math.sqrt(d)
    s = np.where(keep, s, -np.inf)
    m = s.max(axis=1)
    empty = ~np.isfinite(m)
    m_safe = np.where(empty, 0.0, m)
    p = np.exp(s - m_safe[:, None])
    l = p.sum(axis=1)
    o = np.zeros((len(rows), v.shape[1]), dtype=np.float64)
    ok = ~empty
    o[ok] = (p[ok] @ v.astype(np.float64)) / l[ok][:, None]
    lse = np.full(len(rows), -np.inf)
    lse[ok] = m_safe[ok] + np.log(l[ok])
    return o, lse


def masked_attention_weights(q, k, rows, keep):
    """The softmax weights [r, N] themselves (row-sum pin)."""
    d = q.shape[1]
    s = (q[rows].astype(np.float64) @ k.astype(np.float64).T) / math.sqrt(d)
    s = np.where(keep, s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    p = np.exp(s - m)
    return p / p.sum(axis=1, keepdims=True)


def block_keep_rows(order_blocks, bmask, qb, n_tokens):
    """Query tokens of working block ``qb`` and their [r, N] keep matrix.

    The kept keys of every query token in block qb are the valid tokens of the
    key blocks that bmask[qb] keeps.
    """
    rows = order_blocks[qb][order_blocks[qb] >= 0]
    keys = order_blocks[np.nonzero(bmask[qb])[0]].reshape(-1)
    keys = keys[keys >= 0]
    keep = np.zeros((len(rows), n_tokens), dtype=bool)
    keep[:, keys] = True
    return rows, keep


def block_sparse_attention(q, k, v, order_blocks, bmask, query_blocks=None):
    """O [N, d] (NaN for rows not evaluated) and LSE [N] for one head."""
    n = q.shape[0]
    o = np.full((n, v.shape[1]), np.nan)
    lse = np.full(n, np.nan)
    qbs = range(order_blocks.shape[0]) if query_blocks is None else query_blocks
    for qb in qbs:
        rows, keep = block_keep_rows(order_blocks, bmask, qb, n)
        if len(rows) == 0:
            continue
        o[rows], lse[rows] = masked_attention_rows(q, k, v, rows, keep)
    return o, lse


def slice_attention(q, k, v, keep_groups, group, groups=None):
    """M x 1 slices: query token i keeps the keys its group's row keeps.

    keep_groups is bool [G, N]; group g holds queries [g*M, g*M + M).
    Returns O [N, d] and LSE [N] (NaN for groups not evaluated).
    """
    n = q.shape[0]
    o = np.full((n, v.shape[1]), np.nan)
    lse = np.full(n, np.nan)
    gs = range(keep_groups.shape[0]) if groups is None else groups
    for g in gs:
        rows = np.arange(g * group, min(n, g * group + group))
        keep = np.broadcast_to(keep_groups[g], (len(rows), n))
        o[rows], lse[rows] = masked_attention_rows(q, k, v, rows, keep)
    return o, lse
