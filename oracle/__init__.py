"""Plain CPU oracle for mask-driven sparse video attention.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package. The product path (the
C-ABI library and its Python binding) never calls it, and it shares no code,
headers, tables or helpers with the CUDA sources.

The oracle computes what the sparse-attention methods on the pages compute,
written out by the plain definition, step by step:

* ``layout``    working-order permutations: 3D tile order (Sliding Tile
                Attention review, key machinery: tokens of a 3D tile kept
                consecutive) and the token-major to frame-major transpose
                (Sparse VideoGen review, key machinery: layout transformation).
* ``masks``     block mean pooling, the SICS score (SPADE review, "What carries
                the argument" and Eqs. 3-5), pooled block scores, Top-K,
                Top-P with a local window (SPADE review, "Core claim"), the
                sliding tile window, spatial/temporal head rules with sinks,
                and the fine-grained M x 1 key-slice threshold (FG-Attn review,
                skeptic critique and referee major comment 2 on Sec. 4.4).
* ``attention`` masked softmax(q k^T / sqrt(d)) v with its log-sum-exp, one
                full score row at a time (the result block-sparse FlashAttention
                with online softmax reaches exactly: SPADE review, axiom ledger,
                "standard math").

Precision: attention is evaluated in float64 from the bf16-rounded inputs.
Mask decisions (pooled means, SICS, scores, softmax of pooled scores, running
Top-P sums, FG scores and threshold) are taken in float32, the precision the
CUDA kernels decide in, so that both sides decide in the same precision.

Every function is pinned in ``tests/test_oracle_*.py`` against something other
than itself: library routines, closed forms, invariants and brute force.
"""
