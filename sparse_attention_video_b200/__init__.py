"""B200-native mask-driven sparse attention for video diffusion transformers.

The compute path is the native library ``libsparse_attn.so`` (CUDA kernels for
sm_100a behind the C ABI in ``include/sparse_attn.h``); this package is its
Python binding.
"""
from . import _native  # noqa: F401
from ._native import (SA_EXPORT_BLOCK_BITS, SA_EXPORT_FG_BITS, SA_EXPORT_FG_TAU,  # noqa: F401
                      SA_EXPORT_FG_TILE_KEYS,
                      SA_EXPORT_HEAD_INFO, SA_LAYOUT_FRAME_MAJOR, SA_LAYOUT_IDENTITY,
                      SA_LAYOUT_TILE, SparseAttnError, lib)
from .api import (SparseAttention, make_policy, profile_heads,  # noqa: F401
                  quantize_e4m3, sta_window_search)
