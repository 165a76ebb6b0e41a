"""Seeded synthetic inputs shared by the oracle, the tests and the benchmark.

This package holds workload descriptions and random input generation only. It
contains none of the sparse-attention arithmetic: no layouts, pooling, scores,
masks or softmax. Both the CPU oracle (``oracle/``) and the CUDA path read
inputs made here, so that both sides see identical bits.
"""
from .configs import CONFIGS, Workload, get_config  # noqa: F401
from .fields import make_qkv, bf16_bits_to_f32, f32_to_bf16_bits  # noqa: F401
from .sampling import sample_rows  # noqa: F401
