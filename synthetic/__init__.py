"""Seeded synthetic inputs for MiniMax Sparse Attention.

This module only draws numbers: it holds none of the method's arithmetic, and
both the CUDA library's tests/benchmark and the CPU oracle consume the bytes it
produces (the oracle after a device-to-host copy).
"""
from .inputs import (WORKLOADS, Workload, bf16_bits, make_inputs, make_workload,  # noqa: F401
                     quantize_e4m3_rows, ragged_lens)
