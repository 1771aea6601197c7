"""Seeded synthetic inputs for the paged decode-attention path.

This module is shared by the tests, the benchmark and the smoke check. It
holds only random draws and their packing into the storage dtypes (bf16 /
fp16 bit patterns, the fp8 calibration scales); none of the method's own
arithmetic (no block tables, no slot mapping, no attention, no fp8 encoding)
lives here, so both the CUDA path and the oracle can consume it without
sharing any code with each other.
"""
from .configs import (  # noqa: F401
    WORKLOADS,
    Workload,
    workload,
)
from .gen import (  # noqa: F401
    Purpose,
    fp8_scales,
    normal_bits,
    prefill_kv_bits,
    prefix_kv_bits,
    rng,
    step_kv_bits,
    step_q_bits,
)
