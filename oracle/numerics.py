"""Storage dtypes to float64 (oracle).

Test infrastructure only: imported by tests and the benchmark's CPU leg.

bf16 is the upper half of an IEEE binary32; fp16 is IEEE binary16.  Both
widen to float64 exactly.
"""
from __future__ import annotations

import numpy as np


def bits_to_f64(bits, dtype: str) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16)
    if dtype == "bf16":
        return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    if dtype == "fp16":
        return b.view(np.float16).astype(np.float64)
    raise ValueError(f"not a 16-bit float dtype: {dtype!r}")


def bits_to_f32(bits, dtype: str) -> np.ndarray:
    """Same widening, stopping at fp32 (exact for both formats)."""
    return bits_to_f64(bits, dtype).astype(np.float32)
