"""OCP FP8 E4M3 codec (oracle).

Test infrastructure only: imported by tests and the benchmark's CPU leg.

"Managing the KV Cache", Quantized KV, names FP8 KV storage with
quantization scales; the format itself is the OCP 8-bit floating point
E4M3 format: 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits, no
infinities, NaN = S.1111.111, largest finite magnitude 1.75 x 2^8 = 448,
smallest normal 2^-6, subnormals m/8 x 2^-6 (so the grid spacing below
2^-5 is 2^-9).

Encoding reading used here (the pages fix only that scales exist):
``code = E4M3(RNE(fp32(x) * inv_scale))`` where the product is one IEEE
fp32 round-to-nearest multiply, the rounding to E4M3 is round to nearest,
ties to even mantissa, and out-of-range magnitudes (including infinity)
saturate to +-448.  NaN encodes as 0x7F.
"""
from __future__ import annotations

import numpy as np

MAX_FINITE = 448.0
NAN_CODE = 0x7F


def decode(codes) -> np.ndarray:
    """E4M3 codes (uint8) to exact float64 values."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, m * 2.0 ** -9, (8 + m) * np.exp2(e.astype(np.float64) - 10.0))
    out = sign * mag
    return np.where((e == 15) & (m == 7), np.nan, out)


def is_nan_code(codes) -> np.ndarray:
    c = np.asarray(codes, dtype=np.uint8)
    return (c & 0x7F) == 0x7F


def encode_f32(x) -> np.ndarray:
    """Round fp32 values to E4M3 codes: nearest, ties to even, saturating.

    The decision is taken on the exact fp32 value (converted to float64
    without loss); division by the power-of-two grid spacing is exact.
    """
    with np.errstate(invalid="ignore"):
        x = np.asarray(x, dtype=np.float32).astype(np.float64)
    sign = np.where(np.signbit(x), 0x80, 0x00).astype(np.int64)
    a = np.abs(x)
    code = np.zeros(a.shape, dtype=np.int64)

    finite_small = np.isfinite(a) & (a < MAX_FINITE) & (a > 0)
    # exponent of the binade holding a: a = f * 2^ex with f in [0.5, 1)
    _, ex = np.frexp(np.where(finite_small, a, 1.0))
    e = np.maximum(ex - 1, -6)                       # binades below 2^-6 share 2^-9 spacing
    quantum = np.exp2((e - 3).astype(np.float64))
    k = np.rint(np.where(finite_small, a, 0.0) / quantum).astype(np.int64)   # half to even
    carry = k == 16                                   # rounded up into the next binade
    e = np.where(carry, e + 1, e)
    k = np.where(carry, 8, k)
    sub = (e == -6) & (k < 8)
    normal_code = ((e + 7) << 3) | (k - 8)
    code = np.where(finite_small, np.where(sub, k, normal_code), code)

    code = np.where(np.isfinite(a) & (a >= MAX_FINITE), 0x7E, code)
    code = np.where(np.isinf(a), 0x7E, code)
    code = code | sign
    code = np.where(np.isnan(a), NAN_CODE, code)
    return code.astype(np.uint8)


def quantize(values_f32, inv_scale_f32) -> np.ndarray:
    """Storage encoding of a KV value: E4M3(fp32(x * inv_scale)).

    `values_f32` and `inv_scale_f32` broadcast; the product is computed in
    IEEE fp32 (numpy float32 multiply, round to nearest).
    """
    y = np.multiply(np.asarray(values_f32, np.float32), np.asarray(inv_scale_f32, np.float32),
                    dtype=np.float32)
    return encode_f32(y)
