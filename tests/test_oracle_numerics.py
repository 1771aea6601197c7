"""Pins the oracle's widening of 16-bit storage patterns to float64.

Both formats are decoded here a second way, straight from their definitions
with integer fields and math.ldexp, over all 65,536 patterns:

* IEEE 754 binary16 (fp16): 1 sign bit, 5 exponent bits (bias 15), 10
  fraction bits; exponent 0 = subnormal (fraction x 2^-24), exponent 31 =
  infinity (fraction 0) or NaN;
* bfloat16: the upper 16 bits of an IEEE binary32: 1 sign bit, 8 exponent
  bits (bias 127), 7 fraction bits; exponent 0 = subnormal (fraction x
  2^-133), exponent 255 = infinity or NaN.

Named values worked by hand from the same definitions, and Python's own
binary16 codec (struct format 'e'), pin the decoders themselves.
"""
import math
import struct

import numpy as np

from oracle import numerics

ALL = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)


def fp16_from_fields(b: int) -> float:
    s, e, m = b >> 15, (b >> 10) & 0x1F, b & 0x3FF
    sign = -1.0 if s else 1.0
    if e == 0:
        return sign * math.ldexp(m, -24)
    if e == 31:
        return sign * math.inf if m == 0 else math.nan
    return sign * math.ldexp(1024 + m, e - 25)


def bf16_from_fields(b: int) -> float:
    s, e, m = b >> 15, (b >> 7) & 0xFF, b & 0x7F
    sign = -1.0 if s else 1.0
    if e == 0:
        return sign * math.ldexp(m, -133)
    if e == 255:
        return sign * math.inf if m == 0 else math.nan
    return sign * math.ldexp(128 + m, e - 134)


def _same(got: np.ndarray, want: np.ndarray):
    nan = np.isnan(want)
    assert (np.isnan(got) == nan).all()
    assert (got[~nan] == want[~nan]).all()
    # signed zeros keep their sign
    assert (np.signbit(got[~nan]) == np.signbit(want[~nan])).all()


def test_fp16_values_from_definition():
    got = numerics.bits_to_f64(ALL, "fp16")
    want = np.array([fp16_from_fields(int(b)) for b in ALL])
    _same(got, want)


def test_bf16_values_from_definition():
    got = numerics.bits_to_f64(ALL, "bf16")
    want = np.array([bf16_from_fields(int(b)) for b in ALL])
    _same(got, want)


def test_named_fp16_values():
    named = {
        0x3C00: 1.0,                 # exponent 15 = bias, fraction 0
        0x7BFF: 65504.0,             # largest finite: (2 - 2^-10) x 2^15
        0x0001: 2.0 ** -24,          # smallest subnormal
        0x03FF: 1023 * 2.0 ** -24,   # largest subnormal
        0x0400: 2.0 ** -14,          # smallest normal
        0xC000: -2.0,
        0x3555: 1365 * 2.0 ** -12,   # 0.333251953125, nearest binary16 to 1/3
        0x7C00: math.inf,
        0xFC00: -math.inf,
    }
    got = numerics.bits_to_f64(np.array(list(named), np.uint16), "fp16")
    assert got.tolist() == list(named.values())
    z = numerics.bits_to_f64(np.array([0x8000, 0x0000], np.uint16), "fp16")
    assert z.tolist() == [0.0, 0.0] and np.signbit(z).tolist() == [True, False]
    assert np.isnan(numerics.bits_to_f64(np.array([0x7E00, 0x7C01], np.uint16), "fp16")).all()


def test_named_bf16_values():
    named = {
        0x3F80: 1.0,
        0x3FC0: 1.5,
        0x4049: 3.140625,            # 1.5703125 x 2
        0x7F7F: (2 - 2.0 ** -7) * 2.0 ** 127,
        0x0001: 2.0 ** -133,
        0x0080: 2.0 ** -126,
        0xBF80: -1.0,
        0x7F80: math.inf,
    }
    got = numerics.bits_to_f64(np.array(list(named), np.uint16), "bf16")
    assert got.tolist() == list(named.values())


def test_fp16_agrees_with_python_binary16_codec():
    want = np.array([struct.unpack("<e", struct.pack("<H", int(b)))[0] for b in ALL])
    _same(numerics.bits_to_f64(ALL, "fp16"), want)


def test_decoders_are_pinned_against_each_other():
    # the two field decoders above differ on every normal pattern but +-0:
    # a slip that swapped them would fail the exhaustive tests
    assert fp16_from_fields(0x3C00) == 1.0 and bf16_from_fields(0x3C00) == 2.0 ** -7
    assert bf16_from_fields(0x3F80) == 1.0 and fp16_from_fields(0x3F80) == 1.875


def test_unknown_dtype_is_refused():
    try:
        numerics.bits_to_f64(ALL[:4], "fp8_e4m3")
    except ValueError:
        return
    raise AssertionError("bits_to_f64 accepted a non-16-bit dtype")
