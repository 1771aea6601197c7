"""Pins the oracle's FP8 E4M3 codec.

Independent checks: the 256 code values from the format's definition,
nearest-value brute force over every bf16 bit pattern, round trips, and
torch's own float8_e4m3fn cast where that cast is defined to agree
(magnitudes up to 448; torch turns larger values into NaN instead of
saturating).
"""
import numpy as np
import pytest
import torch

from oracle import fp8


def _all_bf16_as_f32():
    bits = np.arange(65536, dtype=np.uint32)
    return (bits << 16).view(np.float32)


def _finite_table():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    return codes, fp8.decode(codes)


def _brute_force_encode(x32):
    """Nearest finite E4M3 value by exhaustive search; ties to even code."""
    codes, vals = _finite_table()
    out = np.empty(x32.shape, np.uint8)
    xs = x32.astype(np.float64)
    for i, x in enumerate(xs):
        if np.isnan(x):
            out[i] = 0x7F
            continue
        if np.isinf(x) or abs(x) > 448.0:
            out[i] = 0x7E | (0x80 if x < 0 else 0)
            continue
        # candidates with the sign of x (so -0.0 and tiny negatives keep their sign)
        neg = np.signbit(x)
        sel = (codes & 0x80) == (0x80 if neg else 0)
        cs, vs = codes[sel], vals[sel]
        dist = np.abs(vs - x)
        best = dist.min()
        cand = cs[dist == best]
        if len(cand) > 1:
            cand = cand[(cand & 1) == 0]
        out[i] = cand[0]
    return out


def test_code_values_from_definition():
    assert fp8.decode([0x7E])[0] == 448.0
    assert fp8.decode([0xFE])[0] == -448.0
    assert fp8.decode([0x38])[0] == 1.0
    assert fp8.decode([0x08])[0] == 2.0 ** -6
    assert fp8.decode([0x01])[0] == 2.0 ** -9
    assert fp8.decode([0x07])[0] == 7 * 2.0 ** -9
    assert fp8.decode([0x00])[0] == 0.0 and not np.signbit(fp8.decode([0x00])[0])
    assert fp8.decode([0x80])[0] == 0.0 and np.signbit(fp8.decode([0x80])[0])
    assert np.isnan(fp8.decode([0x7F])[0]) and np.isnan(fp8.decode([0xFF])[0])
    _, vals = _finite_table()
    assert len(vals) == 254 and np.isfinite(vals).all()
    # strictly increasing over non-negative codes 0..0x7E
    pos = fp8.decode(np.arange(0x7F, dtype=np.uint8))
    assert (np.diff(pos) > 0).all()


def test_round_trip_all_codes():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    back = fp8.encode_f32(fp8.decode(codes).astype(np.float32))
    assert (back == codes).all()


def test_encode_matches_brute_force_all_bf16():
    x = _all_bf16_as_f32()
    got = fp8.encode_f32(x)
    want = _brute_force_encode(x)
    nan = np.isnan(x)
    assert fp8.is_nan_code(got[nan]).all()
    assert (got[~nan] == want[~nan]).all()


def test_encode_brute_force_random_fp32():
    g = np.random.default_rng(7)
    x = np.concatenate([
        g.standard_normal(4000).astype(np.float32),
        (g.standard_normal(4000) * 2.0 ** -8).astype(np.float32),
        (g.standard_normal(2000) * 300).astype(np.float32),
    ])
    assert (fp8.encode_f32(x) == _brute_force_encode(x)).all()


def test_ties_to_even_and_saturation():
    # midpoint of 1.0 (0x38, even) and 1.125 (0x39): rounds to 1.0
    assert fp8.encode_f32(np.float32(1.0625))[()] == 0x38
    # midpoint of 1.125 (0x39) and 1.25 (0x3A): rounds to 1.25 (even)
    assert fp8.encode_f32(np.float32(1.1875))[()] == 0x3A
    # midpoint of the largest subnormal 7*2^-9 (odd) and 2^-6 (0x08): goes up
    assert fp8.encode_f32(np.float32(7.5 * 2.0 ** -9))[()] == 0x08
    # half the smallest subnormal: ties to zero
    assert fp8.encode_f32(np.float32(2.0 ** -10))[()] == 0x00
    assert fp8.encode_f32(np.float32(-(2.0 ** -10)))[()] == 0x80
    for v in (448.0, 449.0, 464.0, 480.0, 1e30, np.inf):
        assert fp8.encode_f32(np.float32(v))[()] == 0x7E
        assert fp8.encode_f32(np.float32(-v))[()] == 0xFE
    assert fp8.encode_f32(np.float32(np.nan))[()] == 0x7F


def test_matches_torch_cast_in_range():
    x = _all_bf16_as_f32()
    keep = np.isfinite(x) & (np.abs(x) <= 448.0)
    xs = x[keep]
    ours = fp8.encode_f32(xs)
    ref = torch.from_numpy(xs).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert (ours == ref).all()


@pytest.mark.parametrize("inv", [1.0, 1 / 0.37, 448.0 / 4.75])
def test_quantize_is_fp32_product_then_round(inv):
    g = np.random.default_rng(3)
    x = g.standard_normal(5000).astype(np.float32)
    inv32 = np.float32(inv)
    prod = x * inv32  # numpy float32 * float32: IEEE single, round to nearest
    assert prod.dtype == np.float32
    assert (fp8.quantize(x, inv32) == fp8.encode_f32(prod)).all()
    # dequantised error is bounded by half the grid spacing at |y| (relative 2^-4) times scale
    y = fp8.decode(fp8.quantize(x, inv32)) / float(inv32)
    big = (np.abs(prod) >= 2.0 ** -6) & (np.abs(prod) <= 448.0)
    rel = np.abs(y[big] - x[big]) / np.abs(x[big])
    assert rel.max() <= 2.0 ** -4 * (1 + 1e-6)
