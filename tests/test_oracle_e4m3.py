"""Pins of the oracle's E4M3 encode/decode and BF16 rounding against things other
than the oracle: the OCP FP8 definition (golden fixture), torch's float8_e4m3fn
conversions (a library routine), and an exact brute-force argmin in Python."""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _finite_codes():
    return [c for c in range(256) if (c & 0x7F) != 0x7F]


def _exact_values():
    """Exact rational value of every finite code, from the OCP definition (independent
    of the oracle): bias 7, E = 0 subnormal."""
    out = {}
    for c in _finite_codes():
        s = -1 if c & 0x80 else 1
        e, m = (c >> 3) & 0xF, c & 7
        v = Fraction(m, 8) * Fraction(2) ** -6 if e == 0 else \
            (1 + Fraction(m, 8)) * Fraction(2) ** (e - 7)
        out[c] = s * v
    return out


EXACT = _exact_values()


def brute_encode(t: float) -> int:
    """argmin over the 253 finite codes of |t - v| (exact), ties to even mantissa,
    saturating; the sign of t is kept for zero."""
    tf = Fraction(float(np.float32(t)))
    neg = math.copysign(1.0, t) < 0
    best, bestd = None, None
    for c, v in EXACT.items():
        if (c & 0x80) != (0x80 if neg else 0):
            continue
        d = abs(tf - v)
        if bestd is None or d < bestd or (d == bestd and (c & 1) == 0 and (best & 1) == 1):
            best, bestd = c, d
    return best


def test_golden_special_values(oracle_mod):
    with open(os.path.join(GOLDEN, "e4m3_special_values.txt")) as f:
        rows = [l.split() for l in f if l.strip() and not l.startswith("#")]
    assert len(rows) >= 10
    for code, val in rows:
        got = oracle_mod.e4m3_decode(int(code, 16))
        if val == "nan":
            assert math.isnan(got), code
        else:
            assert got == float(val) and math.copysign(1, got) == math.copysign(1, float(val)), code


def test_decode_matches_torch_float8(oracle_mod):
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    got = oracle_mod.e4m3_table()
    both_nan = np.isnan(ref) & np.isnan(got)
    assert np.array_equal(np.isnan(ref), np.isnan(got))
    assert np.array_equal(ref[~both_nan], got[~both_nan])
    assert np.array_equal(np.signbit(ref[~both_nan]), np.signbit(got[~both_nan]))


def test_decode_matches_definition(oracle_mod):
    for c, v in EXACT.items():
        assert Fraction(oracle_mod.e4m3_decode(c)) == v


def test_round_trip_all_finite_codes(oracle_mod):
    for c in _finite_codes():
        assert oracle_mod.e4m3_encode(oracle_mod.e4m3_decode(c)) == c


def _probe_points():
    """Every finite value, every midpoint between neighbours, and the fp32 numbers
    one ulp either side of each midpoint (the places a rounding error shows)."""
    mags = sorted({float(v) for c, v in EXACT.items() if not (c & 0x80)})
    pts = set(mags)
    for a, b in zip(mags, mags[1:]):
        mid = np.float32((a + b) / 2)  # exact: the midpoint needs <= 5 bits
        pts.add(float(mid))
        pts.add(float(np.nextafter(mid, np.float32(0))))
        pts.add(float(np.nextafter(mid, np.float32(1e9))))
    for v in (448.0, 449.0, 464.0, 465.0, 480.0, 1e6, 3.0e38):
        pts.add(v)
    pts.add(2.0 ** -10)
    pts.add(float(np.nextafter(np.float32(2.0 ** -10), np.float32(1))))
    pts.add(1e-30)
    return sorted(pts)


def test_encode_brute_force(oracle_mod):
    for t in _probe_points():
        for sgn in (1.0, -1.0):
            v = sgn * t
            assert oracle_mod.e4m3_encode(v) == brute_encode(v), v


def test_encode_random_brute_force(oracle_mod):
    rng = np.random.default_rng(1)
    vals = np.concatenate([rng.standard_normal(300) * 100, rng.standard_normal(300) * 0.01,
                           rng.uniform(-460, 460, 300)]).astype(np.float32)
    for v in vals:
        assert oracle_mod.e4m3_encode(float(v)) == brute_encode(float(v)), v


def test_encode_matches_torch_in_range(oracle_mod):
    """torch's fp32 -> float8_e4m3fn conversion rounds to nearest even; inside the
    finite range it must agree with the oracle on every BF16 bit pattern."""
    bits = np.arange(65536, dtype=np.uint32) << 16
    vals = bits.view(np.float32)
    vals = vals[np.isfinite(vals) & (np.abs(vals) <= 448.0)]
    ref = torch.from_numpy(vals.copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    lib = oracle_mod._load()
    got = np.array([lib.oracle_e4m3_encode(float(v)) for v in vals], np.uint8)
    assert np.array_equal(ref, got)


def test_saturation_and_sign(oracle_mod):
    assert oracle_mod.e4m3_encode(448.0) == 0x7E
    assert oracle_mod.e4m3_encode(1e30) == 0x7E
    assert oracle_mod.e4m3_encode(-1e30) == 0xFE
    assert oracle_mod.e4m3_encode(-1e-6) == 0x80
    assert oracle_mod.e4m3_encode(-0.0) == 0x80
    assert oracle_mod.e4m3_encode(0.0) == 0x00


def test_bf16_rounding_matches_torch(oracle_mod):
    rng = np.random.default_rng(2)
    vals = np.concatenate([
        rng.standard_normal(2000).astype(np.float32),
        (rng.standard_normal(500) * 1e-39).astype(np.float32),   # subnormal range
        np.array([3.389e38, 3.3961e38, 3.4e38, -3.4e38, 1.00390625, 1.01171875], np.float32),
    ])
    # ties: values exactly halfway between BF16 neighbours
    mids = ((rng.integers(0x3F00, 0x4100, 200).astype(np.uint32) << 16) | 0x8000).view(np.float32)
    vals = np.concatenate([vals, mids])
    ref = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle_mod.f32_to_bf16(float(v)) for v in vals], np.uint16)
    assert np.array_equal(ref, got)
