"""The FP8 requantizer (a8) forms t = fl32(x / s) for fp32 x and s as
t = fl32(x * fl64(1 / s)), the product taken in fp64, instead of an fp32 IEEE division.

Why this equals the IEEE quotient: write x = X 2^a and s = S 2^b with 24-bit integer
significands, and let m = P 2^c be an fp32 rounding midpoint (P odd, 25 bits). x - m s
is a nonzero multiple of 2^min(a, b + c): it cannot vanish, since P odd and P >= 2^24 > X
rule out X 2^j = P S. So x / s stays at least ~2^-49 (relative) away from every fp32
midpoint, while the fp64 product is within ~2^-52 of x / s; rounding it to fp32 therefore
lands where the exact quotient rounds. The test checks the identity on CPU over random
operands of every magnitude the requantizer meets, over quotients built to sit as close
to midpoints as fp32 allows, and over subnormal divisors and results. It checks the
kernel's arithmetic identity only and shares nothing with the oracle."""
import numpy as np


def fp64_quot(x: np.ndarray, s: np.ndarray) -> np.ndarray:
    r = 1.0 / s.astype(np.float64)
    return (x.astype(np.float64) * r).astype(np.float32)


def ieee_quot(x: np.ndarray, s: np.ndarray) -> np.ndarray:
    return (x / s).astype(np.float32)   # numpy float32 division is IEEE, round to nearest


def test_random_operands():
    rng = np.random.default_rng(0)
    for _ in range(20):
        s = (rng.random(500_000) + 0.5).astype(np.float32) * np.float32(2.0) ** rng.integers(
            -140, 60, 500_000).astype(np.float32)
        s = s.astype(np.float32)
        x = (s.astype(np.float64) * rng.uniform(-448.0, 448.0, s.size)).astype(np.float32)
        assert np.array_equal(fp64_quot(x, s).view(np.uint32), ieee_quot(x, s).view(np.uint32))


def test_quotients_next_to_midpoints():
    # x = fl32(m s) for midpoints m between adjacent fp32 values: the exact quotient then
    # lies as close to a midpoint as fp32 operands allow
    rng = np.random.default_rng(1)
    for _ in range(20):
        q = rng.uniform(1.0, 448.0, 500_000).astype(np.float32)
        mid = q.astype(np.float64) + np.spacing(q).astype(np.float64) / 2
        s = (rng.random(q.size) + 0.5).astype(np.float32) * np.float32(2.0) ** rng.integers(
            -100, 30, q.size).astype(np.float32)
        s = s.astype(np.float32)
        x = (mid * s.astype(np.float64)).astype(np.float32)
        for xx in (x, np.nextafter(x, np.float32(np.inf)), np.nextafter(x, np.float32(-np.inf))):
            assert np.array_equal(fp64_quot(xx, s).view(np.uint32), ieee_quot(xx, s).view(np.uint32))


def test_subnormal_scales_and_signed_zero():
    s = np.array([1e-45, 3e-41, 2 ** -126, 7e-39], np.float32)
    for k in range(-20, 20):
        x = (s.astype(np.float64) * (k * 13.7)).astype(np.float32)
        assert np.array_equal(fp64_quot(x, s).view(np.uint32), ieee_quot(x, s).view(np.uint32))
    z = fp64_quot(np.array([-0.0, 0.0], np.float32), np.array([0.5, 0.5], np.float32))
    assert np.array_equal(z.view(np.uint32), np.array([-0.0, 0.0], np.float32).view(np.uint32))
