"""Pins of the oracle's group quantizers (1x128, 128x128, 128x1 and the transposed
requantizer) against the mathematics: exact round trips, the half-ulp bound, a
hand-worked group, an independent exact re-derivation, and layout identities."""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from test_oracle_e4m3 import EXACT, brute_encode

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def f32_of_bits(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32)


def nearest_f32(fr: Fraction) -> np.float32:
    """Correctly rounded fp32 of an exact rational (ties to even), independent of C."""
    c = np.float32(float(fr))
    cands = [c, np.nextafter(c, np.float32(-np.inf)), np.nextafter(c, np.float32(np.inf))]
    cands = [x for x in cands if np.isfinite(x)]
    best = None
    for x in cands:
        d = abs(Fraction(float(x)) - fr)
        if best is None or d < best[0] or (d == best[0] and (int(np.float32(x).view(np.uint32)) & 1) == 0):
            best = (d, x)
    return np.float32(best[1])


def exact_group(vals: np.ndarray):
    """Independent derivation of one group: s = RN32(amax/448), t = RN32(x/s), brute enc."""
    amax = max(abs(float(v)) for v in vals)
    s = np.float32(1.0) if amax == 0 else nearest_f32(Fraction(amax) / 448)
    codes = [brute_encode(float(nearest_f32(Fraction(float(v)) / Fraction(float(s)))))
             if v != 0 else (0x80 if math.copysign(1, float(v)) < 0 else 0) for v in vals]
    return s, np.array(codes, np.uint8)


def test_worked_group(oracle_mod):
    rows = []
    with open(os.path.join(GOLDEN, "quant_group_worked.txt")) as f:
        for l in f:
            if l.startswith("# scale"):
                scale = float(l.split()[2])
            elif l.strip() and not l.startswith("#"):
                i, v, c = l.split()
                rows.append((int(i), float(v), int(c, 16)))
    x = np.zeros((1, 128), np.float32)
    for i, v, _ in rows:
        x[0, i] = v
    xb = bits(torch.from_numpy(x).to(torch.bfloat16))
    q, s = oracle_mod.quant_act_1x128(xb)
    assert s[0, 0] == np.float32(scale)
    for i, _, c in rows:
        assert q[0, i] == c, (i, hex(q[0, i]), hex(c))


def test_exact_round_trip_scaled_codes(oracle_mod):
    """Groups built as c_i * 2^e, with c_i E4M3 values including +-448, quantize to
    s = 2^e and codes c_i exactly."""
    rng = np.random.default_rng(3)
    finite = [c for c in range(256) if (c & 0x7F) != 0x7F]
    for e in (-20, -7, 0, 5, 30):
        codes = rng.choice(finite, size=(4, 128)).astype(np.uint8)
        codes[:, 0] = rng.choice([0x7E, 0xFE], size=4)
        vals = np.array([[float(EXACT[c]) for c in row] for row in codes]) * 2.0 ** e
        # values with <= 4 significant bits and exponent in range are exact in BF16
        xb = bits(torch.from_numpy(vals.astype(np.float32)).to(torch.bfloat16))
        assert np.array_equal(f32_of_bits(xb).astype(np.float64), vals)
        q, s = oracle_mod.quant_act_1x128(xb)
        assert np.all(s[0, :4] == np.float32(2.0 ** e))
        # -0 and +0 both decode to 0: compare values, and signs where nonzero
        dec = oracle_mod.e4m3_table()
        assert np.array_equal(dec[q], dec[codes])


def test_zero_group_and_negative_zero(oracle_mod):
    x = np.zeros((2, 256), np.float32)
    x[0, 5] = -0.0
    x[1, 128:] = np.linspace(-1, 1, 128)
    x[1, 130] = -0.0
    xb = bits(torch.from_numpy(x).to(torch.bfloat16))
    xb[0, 5] = 0x8000
    xb[1, 130] = 0x8000
    q, s = oracle_mod.quant_act_1x128(xb)
    assert s[0, 0] == 1.0 and s[1, 0] == 1.0
    assert q[0, 5] == 0x80 and np.all(np.delete(q[0], 5) == 0)
    assert q[1, 130] == 0x80


def test_half_ulp_invariant_all_quantizers(oracle_mod):
    """|t - dec(q)| <= half an E4M3 ulp at t (2^-10 in the subnormal range): for every
    element, with t = fl32(x/s), i.e. |x - s*dec(q)| <= s*(ulp/2) + |x|*2^-24."""
    x, w, dy = [bits(t) for t in __import__("workloads").tiny_inputs()]

    def check(xv, sv, q):
        xv = xv.astype(np.float64)
        dec = oracle_mod.e4m3_table()[q]
        a = np.abs(xv / sv)
        e = np.floor(np.log2(np.maximum(a, 2.0 ** -6)))
        half_ulp = np.where(a < 2.0 ** -6, 2.0 ** -10, 2.0 ** (e - 4))
        sat = a > 448
        err = np.abs(xv - sv * dec)
        bound = sv * half_ulp + np.abs(xv) * 2.0 ** -24
        assert np.all((err <= bound) | sat)
        assert np.all(np.abs(dec) <= 448)

    q, s = oracle_mod.quant_act_1x128(x)
    check(f32_of_bits(x), np.repeat(s[:, :256].T, 128, axis=1), q)
    qw, sw, qwT = oracle_mod.quant_weight_128x128(w)
    check(f32_of_bits(w), np.kron(sw, np.ones((128, 128))), qw)
    _, _, qc, sc = oracle_mod.transpose_quant_bf16(dy)
    check(f32_of_bits(dy).T, np.repeat(sc.T, 128, axis=1), qc)
    # a8: the requantized values of the saved activation
    xh = oracle_mod.dequant_rows(q, s).astype(np.float32)  # fl32(s*dec) == exact here
    qT, sT = oracle_mod.transpose_quant_fp8(q, s)
    check(xh.T, np.repeat(sT.T, 128, axis=1), qT)


def test_group_max_reaches_448(oracle_mod):
    x, _, _ = [bits(t) for t in __import__("workloads").tiny_inputs()]
    q, s = oracle_mod.quant_act_1x128(x)
    xv = np.abs(f32_of_bits(x)).reshape(256, 4, 128)
    arg = xv.argmax(-1)
    qg = q.reshape(256, 4, 128)
    top = np.take_along_axis(qg, arg[..., None], -1)[..., 0]
    assert np.all((top & 0x7F) == 0x7E)


def test_brute_force_small_groups(oracle_mod):
    """Exact re-derivation (Fractions) of random groups, including subnormal-range
    scales and values that round across E4M3 binades."""
    rng = np.random.default_rng(4)
    for trial in range(6):
        scale = [1.0, 1e-3, 3e4, 1e-30, 0.37, 5e-39][trial]
        v = (rng.standard_normal((1, 128)) * scale).astype(np.float32)
        xb = bits(torch.from_numpy(v).to(torch.bfloat16))
        q, s = oracle_mod.quant_act_1x128(xb)
        s_ref, q_ref = exact_group(f32_of_bits(xb)[0])
        assert s[0, 0] == s_ref
        assert np.array_equal(q[0], q_ref)


def test_weight_block_brute_force_and_transpose(oracle_mod):
    rng = np.random.default_rng(5)
    w = (rng.standard_normal((256, 128)) * 0.02).astype(np.float32)
    w[3, 7] = 0.9  # one large value dominates block 0 only
    wb = bits(torch.from_numpy(w).to(torch.bfloat16))
    q, s, qT = oracle_mod.quant_weight_128x128(wb)
    assert s.shape == (2, 1)
    assert np.array_equal(qT, q.T)
    for nb in range(2):
        blk = f32_of_bits(wb)[nb * 128:(nb + 1) * 128].reshape(-1)
        amax = np.abs(blk).max()
        assert s[nb, 0] == nearest_f32(Fraction(float(amax)) / 448)
        sub = blk[::97]
        codes = [brute_encode(float(nearest_f32(Fraction(float(v)) / Fraction(float(s[nb, 0])))))
                 for v in sub]
        assert np.array_equal(q[nb * 128:(nb + 1) * 128].reshape(-1)[::97], codes)


def test_column_groups_equal_row_groups_of_transpose(oracle_mod):
    """Layout independence: 128x1 groups of dY equal 1x128 groups of dY^T, and the
    row-wise half of the dual quantizer equals the 1x128 quantizer."""
    _, _, dy = __import__("workloads").tiny_inputs()
    dyb = bits(dy)
    q_row, s_row, q_colT, s_col = oracle_mod.transpose_quant_bf16(dyb)
    qa, sa = oracle_mod.quant_act_1x128(dyb)
    assert np.array_equal(q_row, qa) and np.array_equal(s_row, sa)
    qt, st = oracle_mod.quant_act_1x128(np.ascontiguousarray(dyb.T), lds=dyb.shape[1])
    assert np.array_equal(q_colT, qt)
    assert np.array_equal(s_col, st[:, : dyb.shape[1]])


def test_fp8_requant_of_representable_columns(oracle_mod):
    """When every 1x128 row scale is 1 and every 128x1 column group already holds an
    element of magnitude 448, the requantizer must return the same codes, transposed,
    with scale 1."""
    rng = np.random.default_rng(6)
    finite = [c for c in range(256) if (c & 0x7F) != 0x7F]
    q = rng.choice(finite, size=(256, 256)).astype(np.uint8)
    q[0, :] = 0x7E
    q[128, :] = 0xFE
    s = np.ones((2, 256), np.float32)
    qT, sT = oracle_mod.transpose_quant_fp8(q, s)
    assert np.all(sT == 1.0)
    dec = oracle_mod.e4m3_table()
    assert np.array_equal(dec[qT], dec[q.T])


def test_fp8_requant_brute_force(oracle_mod):
    rng = np.random.default_rng(7)
    x = (rng.standard_normal((128, 128)) * np.exp(rng.uniform(-3, 3, (1, 128)))).astype(np.float32)
    xb = bits(torch.from_numpy(x).to(torch.bfloat16))
    q, s = oracle_mod.quant_act_1x128(xb)
    qT, sT = oracle_mod.transpose_quant_fp8(q, s)
    for k in (0, 17, 127):
        col = [nearest_f32(Fraction(float(s[0, m])) * EXACT.get(int(q[m, k]), 0)) for m in range(128)]
        col = np.array(col, np.float32)
        # an E4M3 zero keeps its sign
        col = np.where(q[:, k] == 0x80, np.float32(-0.0), col)
        s_ref, q_ref = exact_group(col)
        assert sT[0, k] == s_ref
        assert np.array_equal(qT[k], q_ref)
