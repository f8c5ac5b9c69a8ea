"""Pins of the oracle's FP8 GEMMs (fwd, DGrad, WGrad): exact rational brute force on
tiny shapes, the transposition identities, and an integer special case."""
from fractions import Fraction

import numpy as np
import pytest
import torch

from test_oracle_e4m3 import EXACT
from test_oracle_quant import bits

import workloads


def frac_dot(codes_a, scales_a, codes_b, scales_b):
    """sum_k (sa_k * dec(a_k)) * (sb_k * dec(b_k)) in exact rationals."""
    tot = Fraction(0)
    for ca, sa, cb, sb in zip(codes_a, scales_a, codes_b, scales_b):
        tot += Fraction(float(sa)) * EXACT.get(int(ca), 0) * Fraction(float(sb)) * EXACT.get(int(cb), 0)
    return tot


@pytest.fixture(scope="module")
def tiny(oracle_mod):
    x, w, dy = [bits(t) for t in workloads.tiny_inputs()]
    qx, sx = oracle_mod.quant_act_1x128(x)
    qw, sw, qwT = oracle_mod.quant_weight_128x128(w)
    qdy, sdy, qdyT, sdyc = oracle_mod.transpose_quant_bf16(dy)
    qxT, sxc = oracle_mod.transpose_quant_fp8(qx, sx)
    return dict(qx=qx, sx=sx, qw=qw, sw=sw, qwT=qwT, qdy=qdy, sdy=sdy, qdyT=qdyT,
                sdyc=sdyc, qxT=qxT, sxc=sxc)


def test_fwd_brute_force(oracle_mod, tiny):
    t = tiny
    y, ab = oracle_mod.linear_fwd(t["qx"], t["sx"], t["qw"], t["sw"])
    K = t["qx"].shape[1]
    for (m, n) in [(0, 0), (3, 511), (255, 128), (100, 300)]:
        sa = [t["sx"][k // 128, m] for k in range(K)]
        sb = [t["sw"][n // 128, k // 128] for k in range(K)]
        ref = frac_dot(t["qx"][m], sa, t["qw"][n], sb)
        assert abs(Fraction(float(y[m, n])) - ref) <= abs(ref) * Fraction(1, 2 ** 40) + Fraction(1, 2 ** 80)


def test_dgrad_brute_force(oracle_mod, tiny):
    t = tiny
    dx, _ = oracle_mod.linear_dgrad(t["qdy"], t["sdy"], t["qw"], t["sw"])
    N = t["qdy"].shape[1]
    for (m, k) in [(0, 0), (7, 511), (255, 200)]:
        sa = [t["sdy"][n // 128, m] for n in range(N)]
        sb = [t["sw"][n // 128, k // 128] for n in range(N)]
        ref = frac_dot(t["qdy"][m], sa, t["qw"][:, k], sb)
        assert abs(Fraction(float(dx[m, k])) - ref) <= abs(ref) * Fraction(1, 2 ** 40) + Fraction(1, 2 ** 80)


def test_wgrad_brute_force(oracle_mod, tiny):
    """dW[n,k] = sum over token blocks mb of sdy_c[mb,n]*sx_c[mb,k]*sum_m qdy*qx."""
    t = tiny
    dw, _ = oracle_mod.linear_wgrad(t["qdyT"], t["sdyc"], t["qxT"], t["sxc"])
    M = t["qdyT"].shape[1]
    for (n, k) in [(0, 0), (511, 3), (200, 300)]:
        sa = [t["sdyc"][m // 128, n] for m in range(M)]
        sb = [t["sxc"][m // 128, k] for m in range(M)]
        ref = frac_dot(t["qdyT"][n], sa, t["qxT"][k], sb)
        assert abs(Fraction(float(dw[n, k])) - ref) <= abs(ref) * Fraction(1, 2 ** 40) + Fraction(1, 2 ** 80)


def test_dgrad_is_fwd_with_transposed_weight(oracle_mod, tiny):
    """DGrad computes dY * W: the same numbers as a forward GEMM whose "weight" is W^T
    (rows k, reduction n), with the 128x128 block scales transposed."""
    t = tiny
    dx, ab = oracle_mod.linear_dgrad(t["qdy"], t["sdy"], t["qw"], t["sw"])
    fwd_t, ab_t = oracle_mod.linear_fwd(t["qdy"], t["sdy"], t["qwT"],
                                        np.ascontiguousarray(t["sw"].T))
    assert np.array_equal(dx, fwd_t) or np.allclose(dx, fwd_t, rtol=1e-13, atol=0)
    assert np.allclose(ab, ab_t, rtol=1e-13, atol=0)


def test_wgrad_is_transposed_product(oracle_mod, tiny):
    """WGrad = dY^T X over the 128x1-grouped operands: equal to an explicit fp64 product
    of the transposed dequantized matrices."""
    t = tiny
    dw, _ = oracle_mod.linear_wgrad(t["qdyT"], t["sdyc"], t["qxT"], t["sxc"])
    dyd = oracle_mod.dequant_cols(t["qdyT"], t["sdyc"]).T   # [M, N]
    xd = oracle_mod.dequant_cols(t["qxT"], t["sxc"]).T      # [M, K]
    assert np.allclose(dw, dyd.T @ xd, rtol=1e-13, atol=0)


def test_integer_special_case_exact(oracle_mod):
    """Scales 1 and codes in {-2,...,2}: the sums are integers with |y| <= 2048."""
    rng = np.random.default_rng(13)
    small = {-2: 0xC0, -1: 0xB8, 0: 0x00, 1: 0x38, 2: 0x40}
    va = rng.integers(-2, 3, (64, 512))
    vb = rng.integers(-2, 3, (128, 512))
    qa = np.vectorize(small.get)(va).astype(np.uint8)
    qb = np.vectorize(small.get)(vb).astype(np.uint8)
    sa = np.ones((4, 64), np.float32)
    sb = np.ones((1, 4), np.float32)
    y, ab = oracle_mod.linear_fwd(qa, sa, qb, sb)
    assert np.array_equal(y, (va @ vb.T).astype(np.float64))
    assert np.array_equal(ab, (np.abs(va) @ np.abs(vb).T).astype(np.float64))


def test_scale_placement(oracle_mod):
    """Doubling one activation group's scale doubles exactly that group's contribution;
    a transposed index or a wrong group would move it elsewhere."""
    rng = np.random.default_rng(14)
    qa = rng.integers(0, 0x70, (8, 256)).astype(np.uint8)
    qb = rng.integers(0, 0x70, (128, 256)).astype(np.uint8)
    sa = np.ones((2, 8), np.float32)
    sb = np.ones((1, 2), np.float32)
    y0, _ = oracle_mod.linear_fwd(qa, sa, qb, sb)
    sa2 = sa.copy()
    sa2[1, 5] = 2.0
    y1, _ = oracle_mod.linear_fwd(qa, sa2, qb, sb)
    dec = oracle_mod.e4m3_table()
    part = dec[qa[5, 128:]] @ dec[qb[:, 128:]].T
    assert np.array_equal(np.delete(y1, 5, 0), np.delete(y0, 5, 0))
    assert np.allclose(y1[5] - y0[5], part, rtol=1e-14, atol=0)


def test_bf16_ulp(oracle_mod):
    v = np.array([1.0, 1.5, 2.0, -3.0, 0.0, 2.0 ** -130])
    assert np.array_equal(oracle_mod.bf16_ulp(v), [2.0 ** -7, 2.0 ** -7, 2.0 ** -6, 2.0 ** -6, 0.0, 2.0 ** -137])
