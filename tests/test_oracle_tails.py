"""Pins of the oracle's partial groups (dimensions that are not multiples of 128).

Reading ("Resumen Técnico: Jet-RL", «Esquema de Cuantización», which fixes the 1x128 and
128x128 groupings and says nothing about sizes that do not divide them): a partial group
is the full group with zeros in the missing places. Zeros raise no maximum, so its scale
comes from its valid elements alone; the codes of the missing places are not stored.

So every quantizer on a ragged tensor must equal the same quantizer on the tensor
zero-padded to whole groups, restricted to the valid region, with the same scales; and
every GEMM on ragged operands must equal the GEMM on the zero-padded operands. RMSNorm
is the exception (padding would change the mean over the row): it is pinned as the
composition of the normalisation over the valid H and the (padded-pinned) 1x128
quantizer."""
import numpy as np
import torch

import workloads
from test_oracle_quant import bits


def pad_to(a: np.ndarray, shape, fill=0):
    out = np.full(shape, fill, dtype=a.dtype)
    out[tuple(slice(0, n) for n in a.shape)] = a
    return out


def up128(n: int) -> int:
    return (n + 127) // 128 * 128


RAGGED = [(200, 300), (129, 144), (37, 16), (256, 400)]


def test_quant_act_tail_equals_zero_padded(oracle_mod):
    for i, (M, K) in enumerate(RAGGED):
        x = bits(workloads.activations_bf16((M, K), 0, 1100 + i, "cpu", outlier_count=3,
                                            outlier_scale=40.0))
        q, s = oracle_mod.quant_act_1x128(x)
        qp, sp = oracle_mod.quant_act_1x128(pad_to(x, (M, up128(K))))
        assert s.shape[0] == (K + 127) // 128
        assert np.array_equal(q, qp[:, :K])
        assert np.array_equal(s.view(np.uint32), sp.view(np.uint32))


def test_quant_weight_tail_equals_zero_padded(oracle_mod):
    for i, (N, K) in enumerate(RAGGED):
        w = bits(workloads.normal_bf16((N, K), 0.02, 0, 1200 + i, "cpu"))
        q, s, qT = oracle_mod.quant_weight_128x128(w)
        qp, sp, _ = oracle_mod.quant_weight_128x128(pad_to(w, (up128(N), up128(K))))
        assert np.array_equal(q, qp[:N, :K])
        assert np.array_equal(qT, q.T)
        assert np.array_equal(s.view(np.uint32), sp.view(np.uint32))


def test_swiglu_tail_equals_zero_padded(oracle_mod):
    # zero gate and up in the padding give h = 0 there
    for i, (M, I) in enumerate(RAGGED):
        g = workloads.normal_bf16((M, I), 2.0, 0, 1300 + i, "cpu")
        u = workloads.normal_bf16((M, I), 1.0, 0, 1400 + i, "cpu")
        q, s, h = oracle_mod.swiglu_quant(bits(torch.cat([g, u], 1)), want_h=True)
        Ip = up128(I)
        gp = torch.zeros((M, Ip), dtype=torch.bfloat16)
        up = torch.zeros((M, Ip), dtype=torch.bfloat16)
        gp[:, :I], up[:, :I] = g, u
        qp, sp = oracle_mod.swiglu_quant(bits(torch.cat([gp, up], 1)))
        assert np.array_equal(q, qp[:, :I])
        assert np.array_equal(s.view(np.uint32), sp.view(np.uint32))
        # and it is the 1x128 quantizer applied to the BF16 SwiGLU output
        qa, sa = oracle_mod.quant_act_1x128(h)
        assert np.array_equal(q, qa) and np.array_equal(s.view(np.uint32), sa.view(np.uint32))


def test_rmsnorm_tail_is_norm_then_quant(oracle_mod):
    for i, (M, H) in enumerate(RAGGED):
        x = bits(workloads.activations_bf16((M, H), 0, 1500 + i, "cpu", outlier_count=2,
                                            outlier_scale=50.0))
        g = bits(workloads.gamma_bf16(H, 0, 1600 + i, "cpu"))
        q, s, y = oracle_mod.rmsnorm_quant(x, g, 1e-5, want_y=True)
        qa, sa = oracle_mod.quant_act_1x128(y)
        assert np.array_equal(q, qa) and np.array_equal(s.view(np.uint32), sa.view(np.uint32))
        # the normalisation runs over the H valid elements of the row: a constant row c
        # has r = 1 / sqrt(c^2 + eps), here with eps = 0 exactly 1/|c|
        xc = np.full(H, bits(torch.tensor([0.5], dtype=torch.bfloat16))[0], np.uint16)
        assert oracle_mod.rmsnorm_rstd(xc, 0.0) == 2.0


def test_transpose_quant_bf16_tails_equal_zero_padded(oracle_mod):
    for i, (M, N) in enumerate(RAGGED):
        dy = bits(workloads.gradients_bf16((M, N), 1e-3, 0, 1700 + i, "cpu"))
        qr, sr, qc, sc = oracle_mod.transpose_quant_bf16(dy)
        Mp, Np = up128(M), up128(N)
        qrp, srp, qcp, scp = oracle_mod.transpose_quant_bf16(pad_to(dy, (Mp, Np)))
        assert np.array_equal(qr, qrp[:M, :N])
        assert np.array_equal(sr[:, :M].view(np.uint32), srp[:, :M].view(np.uint32))
        assert np.array_equal(qc, qcp[:N, :M])
        assert np.array_equal(sc.view(np.uint32), scp[:, :N].view(np.uint32))
        # layout identity: the 128x1 groups of dY are the 1x128 groups of dY^T
        qt, st = oracle_mod.quant_act_1x128(np.ascontiguousarray(dy.T))
        assert np.array_equal(qc, qt)
        assert np.array_equal(sc.view(np.uint32), st[:, :N].view(np.uint32))


def test_transpose_quant_fp8_tails_equal_zero_padded(oracle_mod):
    for i, (M, K) in enumerate(RAGGED):
        x = bits(workloads.activations_bf16((M, K), 0, 1800 + i, "cpu", outlier_count=2,
                                            outlier_scale=30.0))
        q, s = oracle_mod.quant_act_1x128(x)
        qT, sT = oracle_mod.transpose_quant_fp8(q, s)
        Mp, Kp = up128(M), up128(K)
        # zero codes in the padding dequantize to zero whatever their scale
        sp = pad_to(s, (Kp // 128, s.shape[1] + Mp), fill=np.float32(1.0))
        qTp, sTp = oracle_mod.transpose_quant_fp8(pad_to(q, (Mp, Kp)), sp)
        assert np.array_equal(qT, qTp[:K, :M])
        assert np.array_equal(sT.view(np.uint32), sTp[:, :K].view(np.uint32))


def test_gemms_with_tails_equal_zero_padded(oracle_mod):
    rng = np.random.default_rng(5)
    M, N, K = 200, 272, 300
    x = bits(workloads.activations_bf16((M, K), 0, 1900, "cpu", outlier_count=3,
                                        outlier_scale=30.0))
    w = bits(workloads.normal_bf16((N, K), 0.02, 0, 1901, "cpu"))
    dy = bits(workloads.gradients_bf16((M, N), 1e-3, 0, 1902, "cpu"))
    qx, sx = oracle_mod.quant_act_1x128(x)
    qw, sw, _ = oracle_mod.quant_weight_128x128(w)
    qr, sr, qc, scl = oracle_mod.transpose_quant_bf16(dy)
    qxT, sxT = oracle_mod.transpose_quant_fp8(qx, sx)
    Mp, Np, Kp = up128(M), up128(N), up128(K)
    # the fp64 products agree up to fp64 rounding (the library matmul may block the
    # longer padded reduction differently)
    y, ay = oracle_mod.linear_fwd(qx, sx, qw, sw)
    yp, _ = oracle_mod.linear_fwd(pad_to(qx, (M, Kp)), sx, pad_to(qw, (Np, Kp)), sw)
    assert y.shape == (M, N) and np.all(np.abs(y - yp[:, :N]) <= 1e-13 * ay)
    dx, adx = oracle_mod.linear_dgrad(qr, sr, qw, sw)
    dxp, _ = oracle_mod.linear_dgrad(pad_to(qr, (M, Np)), sr, pad_to(qw, (Np, Kp)), sw)
    assert dx.shape == (M, K) and np.all(np.abs(dx - dxp[:, :K]) <= 1e-13 * adx)
    dw, adw = oracle_mod.linear_wgrad(qc, scl, qxT, sxT)
    dwp, _ = oracle_mod.linear_wgrad(pad_to(qc, (N, Mp)), scl, pad_to(qxT, (K, Mp)), sxT)
    assert dw.shape == (N, K) and np.all(np.abs(dw - dwp) <= 1e-13 * adw)
    # a sampled entry of each, by its definition over the valid indices only
    i, j = int(rng.integers(M)), int(rng.integers(N))
    dec = oracle_mod.e4m3_table()
    ref = sum(float(sx[k // 128, i]) * float(sw[j // 128, k // 128]) * dec[qx[i, k]] * dec[qw[j, k]]
              for k in range(K))
    assert abs(y[i, j] - ref) <= 1e-12 * (abs(ref) + 1e-30)
