"""Pins of the oracle's fused RMSNorm+quantize and SwiGLU+quantize against closed
forms, library routines in fp64 (torch / math) and limits."""
import math

import numpy as np
import torch

from test_oracle_quant import bits, f32_of_bits


def _ulp32(x: float) -> float:
    x = np.float32(abs(x))
    return float(np.nextafter(x, np.float32(np.inf)) - x)


def test_exp_within_two_ulp_of_libm(oracle_mod):
    xs = np.concatenate([np.linspace(-80, 88, 20011), np.linspace(-1, 1, 4001),
                         np.array([0.0, 1e-8, -1e-8, 0.5 * math.log(2), -0.5 * math.log(2)])])
    worst = 0.0
    for x in xs.astype(np.float32):
        got = oracle_mod.exp_cw(float(x))
        ref = math.exp(float(x))
        err = abs(got - ref) / _ulp32(ref)
        worst = max(worst, err)
    assert worst <= 2.0, worst


def test_exp_exact_points(oracle_mod):
    assert oracle_mod.exp_cw(0.0) == 1.0
    # clamped ends: E(x) = E(-80) below -80 and E(88) above 88
    assert oracle_mod.exp_cw(-1000.0) == oracle_mod.exp_cw(-80.0)
    assert oracle_mod.exp_cw(1000.0) == oracle_mod.exp_cw(88.0)
    assert math.isfinite(oracle_mod.exp_cw(88.0))


def test_rmsnorm_constant_rows_closed_form(oracle_mod):
    """x_i = c (a power of two), eps = 0: mean(x^2) = c^2, r = 1/|c| exactly, so
    y_i = sign(c) * gamma_i, and each group's codes are those of gamma."""
    H = 256
    g = torch.linspace(0.5, 1.5, H).to(torch.bfloat16)
    for c in (1.0, -4.0, 2.0 ** -20, 2.0 ** 30):
        x = torch.full((3, H), c).to(torch.bfloat16)
        q, s, y = oracle_mod.rmsnorm_quant(bits(x), bits(g), eps=0.0, want_y=True)
        r = oracle_mod.rmsnorm_rstd(bits(x)[0], 0.0)
        assert r == np.float32(1.0 / abs(c))
        expect = (torch.sign(torch.tensor(c)) * g.float()).to(torch.bfloat16)
        assert np.array_equal(y, np.tile(bits(expect), (3, 1)))
        qg, sg = oracle_mod.quant_act_1x128(np.tile(bits(expect), (3, 1)))
        assert np.array_equal(q, qg) and np.array_equal(s, sg)


def test_rmsnorm_scale_invariance(oracle_mod):
    """With eps = 0, multiplying a row by 2^k leaves the normalised row unchanged."""
    x = torch.randn(4, 384, generator=torch.Generator().manual_seed(9)).to(torch.bfloat16)
    g = torch.ones(384).to(torch.bfloat16)
    _, _, y0 = oracle_mod.rmsnorm_quant(bits(x), bits(g), eps=0.0, want_y=True)
    _, _, y1 = oracle_mod.rmsnorm_quant(bits(x * 2.0 ** 12), bits(g), eps=0.0, want_y=True)
    assert np.array_equal(y0, y1)


def test_rmsnorm_matches_torch_fp64(oracle_mod):
    gen = torch.Generator().manual_seed(10)
    x = (torch.randn(64, 512, generator=gen) * 3).to(torch.bfloat16)
    g = (1 + 0.1 * torch.randn(512, generator=gen)).to(torch.bfloat16)
    _, _, y = oracle_mod.rmsnorm_quant(bits(x), bits(g), eps=1e-5, want_y=True)
    ref = torch.nn.functional.rms_norm(x.double(), (512,), g.double(), eps=1e-5).numpy()
    got = f32_of_bits(y).astype(np.float64)
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref), 1e-30))) - 7)
    # BF16 rounding (1/2 ulp) plus two fp32 products and fp32 r (a few 2^-24)
    assert np.all(np.abs(got - ref) <= 0.5 * ulp + np.abs(ref) * 2.0 ** -21)


def test_swiglu_matches_torch_fp64(oracle_mod):
    gen = torch.Generator().manual_seed(11)
    gu = (torch.randn(32, 512, generator=gen) * 4).to(torch.bfloat16)
    _, _, h = oracle_mod.swiglu_quant(bits(gu), want_h=True)
    gd = gu[:, :256].double()
    ud = gu[:, 256:].double()
    ref = (torch.nn.functional.silu(gd) * ud).numpy()
    got = f32_of_bits(h).astype(np.float64)
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref), 1e-30))) - 7)
    assert np.all(np.abs(got - ref) <= 0.5 * ulp + np.abs(ref) * 2.0 ** -20)


def test_swiglu_limits(oracle_mod):
    """silu(0) = 0; for g >= 17, 1 + e^-g == 1 in fp32 so h = bf16(g*u) exactly;
    for g <= -100, h rounds to a signed zero or a tiny value of sign -u."""
    one = 0x3F80  # BF16 1.0
    zero = 0x0000
    assert oracle_mod.swiglu_one(zero, one) == 0
    for gval, uval in ((17.0, 1.5), (40.0, -3.0), (1000.0, 0.25)):
        gb = oracle_mod.f32_to_bf16(gval)
        ub = oracle_mod.f32_to_bf16(uval)
        expect = oracle_mod.f32_to_bf16(np.float32(oracle_mod.bf16_to_f32(gb)) *
                                        np.float32(oracle_mod.bf16_to_f32(ub)))
        assert oracle_mod.swiglu_one(gb, ub) == expect
    hneg = oracle_mod.bf16_to_f32(oracle_mod.swiglu_one(oracle_mod.f32_to_bf16(-100.0), one))
    assert abs(hneg) < 1e-35 and math.copysign(1, hneg) < 0


def test_swiglu_layout_gate_then_up(oracle_mod):
    """Columns 0..I-1 are the gate, I..2I-1 the up projection: swapping the halves
    changes the result (the function is not symmetric)."""
    gen = torch.Generator().manual_seed(12)
    gu = torch.randn(2, 256, generator=gen).to(torch.bfloat16)
    _, _, h = oracle_mod.swiglu_quant(bits(gu), want_h=True)
    g = bits(gu)[0, 3]
    u = bits(gu)[0, 128 + 3]
    assert h[0, 3] == oracle_mod.swiglu_one(int(g), int(u))
    assert h[0, 3] != oracle_mod.swiglu_one(int(u), int(g)) or g == u


def _bf16_rne_bits(v: np.ndarray) -> np.ndarray:
    """fp32 values -> BF16 bit patterns, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(v, np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def test_rmsnorm_dual_emission_pins(oracle_mod):
    """Option B for the RMSNorm producer: rows are the single-output producer's codes;
    columns (128x1 along tokens, transposed) equal the 1x128 quantization of y^T, a
    layout identity against the separately pinned activation quantizer; and the returned
    r regenerates y as bf16(fl32(fl32(x r) g))."""
    x = torch.randn(256, 384, generator=torch.Generator().manual_seed(41)).to(torch.bfloat16)
    x[:, 17] *= 40.0
    g = (1.0 + 0.1 * torch.randn(384, generator=torch.Generator().manual_seed(42))).to(torch.bfloat16)
    q, s, qT, sT, r = oracle_mod.rmsnorm_quant_dual(bits(x), bits(g), 1e-5)
    q1, s1, y = oracle_mod.rmsnorm_quant(bits(x), bits(g), 1e-5, want_y=True)
    assert np.array_equal(q, q1) and np.array_equal(s.view(np.uint32), s1.view(np.uint32))
    qa, sa = oracle_mod.quant_act_1x128(np.ascontiguousarray(y.T))
    assert np.array_equal(qT, qa)
    assert np.array_equal(sT.view(np.uint32), sa[:, :384].view(np.uint32))
    xf = f32_of_bits(bits(x)).astype(np.float32)
    gf = f32_of_bits(bits(g)).astype(np.float32)
    yy = _bf16_rne_bits((xf * r[:, None].astype(np.float32)).astype(np.float32) * gf)
    assert np.array_equal(yy, y)


def test_swiglu_dual_emission_pins(oracle_mod):
    gu = (1.5 * torch.randn(128, 512, generator=torch.Generator().manual_seed(43))).to(torch.bfloat16)
    q, s, qT, sT = oracle_mod.swiglu_quant_dual(bits(gu))
    q1, s1, h = oracle_mod.swiglu_quant(bits(gu), want_h=True)
    assert np.array_equal(q, q1) and np.array_equal(s.view(np.uint32), s1.view(np.uint32))
    qa, sa = oracle_mod.quant_act_1x128(np.ascontiguousarray(h.T))
    assert np.array_equal(qT, qa)
    assert np.array_equal(sT.view(np.uint32), sa[:, :256].view(np.uint32))


def test_saved_activation_option_b_accuracy(oracle_mod, capsys):
    """Saved-activation groupings for WGrad ("Resumen Técnico: Jet-RL", «Esquema de
    Cuantización»: 1x128 in the forward pass, 128x1 for WGrad). Option A requantizes the
    saved 1x128 codes into 128x1 groups (two roundings); option B quantizes the BF16
    value once per grouping. On these seeded inputs B's WGrad error against the exact
    fp64 product of the BF16 operands is not above A's; the figures are printed."""
    import workloads
    cases = ((512, 512, 256, 0.005, 50.0, 3000), (512, 512, 256, 0.0, 1.0, 3010))
    for M, K, N, frac, scale, seed in cases:
        x = workloads.activations_bf16((M, K), 0, seed, "cpu", outlier_frac=frac,
                                       outlier_scale=scale)
        dy = workloads.gradients_bf16((M, N), 1e-3, 0, seed + 1, "cpu")
        xb, dyb = bits(x), bits(dy)
        exact = dy.double().numpy().T @ x.double().numpy()
        _, _, qdyT, sdyc = oracle_mod.transpose_quant_bf16(dyb, want_row=False)
        qa, sa = oracle_mod.quant_act_1x128(xb)
        qaT, saT = oracle_mod.transpose_quant_fp8(qa, sa)
        _, _, qbT, sbT = oracle_mod.transpose_quant_bf16(xb, want_row=False)
        ra, _ = oracle_mod.linear_wgrad(qdyT, sdyc, qaT, saT)
        rb, _ = oracle_mod.linear_wgrad(qdyT, sdyc, qbT, sbT)
        ea = np.linalg.norm(ra - exact) / np.linalg.norm(exact)
        eb = np.linalg.norm(rb - exact) / np.linalg.norm(exact)
        with capsys.disabled():
            print(f"\n[{M}x{K}x{N} outliers {frac}] WGrad rel. error: option A {ea:.3e}, "
                  f"option B {eb:.3e}")
        assert 0.0 < eb <= ea < 0.1
