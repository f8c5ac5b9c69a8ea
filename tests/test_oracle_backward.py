"""Pins of the oracle's BF16 backward producers (SwiGLU and RMSNorm) against torch
fp64 autograd, closed forms, exact scaling identities and the
independently pinned forward producers. The pages ("Resumen Técnico: Jet-RL",
«Esquema de Cuantización») fix only that gradients between operators stay BF16; the
formulas are the operators' derivatives."""
import numpy as np
import torch

import workloads
from test_oracle_quant import bits, f32_of_bits


def _bf(a) -> np.ndarray:
    """BF16 bits of float values (round to nearest even through torch)."""
    return bits(torch.as_tensor(np.asarray(a, np.float32)).to(torch.bfloat16))


def _f(b) -> np.ndarray:
    return f32_of_bits(np.asarray(b, np.uint16)).astype(np.float64)


def _ulp_bf16(v: np.ndarray) -> np.ndarray:
    a = np.abs(v)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, 2.0 ** (e - 7), 0.0)


# ----------------------------------------------------------------------- SwiGLU backward

def _swiglu_bwd_torch(gu_b: np.ndarray, dh_b: np.ndarray):
    gu = torch.from_numpy(_f(gu_b)).requires_grad_(True)
    I = dh_b.shape[1]
    h = torch.nn.functional.silu(gu[:, :I]) * gu[:, I:]
    h.backward(torch.from_numpy(_f(dh_b)))
    return gu.grad.numpy()


def test_swiglu_bwd_matches_torch_fp64(oracle_mod):
    M, I = 64, 256
    gu = workloads.normal_bf16((M, 2 * I), 2.0, 0, 41, "cpu")
    dh = workloads.normal_bf16((M, I), 1e-2, 0, 42, "cpu")
    got = _f(oracle_mod.swiglu_bwd(bits(gu), bits(dh)))
    ref = _swiglu_bwd_torch(bits(gu), bits(dh))
    # a handful of fp32 roundings before the final BF16 rounding: within one BF16 ulp
    err = np.abs(got - ref)
    assert np.all(err <= _ulp_bf16(ref) + 1e-30), float(np.max(err / (_ulp_bf16(ref) + 1e-30)))
    # and almost always the BF16 rounding of the exact gradient itself
    assert np.mean(got == _f(_bf(ref))) > 0.9


def test_swiglu_bwd_closed_forms(oracle_mod):
    one = int(_bf([1.0])[0])
    for u, dh in ((2.0, 1.0), (-3.0, 0.5), (0.75, -4.0)):
        ub, dhb = int(_bf([u])[0]), int(_bf([dh])[0])
        # g = 0: E(0) = 1, sigma = 1/2, silu = 0 -> d_up = 0, d_gate = dh * u / 2
        dg, du = oracle_mod.swiglu_bwd_one(0, ub, dhb)
        assert _f([du])[0] == 0.0
        assert _f([dg])[0] == dh * u / 2
        # g = 40: E(-40) < 2^-24 so sigma = 1, silu = g: d_up = dh * g, d_gate = dh * u
        gb = int(_bf([40.0])[0])
        dg, du = oracle_mod.swiglu_bwd_one(gb, ub, dhb)
        assert _f([du])[0] == dh * 40.0
        assert _f([dg])[0] == dh * u
    # g = -100: silu and its derivative vanish (tiny, with the sign of g * u * dh)
    dg, du = oracle_mod.swiglu_bwd_one(int(_bf([-100.0])[0]), int(_bf([2.0])[0]), one)
    assert -1e-30 < _f([du])[0] <= 0.0 and -1e-30 < _f([dg])[0] <= 0.0


def test_swiglu_bwd_up_gradient_is_forward_silu(oracle_mod):
    """d_up with dh = 1 is bf16(silu(g)), which the forward producer gives for u = 1."""
    one = int(_bf([1.0])[0])
    gs = bits(workloads.normal_bf16((4096,), 3.0, 0, 43, "cpu"))
    for g in gs[:2048]:
        _, du = oracle_mod.swiglu_bwd_one(int(g), one, one)
        assert du == oracle_mod.swiglu_one(int(g), one)


def test_swiglu_bwd_layout_gate_then_up(oracle_mod):
    M, I = 4, 128
    gu = workloads.normal_bf16((M, 2 * I), 1.0, 0, 44, "cpu")
    dh = workloads.normal_bf16((M, I), 1.0, 0, 45, "cpu")
    dgu = oracle_mod.swiglu_bwd(bits(gu), bits(dh))
    b, d = bits(gu), bits(dh)
    for m in range(M):
        for c in (0, 7, 127):
            dg, du = oracle_mod.swiglu_bwd_one(int(b[m, c]), int(b[m, I + c]), int(d[m, c]))
            assert dgu[m, c] == dg and dgu[m, I + c] == du


def test_swiglu_bwd_dual_is_a6_of_the_gradient(oracle_mod):
    M, I = 256, 256
    gu = workloads.normal_bf16((M, 2 * I), 2.0, 0, 46, "cpu")
    dh = workloads.normal_bf16((M, I), 1e-3, 0, 47, "cpu")
    q, s, qT, sT, dgu = oracle_mod.swiglu_bwd_dual(bits(gu), bits(dh))
    q2, s2, qT2, sT2 = oracle_mod.transpose_quant_bf16(dgu)
    assert np.array_equal(q, q2) and np.array_equal(qT, qT2)
    assert np.array_equal(s, s2) and np.array_equal(sT, sT2)
    assert q.shape == (M, 2 * I) and qT.shape == (2 * I, M)


# ---------------------------------------------------------------------- RMSNorm backward

def _rmsnorm_bwd_torch(x_b, g_b, dy_b, dres_b, eps):
    x = torch.from_numpy(_f(x_b)).requires_grad_(True)
    g = torch.from_numpy(_f(g_b)).requires_grad_(True)
    y = x * torch.rsqrt((x * x).mean(dim=1, keepdim=True) + eps) * g
    y.backward(torch.from_numpy(_f(dy_b)))
    out = x.grad.numpy() + (0.0 if dres_b is None else _f(dres_b))
    return out, g.grad.numpy()


def test_rmsnorm_bwd_matches_torch_fp64(oracle_mod):
    M, H, eps = 48, 512, 1e-5
    x = workloads.activations_bf16((M, H), 0, 51, "cpu", outlier_count=3, outlier_scale=20.0)
    g = workloads.gamma_bf16(H, 0, 52, "cpu")
    dy = workloads.gradients_bf16((M, H), 1e-3, 0, 53, "cpu")
    dres = workloads.gradients_bf16((M, H), 1e-3, 0, 54, "cpu")
    out, dgamma, r, k = oracle_mod.rmsnorm_bwd(bits(x), bits(g), bits(dy), bits(dres), eps)
    ref, ref_dg = _rmsnorm_bwd_torch(bits(x), bits(g), bits(dy), bits(dres), eps)
    got = _f(out)
    # two BF16 roundings (dx, then dx + dres) and fp32 steps whose error is relative to
    # the terms r*gamma*dy and k*x before they cancel
    xf, gf, dyf = _f(bits(x)), _f(bits(g)), _f(bits(dy))
    rr = r.astype(np.float64)[:, None]
    terms = np.abs(rr * gf * dyf) + np.abs(k.astype(np.float64)[:, None] * xf)
    tol = 2 * _ulp_bf16(ref) + 2 * _ulp_bf16(terms) + 1e-30
    assert np.all(np.abs(got - ref) <= tol)
    assert np.mean(np.abs(got - ref) <= _ulp_bf16(ref)) > 0.9  # two BF16 roundings
    # dgamma: fp32 products summed in fp64
    scale = np.abs(_f(bits(dy)) * xf * rr).sum(axis=0)
    assert np.all(np.abs(dgamma - ref_dg) <= 4e-7 * scale + 1e-30)
    # r is the forward producer's reciprocal RMS
    for m in (0, 17, M - 1):
        assert r[m] == np.float32(oracle_mod.rmsnorm_rstd(bits(x)[m], eps))


def test_rmsnorm_bwd_constant_rows_closed_form(oracle_mod):
    """x = 1, gamma = 1, eps = 0: r = 1 and dx = dy - mean(dy) (exact for these dy)."""
    M, H = 4, 128
    x = np.full((M, H), int(_bf([1.0])[0]), np.uint16)
    g = np.full(H, int(_bf([1.0])[0]), np.uint16)
    rng = np.random.default_rng(55)
    dyv = rng.integers(-8, 9, size=(M, H)).astype(np.float64)
    dyv[:, 0] -= dyv.sum(axis=1) - 64 * np.sign(dyv.sum(axis=1))  # mean = +-1/2 or 0
    dyv[:, 0] = np.clip(dyv[:, 0], -200, 200)
    mean = dyv.mean(axis=1, keepdims=True)
    out, dgamma, r, k = oracle_mod.rmsnorm_bwd(x, g, _bf(dyv), None, 0.0)
    assert np.all(r == 1.0)
    assert np.array_equal(_f(out), dyv - mean)
    assert np.array_equal(dgamma.astype(np.float64), dyv.sum(axis=0))


def test_rmsnorm_bwd_exact_scaling(oracle_mod):
    """eps = 0: x -> 2x halves out exactly; dy -> 2dy doubles out and dgamma exactly."""
    M, H = 16, 256
    x = workloads.activations_bf16((M, H), 0, 56, "cpu")
    g = workloads.gamma_bf16(H, 0, 57, "cpu")
    dy = workloads.gradients_bf16((M, H), 1e-3, 0, 58, "cpu")
    xb, gb, dyb = bits(x), bits(g), bits(dy)
    out, dg, _, _ = oracle_mod.rmsnorm_bwd(xb, gb, dyb, None, 0.0)
    out2x, dg2x, _, _ = oracle_mod.rmsnorm_bwd(_bf(2 * _f(xb)), gb, dyb, None, 0.0)
    out2d, dg2d, _, _ = oracle_mod.rmsnorm_bwd(xb, gb, _bf(2 * _f(dyb)), None, 0.0)
    assert np.array_equal(_f(out2x), _f(out) / 2)
    assert np.array_equal(dg2x, dg)  # x r is unchanged
    assert np.array_equal(_f(out2d), 2 * _f(out))
    assert np.array_equal(dg2d, 2 * dg)


def test_rmsnorm_bwd_orthogonal_to_x(oracle_mod):
    """eps = 0: the exact dx is orthogonal to x (sum_j x_j dx_j = 0); the BF16 result is
    within its rounding."""
    M, H = 8, 1024
    x = workloads.activations_bf16((M, H), 0, 59, "cpu")
    g = workloads.gamma_bf16(H, 0, 60, "cpu")
    dy = workloads.gradients_bf16((M, H), 1.0, 0, 61, "cpu")
    out, _, _, _ = oracle_mod.rmsnorm_bwd(bits(x), bits(g), bits(dy), None, 0.0)
    xf, of = _f(bits(x)), _f(out)
    dot = (xf * of).sum(axis=1)
    bound = (np.abs(xf) * (_ulp_bf16(of) + 1e-6 * np.abs(of))).sum(axis=1)
    assert np.all(np.abs(dot) <= bound)


def test_rmsnorm_bwd_residual_is_a_bf16_add(oracle_mod):
    """out = bf16(dx + dres) with dx the BF16 gradient without the residual: the same as
    torch's BF16 addition of the two."""
    M, H = 16, 256
    x = workloads.activations_bf16((M, H), 0, 62, "cpu")
    g = workloads.gamma_bf16(H, 0, 63, "cpu")
    dy = workloads.gradients_bf16((M, H), 1e-3, 0, 64, "cpu")
    dres = workloads.gradients_bf16((M, H), 1e-3, 0, 65, "cpu")
    dx, _, _, _ = oracle_mod.rmsnorm_bwd(bits(x), bits(g), bits(dy), None, 1e-5)
    out, _, _, _ = oracle_mod.rmsnorm_bwd(bits(x), bits(g), bits(dy), bits(dres), 1e-5)
    dxt = torch.from_numpy(dx.view(np.int16)).view(torch.bfloat16)
    assert np.array_equal(out, bits(dxt + dres))


def test_rmsnorm_bwd_dual_is_a6_of_the_output(oracle_mod):
    M, H = 256, 384
    x = workloads.activations_bf16((M, H), 0, 66, "cpu")
    g = workloads.gamma_bf16(H, 0, 67, "cpu")
    dy = workloads.gradients_bf16((M, H), 1e-3, 0, 68, "cpu")
    out, q, s, qT, sT, dgamma = oracle_mod.rmsnorm_bwd_dual(bits(x), bits(g), bits(dy), None,
                                                            1e-5)
    q2, s2, qT2, sT2 = oracle_mod.transpose_quant_bf16(out)
    assert np.array_equal(q, q2) and np.array_equal(qT, qT2)
    assert np.array_equal(s, s2) and np.array_equal(sT, sT2)
    assert dgamma.shape == (H,)


# ------------------------------------------------- exact reductions of the RMSNorm backward
# The two reductions (c per row, dgamma per column) are exact sums of fp32 terms rounded
# once, so no summation order enters them. Pinned against math.fsum (the correctly
# rounded double of an exact sum) and exact rational arithmetic.
import math  # noqa: E402
from fractions import Fraction  # noqa: E402


def _hard_sums():
    """fp32 term sets that break naive summation: cancellation, wide exponent spread,
    subnormals, ties of the final rounding, long runs."""
    rng = np.random.default_rng(1234)
    f = np.float32
    sets = [
        np.array([1.0, 2.0 ** -24], f),                      # exactly halfway in fp32
        np.array([1.0, 2.0 ** -24, 2.0 ** -60], f),          # just above halfway
        np.array([1.0, -2.0 ** -24, -2.0 ** -70], f),        # just below halfway, negative
        np.array([2.0 ** 100, 1.0, -2.0 ** 100], f),         # total cancellation of the big part
        np.array([3.0, -3.0], f),                            # exact zero
        np.array([2.0 ** -149, 2.0 ** -149, 3 * 2.0 ** -149], f),   # subnormals
        np.array([2.0 ** 127, 2.0 ** 127, -2.0 ** 127], f),  # beyond fp32 range midway
        np.array([1.0 + 2.0 ** -23] * 7 + [-7.0], f),
    ]
    for k in range(12):
        n = int(rng.integers(2, 3000))
        v = rng.standard_normal(n).astype(np.float64)
        e = rng.integers(-140, 100, n) if k % 3 == 0 else rng.integers(-40, 10, n)
        t = (v * 2.0 ** e).astype(f)
        if k % 4 == 1:  # a large pair that cancels, so the small terms decide
            t = np.concatenate([t, np.array([2.0 ** 90, -2.0 ** 90], f)])
        rng.shuffle(t)
        sets.append(t)
    return sets


def _nearest_f32(S: Fraction) -> float:
    """The fp32 nearest to the rational S (ties to even), from exact comparisons."""
    guess = np.float32(float(S))
    cands = {float(guess), float(np.nextafter(guess, np.float32(np.inf))),
             float(np.nextafter(guess, np.float32(-np.inf)))}
    best = min(cands, key=lambda c: (abs(Fraction(c) - S),
                                     int(np.float32(c).view(np.uint32)) & 1))
    return best


def test_exact_sum_equals_fsum(oracle_mod):
    for t in _hard_sums():
        got = oracle_mod.exact_sum_f32(t)
        ref = math.fsum(float(v) for v in t)
        assert got == ref, (t[:4], got, ref)


def test_exact_sum_rounds_once_to_fp32(oracle_mod):
    for t in _hard_sums():
        S = sum((Fraction(float(v)) for v in t), Fraction(0))
        got = oracle_mod.exact_sum_f32(t, to_f32=True)
        assert got == _nearest_f32(S), (t[:4], got)
    # the double-rounding trap: 1 + 2^-24 + 2^-60 rounds up in one step (to 1 + 2^-23),
    # while rounding to a double first would land on the tie and go down to 1
    t = np.array([1.0, 2.0 ** -24, 2.0 ** -60], np.float32)
    assert oracle_mod.exact_sum_f32(t, to_f32=True) == 1.0 + 2.0 ** -23


def test_exact_sum_is_order_free_and_zero_is_positive(oracle_mod):
    rng = np.random.default_rng(7)
    for t in _hard_sums():
        a = oracle_mod.exact_sum_f32(t)
        b = oracle_mod.exact_sum_f32(t[rng.permutation(t.size)])
        assert a == b
    z = oracle_mod.exact_sum_f32(np.array([5.0, -2.5, -2.5], np.float32))
    assert z == 0.0 and math.copysign(1.0, z) == 1.0


def _rms_bwd_case(M=48, H=384, seed=0):
    x = workloads.activations_bf16((M, H), seed, 61, "cpu", outlier_frac=0.02, outlier_scale=50)
    dy = workloads.gradients_bf16((M, H), 1e-3, seed, 62, "cpu")
    g = workloads.gamma_bf16(H, seed, 63, "cpu")
    return bits(x), bits(dy), bits(g)


def test_rmsnorm_bwd_k_uses_the_exact_row_sum(oracle_mod):
    xb, dyb, gb = _rms_bwd_case()
    M, H = xb.shape
    _, _, r, k = oracle_mod.rmsnorm_bwd(xb, gb, dyb, None, 1e-5)
    x32, dy32, g32 = (f32_of_bits(b).astype(np.float32) for b in (xb, dyb, gb))
    for m in range(M):
        terms = (g32 * dy32[m]) * x32[m]          # fp32 products, IEEE, as the reading says
        c = math.fsum(float(t) for t in terms)
        rd = float(r[m])
        kd = ((c * rd) * rd) * rd / H
        assert np.float32(kd) == k[m], m


def test_rmsnorm_bwd_dgamma_is_the_exact_column_sum(oracle_mod):
    xb, dyb, gb = _rms_bwd_case(M=64, H=256, seed=1)
    _, dgamma, r, _ = oracle_mod.rmsnorm_bwd(xb, gb, dyb, None, 1e-5)
    x32, dy32 = (f32_of_bits(b).astype(np.float32) for b in (xb, dyb))
    terms = dy32 * (x32 * r[:, None].astype(np.float32))   # fl32(dy * fl32(x * r))
    for j in range(0, 256, 5):
        S = sum((Fraction(float(v)) for v in terms[:, j]), Fraction(0))
        assert float(dgamma[j]) == _nearest_f32(S), j
