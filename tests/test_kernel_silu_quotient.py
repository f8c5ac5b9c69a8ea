"""Exhaustive CPU proof of an arithmetic shortcut in the SwiGLU backward kernel: silu =
g / d is formed from sig = RN(1/d), which the backward needs anyway, as
q = RN(g sig), t = RN(q d - g) (a fused multiply-add), silu = RN(q - t sig) (a fused
multiply-add), instead of a second IEEE division. For every finite BF16 gate g, with
d = fl32(1 + E(-g)) as the forward producer forms it, this is checked to equal the
correctly rounded quotient, computed here in exact rationals (signed zeros by the IEEE
signed-zero rules)."""
from fractions import Fraction

import numpy as np

from test_oracle_quant import nearest_f32


def _rn(fr: Fraction) -> np.float32:
    return nearest_f32(fr)


def test_corrected_product_is_the_ieee_quotient_for_every_bf16_gate(oracle_mod):
    checked = 0
    for b in range(1 << 16):
        g = np.uint32(b << 16).view(np.float32)
        if not np.isfinite(g):
            continue
        checked += 1
        e = np.float32(oracle_mod.exp_cw(float(-g)))
        d = np.float32(np.float32(1.0) + e)
        sig = _rn(Fraction(1) / Fraction(float(d)))
        q = np.float32(g * sig)
        if g == 0:
            # q = +-0; t = (q d) + (-g) = +0; silu = (-t sig) + q = (-0) + q = q: the sign of g,
            # which is the sign of the IEEE quotient g / d (d >= 1)
            assert q == 0 and np.signbit(q) == np.signbit(g)
            continue
        t = _rn(Fraction(float(q)) * Fraction(float(d)) - Fraction(float(g)))
        silu = _rn(Fraction(float(q)) - Fraction(float(t)) * Fraction(float(sig)))
        ref = _rn(Fraction(float(g)) / Fraction(float(d)))
        assert silu.view(np.uint32) == ref.view(np.uint32), (hex(b), float(g), float(silu), float(ref))
    assert checked == 65280
