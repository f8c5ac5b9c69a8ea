"""Backward producers with the gradient quantizer fused behind them, against the oracle
through the C ABI, bit for bit: the SwiGLU backward (gradient, codes, scales) and the
RMSNorm backward (BF16 gradient, its codes and scales both ways, dgamma: the reductions
are exact sums rounded once on both sides); the full-size Llama-3.1-8B shapes on sampled
128-row blocks and dgamma over all rows."""
import numpy as np
import pytest
import torch

import workloads
from gpu_util import assert_codes_equal, assert_scales_equal, bits, np_f32

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def fq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import fp8_block_scaled_08_b200 as f
    return f


def _swiglu_inputs(M, I, seed):
    gu = workloads.normal_bf16((M, 2 * I), 2.0, 0, seed, DEV)
    dh = workloads.gradients_bf16((M, I), 1e-3, 0, seed + 1, DEV, small_row_frac=0.02,
                                  small_row_scale=1e-6)
    # saturated, vanishing and signed-zero gates, a zero gradient column
    gu[:, 3] = 40.0
    gu[:, 4] = -100.0
    gu[:, 5] = 0.0
    gu[:, 6] = -0.0
    gu[:, I + 9] = 0.0
    dh[:, 11] = 0.0
    return gu, dh


@pytest.mark.parametrize("M,I", [(128, 128), (256, 384), (384, 256), (128, 1024)])
def test_swiglu_bwd_dual_matches_oracle(fq, oracle_mod, M, I):
    gu, dh = _swiglu_inputs(M, I, 3000 + M + I)
    q, s, qT, sT, dgu = fq.swiglu_bwd_quant_dual_alloc(gu, dh, want_dgu=True)
    torch.cuda.synchronize()
    rq, rs, rqT, rsT, rdgu = oracle_mod.swiglu_bwd_dual(bits(gu), bits(dh))
    g = bits(dgu)
    if not np.array_equal(g, rdgu):
        bad = np.argwhere(g != rdgu)
        i = tuple(bad[0])
        raise AssertionError("dgu: %d mismatches, first at %s: gpu %#x oracle %#x" % (
            len(bad), i, g[i], rdgu[i]))
    assert_codes_equal(q, rq, "swiglu bwd rows")
    assert_scales_equal(s, rs, "swiglu bwd row scales", cols=M)
    assert_codes_equal(qT, rqT, "swiglu bwd columns")
    assert_scales_equal(sT, rsT, "swiglu bwd column scales")


def test_swiglu_bwd_dual_without_bf16_output(fq, oracle_mod):
    M, I = 256, 256
    gu, dh = _swiglu_inputs(M, I, 3100)
    q, s, qT, sT, dgu = fq.swiglu_bwd_quant_dual_alloc(gu, dh, want_dgu=False)
    torch.cuda.synchronize()
    assert dgu is None
    rq, rs, rqT, rsT, _ = oracle_mod.swiglu_bwd_dual(bits(gu), bits(dh))
    assert_codes_equal(q, rq, "swiglu bwd rows (no dgu)")
    assert_codes_equal(qT, rqT, "swiglu bwd columns (no dgu)")
    assert_scales_equal(sT, rsT, "swiglu bwd column scales (no dgu)")


def _rms_inputs(M, H, seed, with_res):
    x = workloads.activations_bf16((M, H), 0, seed, DEV, outlier_frac=0.005, outlier_scale=50.0)
    g = workloads.gamma_bf16(H, 0, seed + 1, DEV)
    dy = workloads.gradients_bf16((M, H), 1e-3, 0, seed + 2, DEV, small_row_frac=0.02,
                                  small_row_scale=1e-4)
    dres = workloads.gradients_bf16((M, H), 1e-3, 0, seed + 3, DEV) if with_res else None
    return x, g, dy, dres


def _check_rms(fq, oracle_mod, x, g, dy, dres, eps, out, q, s, qT, sT, dg, what):
    """Bit for bit against the oracle chain: the BF16 gradient, its codes and scales both
    ways (the oracle quantizing its own gradient), and dgamma (exact sums on both sides)."""
    M, H = x.shape
    rout, rq, rs, rqT, rsT, rdg = oracle_mod.rmsnorm_bwd_dual(
        bits(x), bits(g), bits(dy), None if dres is None else bits(dres), eps)
    got = bits(out)
    if not np.array_equal(got, rout):
        bad = np.argwhere(got != rout)
        i = tuple(bad[0])
        raise AssertionError("%s: %d gradient mismatches, first at %s: gpu %#x oracle %#x" % (
            what, len(bad), i, got[i], rout[i]))
    assert_codes_equal(q, rq, what + " rows")
    assert_scales_equal(s, rs, what + " row scales", cols=M)
    assert_codes_equal(qT, rqT, what + " columns")
    assert_scales_equal(sT, rsT, what + " column scales")
    gd = np_f32(dg)
    if not np.array_equal(gd.view(np.uint32), rdg.view(np.uint32)):
        bad = np.flatnonzero(gd.view(np.uint32) != rdg.view(np.uint32))
        raise AssertionError("%s: %d dgamma mismatches, first at %d: gpu %r oracle %r" % (
            what, len(bad), bad[0], gd[bad[0]], rdg[bad[0]]))


@pytest.mark.parametrize("M,H,eps,with_res", [(128, 128, 1e-5, True), (256, 512, 1e-5, False),
                                              (384, 640, 1e-6, True), (256, 3584, 0.0, True),
                                              (128, 6144, 1e-5, True)])
def test_rmsnorm_bwd_dual_matches_oracle(fq, oracle_mod, M, H, eps, with_res):
    x, g, dy, dres = _rms_inputs(M, H, 3200 + M + H, with_res)
    out, q, s, qT, sT, dg = fq.rmsnorm_bwd_quant_dual_alloc(x, g, dy, dres, eps)
    torch.cuda.synchronize()
    _check_rms(fq, oracle_mod, x, g, dy, dres, eps, out, q, s, qT, sT, dg,
               "rmsnorm bwd %dx%d" % (M, H))


def test_rmsnorm_bwd_dual_repeatable_and_workspace_reuse(fq):
    """Two calls on one workspace give bit-identical results (exact reductions)."""
    M, H = 256, 1024
    x, g, dy, dres = _rms_inputs(M, H, 3300, True)
    a = fq.rmsnorm_bwd_quant_dual_alloc(x, g, dy, dres, 1e-5)
    b = fq.rmsnorm_bwd_quant_dual_alloc(x, g, dy, dres, 1e-5)
    torch.cuda.synchronize()
    for u, v in zip(a, b):
        assert torch.equal(u.view(torch.uint8) if u.dtype != torch.uint8 else u,
                           v.view(torch.uint8) if v.dtype != torch.uint8 else v)


def test_rmsnorm_bwd_rejects_small_workspace(fq):
    M, H = 128, 128
    x, g, dy, _ = _rms_inputs(M, H, 3400, False)
    out = torch.empty_like(x)
    q = torch.empty((M, H), dtype=torch.uint8, device=DEV)
    s = torch.empty((H // 128, M), dtype=torch.float32, device=DEV)
    qT = torch.empty((H, M), dtype=torch.uint8, device=DEV)
    sT = torch.empty((M // 128, H), dtype=torch.float32, device=DEV)
    ws = torch.empty(fq.rmsnorm_bwd_workspace_bytes(M, H) - 16, dtype=torch.uint8, device=DEV)
    with pytest.raises(fq.Fp8qError):
        fq.rmsnorm_bwd_quant_dual(x, g, dy, None, 1e-5, out, q, s, qT, sT, None, ws)


def test_full_size_llama_backward_producers_sampled(fq, oracle_mod):
    """Llama-3.1-8B layer at M = 8192: SwiGLU backward (I = 14336) and RMSNorm backward
    (H = 4096, with the residual gradient) checked on one random 128-row block each;
    dgamma over all rows against the oracle's full sum."""
    wl = workloads.LLAMA_LAYER
    M, H, I = wl.tokens, wl.layer.hidden, wl.layer.intermediate
    rng = np.random.default_rng(7)
    gu, dh = _swiglu_inputs(M, I, 3500)
    q, s, qT, sT, dgu = fq.swiglu_bwd_quant_dual_alloc(gu, dh, want_dgu=True)
    torch.cuda.synchronize()
    mb = int(rng.integers(0, M // 128))
    blk = slice(mb * 128, mb * 128 + 128)
    rq, rs, rqT, rsT, rdgu = oracle_mod.swiglu_bwd_dual(bits(gu[blk]), bits(dh[blk]))
    assert np.array_equal(bits(dgu[blk]), rdgu)
    assert_codes_equal(q[blk], rq, "full swiglu bwd rows")
    assert_codes_equal(qT[:, blk], rqT, "full swiglu bwd columns")
    assert np.array_equal(np_f32(sT[mb:mb + 1]).view(np.uint32), rsT.view(np.uint32))
    del gu, dh, q, s, qT, sT, dgu
    x, g, dy, dres = _rms_inputs(M, H, 3600, True)
    out, q, s, qT, sT, dg = fq.rmsnorm_bwd_quant_dual_alloc(x, g, dy, dres, wl.eps)
    torch.cuda.synchronize()
    mb = int(rng.integers(0, M // 128))
    blk = slice(mb * 128, mb * 128 + 128)
    rout, oq, _, oqT, osT, _ = oracle_mod.rmsnorm_bwd_dual(
        bits(x[blk]), bits(g), bits(dy[blk]), bits(dres[blk]), wl.eps)
    assert np.array_equal(bits(out[blk]), rout)
    assert_codes_equal(q[blk], oq, "full rmsnorm bwd rows")
    assert_codes_equal(qT[:, blk], oqT, "full rmsnorm bwd columns")
    assert np.array_equal(np_f32(sT[mb:mb + 1]).view(np.uint32), osT.view(np.uint32))
    # dgamma sums over all 8192 rows: the oracle's exact sums, bit for bit
    _, rdg, _, _ = oracle_mod.rmsnorm_bwd(bits(x), bits(g), bits(dy), None, wl.eps)
    assert np.array_equal(np_f32(dg).view(np.uint32), rdg.view(np.uint32))


def test_rmsnorm_bwd_degenerate_rows(fq, oracle_mod):
    """A zero input row (r = 1/sqrt(eps), c = 0: dx = r gamma dy), a zero gradient row
    (dx = 0, out = dres), a zero residual gradient, one row block (M = 128)."""
    M, H, eps = 128, 1024, 1e-5
    x, g, dy, dres = _rms_inputs(M, H, 3700, True)
    x[3] = 0.0
    dy[7] = 0.0
    dy[9] = -0.0
    dres[11] = 0.0
    out, q, s, qT, sT, dg = fq.rmsnorm_bwd_quant_dual_alloc(x, g, dy, dres, eps)
    torch.cuda.synchronize()
    _check_rms(fq, oracle_mod, x, g, dy, dres, eps, out, q, s, qT, sT, dg, "degenerate rows")
    assert torch.equal(out[7].float(), dres[7].float())


def test_swiglu_bwd_dual_every_bf16_gate(fq, oracle_mod):
    """Every BF16 bit pattern as a gate (128 x 512 of them) with fixed up and dh values:
    the gradient and its codes bit for bit. Patterns of magnitude 2^127 and up (and the
    non-finite ones) are replaced by zero: with dh = -1.5 their products leave fp32's
    range, and non-finite values are outside the contract."""
    M, I = 128, 512
    pats = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    exp = (pats >> 7) & 0xFF
    pats[exp >= 0xFE] = 0
    gate = torch.from_numpy(pats.view(np.int16).reshape(M, I)).view(torch.bfloat16).to(DEV)
    up = torch.full((M, I), 0.75, dtype=torch.bfloat16, device=DEV)
    gu = torch.cat([gate, up], dim=1).contiguous()
    dh = torch.full((M, I), -1.5, dtype=torch.bfloat16, device=DEV)
    q, s, qT, sT, dgu = fq.swiglu_bwd_quant_dual_alloc(gu, dh, want_dgu=True)
    torch.cuda.synchronize()
    rq, rs, rqT, rsT, rdgu = oracle_mod.swiglu_bwd_dual(bits(gu), bits(dh))
    assert np.array_equal(bits(dgu), rdgu)
    assert_codes_equal(q, rq, "every gate rows")
    assert_codes_equal(qT, rqT, "every gate columns")
    assert_scales_equal(sT, rsT, "every gate column scales")
