"""Option B for the saved activations (producers emit both groupings from BF16): the
RMSNorm and SwiGLU dual producers against the oracle compositions (codes, scales and the
reciprocal RMS bit for bit), their row outputs against the single-output producers, the
full-size Llama-3.1-8B shapes on sampled rows / 128-row blocks, and a WGrad fed by the
dual codes against the fp64 oracle."""
import numpy as np
import pytest
import torch

import workloads
from gpu_util import assert_codes_equal, assert_gemm_close, assert_scales_equal, bits, np_f32, np_u8

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def fq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import fp8_block_scaled_08_b200 as f
    return f


@pytest.mark.parametrize("M,H,eps", [(256, 512, 1e-5), (384, 3584, 1e-6), (128, 128, 0.0),
                                     (256, 6144, 1e-5)])
def test_rmsnorm_dual_matches_oracle(fq, oracle_mod, M, H, eps):
    x = workloads.activations_bf16((M, H), 0, 2000 + M, DEV, outlier_frac=0.005,
                                   outlier_scale=50.0)
    g = workloads.gamma_bf16(H, 0, 2001, DEV)
    q, s, qT, sT, r = fq.rmsnorm_quant_dual_alloc(x, g, eps)
    torch.cuda.synchronize()
    rq, rs, rqT, rsT, rr = oracle_mod.rmsnorm_quant_dual(bits(x), bits(g), eps)
    assert_codes_equal(q, rq, "dual rmsnorm rows")
    assert_scales_equal(s, rs, "dual rmsnorm row scales", cols=M)
    assert_codes_equal(qT, rqT, "dual rmsnorm columns")
    assert_scales_equal(sT, rsT, "dual rmsnorm column scales")
    assert np.array_equal(np_f32(r).view(np.uint32), rr.view(np.uint32))
    q1, s1 = fq.rmsnorm_quant_alloc(x, g, eps)
    assert torch.equal(q, q1) and torch.equal(s[:, :M], s1[:, :M])


@pytest.mark.parametrize("M,I", [(256, 384), (128, 1024), (384, 256)])
def test_swiglu_dual_matches_oracle(fq, oracle_mod, M, I):
    gu = workloads.normal_bf16((M, 2 * I), 1.5, 0, 2100 + M, DEV)
    gu[:, 5] = 0.0
    gu[:, I + 7] = -0.0
    q, s, qT, sT = fq.swiglu_quant_dual_alloc(gu)
    torch.cuda.synchronize()
    rq, rs, rqT, rsT = oracle_mod.swiglu_quant_dual(bits(gu))
    assert_codes_equal(q, rq, "dual swiglu rows")
    assert_scales_equal(s, rs, "dual swiglu row scales", cols=M)
    assert_codes_equal(qT, rqT, "dual swiglu columns")
    assert_scales_equal(sT, rsT, "dual swiglu column scales")
    q1, s1 = fq.swiglu_quant_alloc(gu)
    assert torch.equal(q, q1) and torch.equal(s[:, :M], s1[:, :M])


def test_full_size_llama_dual_producers_sampled(fq, oracle_mod):
    """Llama-3.1-8B layer at M = 8192: RMSNorm (H = 4096) and SwiGLU (I = 14336) dual
    producers; 16 random rows and one random 128-row block checked against the oracle."""
    wl = workloads.LLAMA_LAYER
    rng = np.random.default_rng(5)
    inp = workloads.layer_inputs(wl, DEV, with_grads=False)
    M, H, I = wl.tokens, wl.layer.hidden, wl.layer.intermediate
    q, s, qT, sT, r = fq.rmsnorm_quant_dual_alloc(inp["x_mlp"], inp["gamma2"], wl.eps)
    gu = workloads.normal_bf16((M, 2 * I), 1.5, wl.seed, 700, DEV)
    hq, hs, hqT, hsT = fq.swiglu_quant_dual_alloc(gu)
    torch.cuda.synchronize()
    rows = torch.from_numpy(np.sort(rng.choice(M, 16, replace=False))).to(DEV)
    xr = bits(inp["x_mlp"][rows])
    rq, rs = oracle_mod.rmsnorm_quant(xr, bits(inp["gamma2"]), wl.eps)
    rr = np.array([oracle_mod.rmsnorm_rstd(xr[i], wl.eps) for i in range(len(xr))], np.float32)
    assert_codes_equal(q[rows], rq, "full rmsnorm dual rows")
    assert np.array_equal(np_f32(s[:, rows]).view(np.uint32), rs[:, :16].view(np.uint32))
    assert np.array_equal(np_f32(r[rows]).view(np.uint32), rr.view(np.uint32))
    mb = int(rng.integers(0, M // 128))
    blk = slice(mb * 128, mb * 128 + 128)
    _, _, rqT, rsT, _ = oracle_mod.rmsnorm_quant_dual(bits(inp["x_mlp"][blk]), bits(inp["gamma2"]),
                                                      wl.eps)
    assert_codes_equal(qT[:, blk], rqT, "full rmsnorm dual columns")
    assert np.array_equal(np_f32(sT[mb:mb + 1]).view(np.uint32), rsT.view(np.uint32))
    rq2, rs2, rqT2, rsT2 = oracle_mod.swiglu_quant_dual(bits(gu[blk]))
    assert_codes_equal(hq[blk], rq2, "full swiglu dual rows")
    assert_codes_equal(hqT[:, blk], rqT2, "full swiglu dual columns")
    assert np.array_equal(np_f32(hsT[mb:mb + 1]).view(np.uint32), rsT2.view(np.uint32))


def test_wgrad_from_dual_codes(fq, oracle_mod):
    """WGrad fed by the dual producer's 128x1 codes (no FP8 requantization) against the
    fp64 oracle on the same operands."""
    M, H, N = 256, 512, 384
    x = workloads.activations_bf16((M, H), 0, 2200, DEV, outlier_count=4, outlier_scale=30.0)
    g = workloads.gamma_bf16(H, 0, 2201, DEV)
    dy = workloads.gradients_bf16((M, N), 1e-3, 0, 2202, DEV)
    _, _, qT, sT, _ = fq.rmsnorm_quant_dual_alloc(x, g, 1e-5)
    _, _, qdyT, sdyc = fq.transpose_quant_bf16_alloc(dy, want_row=False)
    dw = fq.linear_wgrad_alloc(qdyT, sdyc, qT, sT)
    torch.cuda.synchronize()
    ref, ab = oracle_mod.linear_wgrad(np_u8(qdyT), np_f32(sdyc), np_u8(qT), np_f32(sT))
    assert_gemm_close(dw.float().cpu().numpy(), ref, ab, "wgrad from dual codes")


def test_swiglu_dual_every_bf16_gate(fq, oracle_mod):
    """Every BF16 gate below 2^61 in magnitude once (the kernel tabulates the gate factor
    for 2^-24 <= |g| < 2^7 and computes it directly elsewhere), up values from N(0, 1):
    both groupings bit for bit."""
    pats = np.arange(65536, dtype=np.uint32)
    pats = pats[((pats >> 7) & 0xFF) < 127 + 61].astype(np.uint16)
    pats = np.resize(pats, 512 * 128)
    g = torch.from_numpy(pats.view(np.int16).reshape(512, 128).copy()).view(torch.bfloat16)
    u = workloads.normal_bf16((512, 128), 1.0, 0, 78, "cpu")
    gu = torch.cat([g, u], 1).contiguous()
    q, s, qT, sT = fq.swiglu_quant_dual_alloc(gu.to(DEV))
    torch.cuda.synchronize()
    rq, rs, rqT, rsT = oracle_mod.swiglu_quant_dual(bits(gu))
    assert_codes_equal(q, rq, "dual every gate rows")
    assert_scales_equal(s, rs, "dual every gate row scales", cols=512)
    assert_codes_equal(qT, rqT, "dual every gate columns")
    assert_scales_equal(sT, rsT, "dual every gate column scales")
