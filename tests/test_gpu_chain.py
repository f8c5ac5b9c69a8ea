"""Integration: one reduced Llama-shaped layer (M = 256, hidden 512, intermediate 768)
through the whole chain on the GPU, each stage fed the GPU's output of the stage before
and compared with the oracle applied to that same input — codes and scales bit for bit,
GEMM outputs within one BF16 ulp + 1e-5 * sum |a b|, the RMSNorm backward's BF16
gradient within one BF16 ulp (its codes bit for bit on the kernel's own gradient).

Forward: RMSNorm+quant -> QKV; 1x128 quant of the attention output (attention itself is
outside the path: a seeded BF16 tensor) -> O; RMSNorm+quant -> gate/up -> SwiGLU+quant
on the gate/up output -> down. Backward of the down projection from a seeded dY (a6,
DGrad, a8 of the saved SwiGLU codes, WGrad), then the fused producers: the SwiGLU
backward on the down DGrad's output, the gate/up DGrad and WGrad from its codes, the
RMSNorm backward (with the residual gradient) on the gate/up DGrad's output."""
import numpy as np
import pytest
import torch

import workloads
from gpu_util import assert_codes_equal, assert_gemm_close, assert_scales_equal, bits, np_f32, np_u8

pytestmark = pytest.mark.gpu
DEV = "cuda"
M, H, I, NQKV = 256, 512, 768, 768
EPS = 1e-5


@pytest.fixture(scope="module")
def fq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import fp8_block_scaled_08_b200 as f
    return f


def _f(b):
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _ulp_bf16(v):
    a = np.abs(v)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, 2.0 ** (e - 7), 2.0 ** -133)


def _fwd(fq, oracle_mod, qa, sa, w, what):
    qw, sw, qwT = fq.quant_weight_alloc(w)
    torch.cuda.synchronize()
    rqw, rsw, rqwT = oracle_mod.quant_weight_128x128(bits(w))
    assert_codes_equal(qw, rqw, what + " weight codes")
    assert_codes_equal(qwT, rqwT, what + " transposed weight codes")
    assert np.array_equal(np_f32(sw).view(np.uint32), rsw.view(np.uint32))
    y = fq.linear_fwd_alloc(qa, sa, qw, sw)
    torch.cuda.synchronize()
    ref, ab = oracle_mod.linear_fwd(np_u8(qa), np_f32(sa), np_u8(qw), np_f32(sw))
    assert_gemm_close(y.float().cpu().numpy(), ref, ab, what + " forward")
    return y, qw, sw, qwT


def test_reduced_llama_layer_chain(fq, oracle_mod):
    x_attn = workloads.activations_bf16((M, H), 0, 6000, DEV, outlier_frac=0.005,
                                        outlier_scale=50.0)
    x_mlp = workloads.activations_bf16((M, H), 0, 6001, DEV, outlier_frac=0.005,
                                       outlier_scale=50.0)
    attn_out = workloads.activations_bf16((M, H), 0, 6002, DEV)
    g1, g2 = workloads.gamma_bf16(H, 0, 6003, DEV), workloads.gamma_bf16(H, 0, 6004, DEV)
    w = {"qkv": workloads.normal_bf16((NQKV, H), 0.02, 0, 6005, DEV),
         "o": workloads.normal_bf16((H, H), 0.02, 0, 6006, DEV),
         "gate_up": workloads.normal_bf16((2 * I, H), 0.02, 0, 6007, DEV),
         "down": workloads.normal_bf16((H, I), 0.02, 0, 6008, DEV)}
    dy_down = workloads.gradients_bf16((M, H), 1e-3, 0, 6009, DEV)

    # ---- forward
    q1, s1 = fq.rmsnorm_quant_alloc(x_attn, g1, EPS)
    torch.cuda.synchronize()
    rq1, rs1 = oracle_mod.rmsnorm_quant(bits(x_attn), bits(g1), EPS)
    assert_codes_equal(q1, rq1, "rmsnorm1")
    assert_scales_equal(s1, rs1, "rmsnorm1 scales", cols=M)
    _fwd(fq, oracle_mod, q1, s1, w["qkv"], "qkv")

    qa, sa = fq.quant_act_1x128_alloc(attn_out)
    torch.cuda.synchronize()
    rqa, rsa = oracle_mod.quant_act_1x128(bits(attn_out))
    assert_codes_equal(qa, rqa, "attention output")
    _fwd(fq, oracle_mod, qa, sa, w["o"], "o")

    q2, s2 = fq.rmsnorm_quant_alloc(x_mlp, g2, EPS)
    torch.cuda.synchronize()
    rq2, rs2 = oracle_mod.rmsnorm_quant(bits(x_mlp), bits(g2), EPS)
    assert_codes_equal(q2, rq2, "rmsnorm2")
    gu, _, _, qguT_w = _fwd(fq, oracle_mod, q2, s2, w["gate_up"], "gate/up")

    qh, sh = fq.swiglu_quant_alloc(gu)           # the stage's input is the GPU's gate/up output
    torch.cuda.synchronize()
    rqh, rsh = oracle_mod.swiglu_quant(bits(gu))
    assert_codes_equal(qh, rqh, "swiglu")
    assert_scales_equal(sh, rsh, "swiglu scales", cols=M)
    _, _, swd, qwdT = _fwd(fq, oracle_mod, qh, sh, w["down"], "down")

    # ---- backward of the down projection (a6, DGrad, a8, WGrad)
    qdy, sdy, qdyT, sdyc = fq.transpose_quant_bf16_alloc(dy_down)
    torch.cuda.synchronize()
    rr, rrs, rc, rcs = oracle_mod.transpose_quant_bf16(bits(dy_down))
    assert_codes_equal(qdy, rr, "down dY rows")
    assert_codes_equal(qdyT, rc, "down dY columns")
    assert_scales_equal(sdyc, rcs, "down dY column scales")
    dh = fq.linear_dgrad_alloc(qdy, sdy, qwdT, swd)
    qhT, shT = fq.transpose_quant_fp8_alloc(qh, sh)
    dw_down = fq.linear_wgrad_alloc(qdyT, sdyc, qhT, shT)
    torch.cuda.synchronize()
    ref, ab = oracle_mod.linear_dgrad(np_u8(qdy), np_f32(sdy),
                                      *oracle_mod.quant_weight_128x128(bits(w["down"]))[:2])
    assert_gemm_close(dh.float().cpu().numpy(), ref, ab, "down DGrad")
    rqhT, rshT = oracle_mod.transpose_quant_fp8(np_u8(qh), np_f32(sh))
    assert_codes_equal(qhT, rqhT, "saved SwiGLU codes, 128x1")
    ref, ab = oracle_mod.linear_wgrad(np_u8(qdyT), np_f32(sdyc), np_u8(qhT), np_f32(shT))
    assert_gemm_close(dw_down.float().cpu().numpy(), ref, ab, "down WGrad")

    # ---- fused producers: SwiGLU backward on the GPU's dh, gate/up DGrad and WGrad
    qg, sg, qgT, sgc, dgu = fq.swiglu_bwd_quant_dual_alloc(gu, dh, want_dgu=True)
    torch.cuda.synchronize()
    rq, rs, rqT, rsT, rdgu = oracle_mod.swiglu_bwd_dual(bits(gu), bits(dh))
    assert np.array_equal(bits(dgu), rdgu)
    assert_codes_equal(qg, rq, "swiglu backward rows")
    assert_codes_equal(qgT, rqT, "swiglu backward columns")
    assert_scales_equal(sgc, rsT, "swiglu backward column scales")
    rqw, rsw, rqwT = oracle_mod.quant_weight_128x128(bits(w["gate_up"]))
    _, swg, qwgT = fq.quant_weight_alloc(w["gate_up"])
    dn2 = fq.linear_dgrad_alloc(qg, sg, qwgT, swg)
    qx2T, sx2T = fq.transpose_quant_fp8_alloc(q2, s2)
    dw_gu = fq.linear_wgrad_alloc(qgT, sgc, qx2T, sx2T)
    torch.cuda.synchronize()
    ref, ab = oracle_mod.linear_dgrad(np_u8(qg), np_f32(sg), rqw, rsw)
    assert_gemm_close(dn2.float().cpu().numpy(), ref, ab, "gate/up DGrad")
    ref, ab = oracle_mod.linear_wgrad(np_u8(qgT), np_f32(sgc), np_u8(qx2T), np_f32(sx2T))
    assert_gemm_close(dw_gu.float().cpu().numpy(), ref, ab, "gate/up WGrad")

    # ---- RMSNorm2 backward on the GPU's gate/up DGrad output, residual gradient dy_down
    out, qo, so, qoT, soc, dgam = fq.rmsnorm_bwd_quant_dual_alloc(x_mlp, g2, dn2, dy_down, EPS)
    torch.cuda.synchronize()
    rout, rdg, _, _ = oracle_mod.rmsnorm_bwd(bits(x_mlp), bits(g2), bits(dn2), bits(dy_down), EPS)
    err = np.abs(_f(bits(out)) - _f(rout))
    assert np.all(err <= _ulp_bf16(_f(rout))), "rmsnorm backward beyond one BF16 ulp"
    oq, _, oqT, osc = oracle_mod.transpose_quant_bf16(bits(out))
    assert_codes_equal(qo, oq, "rmsnorm backward rows")
    assert_codes_equal(qoT, oqT, "rmsnorm backward columns")
    assert_scales_equal(soc, osc, "rmsnorm backward column scales")
    d = np.abs(np_f32(dgam).astype(np.float64) - rdg.astype(np.float64))
    assert np.all(d <= np.spacing(np.abs(rdg)).astype(np.float64) + 1e-30)
