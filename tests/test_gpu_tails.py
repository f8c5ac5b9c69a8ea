"""Sizes that are not multiples of 128 (partial groups) through the C ABI, against the
oracle: the quantizers' codes and scales bit for bit (a1, a2 with its transposed copy,
a3, a4, a6 both ways, a8), and the three GEMMs within the GEMM tolerance, including a
decode-sized batch with a ragged K (which runs on the CTA-pair kernel). A partial group
is the full group with zeros in the missing places: its scale comes from its valid
elements alone ("Resumen Técnico: Jet-RL", «Esquema de Cuantización», read that way)."""
import numpy as np
import pytest
import torch

import workloads
from gpu_util import (assert_codes_equal, assert_gemm_close, assert_scales_equal, bits, np_f32,
                      np_u8)

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def fq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import fp8_block_scaled_08_b200 as f
    return f


SHAPES = [(208, 304), (144, 400), (16, 16), (128, 4096 + 48), (384, 272)]


@pytest.mark.parametrize("M,K", SHAPES + [(7, 1040), (129, 144)])
def test_act_quant_tail(fq, oracle_mod, M, K):
    x = workloads.activations_bf16((M, K), 0, 4000 + K, DEV, outlier_count=3, outlier_scale=40.0)
    q, s = fq.quant_act_1x128_alloc(x)
    torch.cuda.synchronize()
    rq, rs = oracle_mod.quant_act_1x128(bits(x))
    assert_codes_equal(q, rq, "a1 tail codes")
    assert_scales_equal(s, rs, "a1 tail scales", cols=M)


@pytest.mark.parametrize("N,K", [(208, 304), (144, 400), (16, 16), (272, 4096 + 48)])
def test_weight_quant_tail(fq, oracle_mod, N, K):
    w = workloads.normal_bf16((N, K), 0.02, 0, 4100 + K, DEV)
    q, s, qT = fq.quant_weight_alloc(w)
    torch.cuda.synchronize()
    rq, rs, rqT = oracle_mod.quant_weight_128x128(bits(w))
    assert_codes_equal(q, rq, "a2 tail codes")
    assert_codes_equal(qT, rqT, "a2 tail transposed codes")
    assert_scales_equal(s, rs, "a2 tail scales")


@pytest.mark.parametrize("M,H", SHAPES + [(2048, 3584 + 16), (201, 272)])
def test_rmsnorm_quant_tail(fq, oracle_mod, M, H):
    x = workloads.activations_bf16((M, H), 0, 4200 + H, DEV, outlier_count=2, outlier_scale=50.0)
    g = workloads.gamma_bf16(H, 0, 4201 + H, DEV)
    q, s = fq.rmsnorm_quant_alloc(x, g, 1e-5)
    torch.cuda.synchronize()
    rq, rs = oracle_mod.rmsnorm_quant(bits(x), bits(g), 1e-5)
    assert_codes_equal(q, rq, "a3 tail codes")
    assert_scales_equal(s, rs, "a3 tail scales", cols=M)


@pytest.mark.parametrize("M,I", SHAPES + [(33, 400)])
def test_swiglu_quant_tail(fq, oracle_mod, M, I):
    gu = workloads.normal_bf16((M, 2 * I), 1.5, 0, 4300 + I, DEV)
    q, s = fq.swiglu_quant_alloc(gu)
    torch.cuda.synchronize()
    rq, rs = oracle_mod.swiglu_quant(bits(gu))
    assert_codes_equal(q, rq, "a4 tail codes")
    assert_scales_equal(s, rs, "a4 tail scales", cols=M)


@pytest.mark.parametrize("M,N", [(208, 304), (144, 400), (16, 16), (272, 4096 + 48), (48, 128)])
def test_dual_grad_quant_tail(fq, oracle_mod, M, N):
    dy = workloads.gradients_bf16((M, N), 1e-3, 0, 4400 + N, DEV, small_row_frac=0.05,
                                  small_row_scale=1e-3)
    q, s, qT, sT = fq.transpose_quant_bf16_alloc(dy)
    torch.cuda.synchronize()
    rq, rs, rqT, rsT = oracle_mod.transpose_quant_bf16(bits(dy))
    assert_codes_equal(q, rq, "a6 tail rows")
    assert_scales_equal(s, rs, "a6 tail row scales", cols=M)
    assert_codes_equal(qT, rqT, "a6 tail columns")
    assert_scales_equal(sT, rsT, "a6 tail column scales")


@pytest.mark.parametrize("M,K", [(208, 304), (144, 400), (16, 16), (272, 4096 + 48)])
def test_fp8_requant_tail(fq, oracle_mod, M, K):
    x = workloads.activations_bf16((M, K), 0, 4500 + K, DEV, outlier_count=2, outlier_scale=30.0)
    q, s = fq.quant_act_1x128_alloc(x)
    qT, sT = fq.transpose_quant_fp8_alloc(q, s)
    torch.cuda.synchronize()
    rqT, rsT = oracle_mod.transpose_quant_fp8(np_u8(q), np_f32(s))
    assert_codes_equal(qT, rqT, "a8 tail codes")
    assert_scales_equal(sT, rsT, "a8 tail scales")


@pytest.mark.parametrize("M,N,K", [(200, 272, 304), (16, 400, 144), (300, 128, 4096 + 48),
                                   (513, 4096 + 16, 400), (64, 1024, 1040)])
def test_fwd_and_dgrad_tail(fq, oracle_mod, M, N, K):
    x = workloads.activations_bf16((M, K), 0, 4600 + K, DEV, outlier_count=3, outlier_scale=30.0)
    w = workloads.normal_bf16((N, K), 0.02, 0, 4601 + K, DEV)
    dy = workloads.gradients_bf16((M, N), 1e-3, 0, 4602 + K, DEV)
    qx, sx = fq.quant_act_1x128_alloc(x)
    qw, sw, qwT = fq.quant_weight_alloc(w)
    qdy, sdy = fq.quant_act_1x128_alloc(dy)
    y = fq.linear_fwd_alloc(qx, sx, qw, sw)
    dx = fq.linear_dgrad_alloc(qdy, sdy, qwT, sw)
    torch.cuda.synchronize()
    ref, ab = oracle_mod.linear_fwd(np_u8(qx), np_f32(sx), np_u8(qw), np_f32(sw))
    assert_gemm_close(y.float().cpu().numpy(), ref, ab, "fwd tail %dx%dx%d" % (M, N, K))
    ref, ab = oracle_mod.linear_dgrad(np_u8(qdy), np_f32(sdy), np_u8(qw), np_f32(sw))
    assert_gemm_close(dx.float().cpu().numpy(), ref, ab, "dgrad tail %dx%dx%d" % (M, N, K))


@pytest.mark.parametrize("M,N,K", [(208, 272, 304), (144, 400, 128), (4096 + 48, 256, 272)])
def test_wgrad_tail(fq, oracle_mod, M, N, K):
    x = workloads.activations_bf16((M, K), 0, 4700 + M, DEV, outlier_count=3, outlier_scale=30.0)
    dy = workloads.gradients_bf16((M, N), 1e-3, 0, 4701 + M, DEV)
    qx, sx = fq.quant_act_1x128_alloc(x)
    qxT, sxc = fq.transpose_quant_fp8_alloc(qx, sx)
    _, _, qdyT, sdyc = fq.transpose_quant_bf16_alloc(dy, want_row=False)
    dw = fq.linear_wgrad_alloc(qdyT, sdyc, qxT, sxc)
    dw32 = torch.zeros((N, K), dtype=torch.float32, device=DEV)
    fq.linear_wgrad_acc_f32(qdyT, sdyc, qxT, sxc, dw32)
    torch.cuda.synchronize()
    ref, ab = oracle_mod.linear_wgrad(np_u8(qdyT), np_f32(sdyc), np_u8(qxT), np_f32(sxc))
    assert_gemm_close(dw.float().cpu().numpy(), ref, ab, "wgrad tail %dx%dx%d" % (M, N, K))
    # accumulated from zero the fp32 output is the accumulator: it rounds to the BF16 one
    assert torch.equal(dw32.to(torch.bfloat16).view(torch.int16), dw.view(torch.int16))


def test_shapes_off_the_16_grid_are_refused(fq):
    x = torch.zeros((16, 136), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(fq.Fp8qError):
        fq.quant_act_1x128_alloc(x)
    w = torch.zeros((24, 128), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(fq.Fp8qError):
        fq.quant_weight_alloc(w)
