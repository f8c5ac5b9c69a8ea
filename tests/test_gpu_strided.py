"""Row strides and padded scale arrays on the quantizers that form their value on the fly:
each input is a column slice of a wider tensor (row stride > row length), the 1x128
scale arrays have a leading dimension larger than M, and every result must equal the
oracle's on the dense copy."""
import numpy as np
import pytest
import torch

import workloads
from gpu_util import assert_codes_equal, assert_scales_equal, bits

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def fq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import fp8_block_scaled_08_b200 as f
    return f


def _e(*shape, dt=torch.uint8):
    return torch.empty(shape, dtype=dt, device=DEV)


def test_a6_strided_gradient_padded_scales(fq, oracle_mod):
    M, N = 256, 512
    big = workloads.gradients_bf16((M, 1024), 1e-3, 0, 5000, DEV)
    dy = big[:, 384:896]
    lds = M + 8
    q, s, qT, sT = _e(M, N), _e(N // 128, lds, dt=torch.float32), _e(N, M), _e(M // 128, N, dt=torch.float32)
    fq.transpose_quant_bf16(dy, q, s, qT, sT)
    torch.cuda.synchronize()
    rq, rs, rqT, rsT = oracle_mod.transpose_quant_bf16(bits(dy.contiguous()))
    assert_codes_equal(q, rq, "a6 strided rows")
    assert_scales_equal(s, rs, "a6 strided row scales", cols=M)
    assert_codes_equal(qT, rqT, "a6 strided columns")
    assert_scales_equal(sT, rsT, "a6 strided column scales")


def test_rmsnorm_dual_strided_input(fq, oracle_mod):
    M, H = 256, 512
    big = workloads.activations_bf16((M, 1280), 0, 5001, DEV, outlier_frac=0.005,
                                     outlier_scale=50.0)
    x = big[:, 640:1152]
    g = workloads.gamma_bf16(H, 0, 5002, DEV)
    lds = M + 4
    q, s, qT, sT = _e(M, H), _e(H // 128, lds, dt=torch.float32), _e(H, M), _e(M // 128, H, dt=torch.float32)
    r = _e(M, dt=torch.float32)
    fq.rmsnorm_quant_dual(x, g, 1e-5, q, s, qT, sT, r)
    torch.cuda.synchronize()
    rq, rs, rqT, rsT, rr = oracle_mod.rmsnorm_quant_dual(bits(x.contiguous()), bits(g), 1e-5)
    assert_codes_equal(q, rq, "rmsnorm dual strided rows")
    assert_scales_equal(s, rs, "rmsnorm dual strided row scales", cols=M)
    assert_codes_equal(qT, rqT, "rmsnorm dual strided columns")
    assert_scales_equal(sT, rsT, "rmsnorm dual strided column scales")
    assert np.array_equal(r.cpu().numpy().view(np.uint32), rr.view(np.uint32))


def test_swiglu_dual_strided_input(fq, oracle_mod):
    M, I = 256, 384
    big = workloads.normal_bf16((M, 2 * I + 256), 1.5, 0, 5003, DEV)
    gu = big[:, :2 * I]
    q, s, qT, sT = _e(M, I), _e(I // 128, M, dt=torch.float32), _e(I, M), _e(M // 128, I, dt=torch.float32)
    fq.swiglu_quant_dual(gu, q, s, qT, sT)
    torch.cuda.synchronize()
    rq, rs, rqT, rsT = oracle_mod.swiglu_quant_dual(bits(gu.contiguous()))
    assert_codes_equal(q, rq, "swiglu dual strided rows")
    assert_codes_equal(qT, rqT, "swiglu dual strided columns")
    assert_scales_equal(sT, rsT, "swiglu dual strided column scales")


@pytest.mark.parametrize("M", [1100, 64])   # the two-pass warp kernel, and one CTA per row
def test_rmsnorm_quant_strided_input(fq, oracle_mod, M):
    H = 640
    big = workloads.activations_bf16((M, 1024), 0, 5004 + M, DEV)
    x = big[:, 128:768]
    g = workloads.gamma_bf16(H, 0, 5005, DEV)
    q, s = _e(M, H), _e(H // 128, M + 12, dt=torch.float32)
    fq.rmsnorm_quant(x, g, 1e-6, q, s)
    torch.cuda.synchronize()
    rq, rs = oracle_mod.rmsnorm_quant(bits(x.contiguous()), bits(g), 1e-6)
    assert_codes_equal(q, rq, "a3 strided")
    assert_scales_equal(s, rs, "a3 strided scales", cols=M)


def test_swiglu_quant_strided_input(fq, oracle_mod):
    M, I = 96, 256
    big = workloads.normal_bf16((M, 2 * I + 128), 1.5, 0, 5006, DEV)
    gu = big[:, :2 * I]
    q, s = _e(M, I), _e(I // 128, M + 4, dt=torch.float32)
    fq.swiglu_quant(gu, q, s)
    torch.cuda.synchronize()
    rq, rs = oracle_mod.swiglu_quant(bits(gu.contiguous()))
    assert_codes_equal(q, rq, "a4 strided")
    assert_scales_equal(s, rs, "a4 strided scales", cols=M)
