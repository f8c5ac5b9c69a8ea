"""WGrad accumulated into an fp32 dW (gradient accumulation): dw += the fp32
accumulator, against the oracle (dw_in + the fp64 product, within one fp32 ulp of the
sum + 1e-5 * sum |a b|), two calls summing, the BF16 WGrad equal to the BF16 rounding of
the accumulator added to zero, an N tail, and the full Llama-3.1-8B gate/up shape on
sampled rows."""
import numpy as np
import pytest
import torch

import workloads
from gpu_util import np_f32, np_u8

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def fq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import fp8_block_scaled_08_b200 as f
    return f


def _operands(fq, M, N, K, seed):
    x = workloads.activations_bf16((M, K), 0, seed, DEV, outlier_count=4, outlier_scale=30.0)
    dy = workloads.gradients_bf16((M, N), 1e-3, 0, seed + 1, DEV)
    qx, sx = fq.quant_act_1x128_alloc(x)
    qxT, sxc = fq.transpose_quant_fp8_alloc(qx, sx)
    _, _, qdyT, sdyc = fq.transpose_quant_bf16_alloc(dy, want_row=False)
    return qdyT, sdyc, qxT, sxc


def _assert_acc_close(got, expect, ab, what):
    got = np.asarray(got, np.float64)
    tol = np.spacing(np.abs(expect).astype(np.float32)).astype(np.float64) + 1e-5 * ab + 1e-40
    bad = np.abs(got - expect) > tol
    if bad.any():
        i = tuple(np.argwhere(bad)[0])
        raise AssertionError("%s: %d outside the tolerance, first at %s: gpu %r expected %r" % (
            what, int(bad.sum()), i, got[i], expect[i]))


@pytest.mark.parametrize("M,N,K", [(256, 512, 512), (128, 128, 128), (384, 384, 640),
                                   (256, 640, 384)])
def test_wgrad_acc_f32_matches_oracle(fq, oracle_mod, M, N, K):
    qdyT, sdyc, qxT, sxc = _operands(fq, M, N, K, 4000 + M + N)
    dw = (torch.randn((N, K), device=DEV, generator=torch.Generator(DEV).manual_seed(N + K))
          * 1e-2).float()
    dw0 = dw.cpu().numpy().astype(np.float64)
    fq.linear_wgrad_acc_f32(qdyT, sdyc, qxT, sxc, dw)
    torch.cuda.synchronize()
    ref, ab = oracle_mod.linear_wgrad(np_u8(qdyT), np_f32(sdyc), np_u8(qxT), np_f32(sxc))
    _assert_acc_close(dw.cpu().numpy(), dw0 + ref, ab, "wgrad acc %dx%dx%d" % (M, N, K))


def test_wgrad_acc_two_calls_and_bf16_identity(fq, oracle_mod):
    M, N, K = 384, 512, 384
    a = _operands(fq, M, N, K, 4100)
    b = _operands(fq, M, N, K, 4200)
    dw = torch.zeros((N, K), dtype=torch.float32, device=DEV)
    fq.linear_wgrad_acc_f32(*a, dw)
    torch.cuda.synchronize()
    once = dw.clone()
    # added to zero, the fp32 result is the accumulator itself: its BF16 rounding is the
    # BF16 WGrad's output
    dw_bf16 = fq.linear_wgrad_alloc(*a)
    torch.cuda.synchronize()
    assert torch.equal(once.to(torch.bfloat16).float(), dw_bf16.float())
    fq.linear_wgrad_acc_f32(*b, dw)
    torch.cuda.synchronize()
    ra, aba = oracle_mod.linear_wgrad(*(np_u8(t) if t.dtype == torch.uint8 else np_f32(t) for t in a))
    rb, abb = oracle_mod.linear_wgrad(*(np_u8(t) if t.dtype == torch.uint8 else np_f32(t) for t in b))
    _assert_acc_close(dw.cpu().numpy(), ra + rb, aba + abb, "two accumulations")


def test_wgrad_acc_full_size_gate_up_sampled(fq, oracle_mod):
    """Llama-3.1-8B gate/up WGrad (N = 28672, K = 4096, M = 8192) added into a non-zero
    fp32 dW; 32 sampled rows of dW against the oracle."""
    M, N, K = 8192, 28672, 4096
    qdyT, sdyc, qxT, sxc = _operands(fq, M, N, K, 4300)
    dw = torch.full((N, K), 0.25, dtype=torch.float32, device=DEV)
    fq.linear_wgrad_acc_f32(qdyT, sdyc, qxT, sxc, dw)
    torch.cuda.synchronize()
    rng = np.random.default_rng(11)
    r0 = int(rng.integers(0, N - 32))
    ref, ab = oracle_mod.linear_wgrad(np_u8(qdyT), np_f32(sdyc), np_u8(qxT), np_f32(sxc),
                                      rows=(r0, 32))
    _assert_acc_close(dw[r0:r0 + 32].cpu().numpy(), 0.25 + ref, ab, "full-size gate/up rows")
