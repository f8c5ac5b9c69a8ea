"""The split-K forward on the library's static workspace (fp8q_linear_fwd_splitk_noalloc),
against the entry point with a caller workspace (fp8q_linear_fwd_splitk) and the plain
forward: two calls in a row must each give the same bits. Collected last, so it also runs
after every other test has used the library in the same process."""
import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def fq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import fp8_block_scaled_08_b200 as f
    return f


def quantized(fq, M, N, K, seed_id):
    x = workloads.activations_bf16((M, K), 0, seed_id, DEV, outlier_count=4, outlier_scale=30.0)
    w = workloads.normal_bf16((N, K), 0.02, 0, seed_id + 1, DEV)
    qx, sx = fq.quant_act_1x128_alloc(x)
    qw, sw, _ = fq.quant_weight_alloc(w, want_t=False)
    return qx, sx, qw, sw


# (16, 4096, 4096) and (1, 4608, 3584) split K; (8, 24576, 512) fills the GPU without a
# split; the order makes a smaller call follow a larger one on the same array
@pytest.mark.parametrize("M,N,K", [(16, 4096, 4096), (1, 4608, 3584), (8, 24576, 512),
                                   (32, 1024, 2048)])
def test_noalloc_matches_workspace_entry_twice(fq, M, N, K):
    qx, sx, qw, sw = quantized(fq, M, N, K, 1600 + M)
    ref = fq.linear_fwd_alloc(qx, sx, qw, sw)
    ws = fq.splitk_workspace(M, N, K, DEV)
    y_ws = torch.empty_like(ref)
    fq.linear_fwd_splitk(qx, sx, qw, sw, y_ws, ws)
    torch.cuda.synchronize()
    assert torch.equal(y_ws.view(torch.int16), ref.view(torch.int16))
    for _ in range(2):
        y = torch.full_like(ref, float("nan"))
        fq.linear_fwd_splitk_noalloc(qx, sx, qw, sw, y)
        torch.cuda.synchronize()
        assert fq.device_error() == fq.FP8Q_OK
        assert torch.equal(y.view(torch.int16), y_ws.view(torch.int16)), (M, N, K)


def test_noalloc_rejects_shapes_beyond_the_array(fq):
    # partial products of 128 x 4096 x 8192 need 4096 * 64 * 128 * 4 = 134 MB > 64 MiB
    M, N, K = 128, 4096, 8192
    qx, sx, qw, sw = quantized(fq, M, N, K, 1700)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(fq.Fp8qError) as e:
        fq.linear_fwd_splitk_noalloc(qx, sx, qw, sw, y)
    assert e.value.status == fq.FP8Q_ERR_SHAPE
    assert "static workspace" in fq.last_error_message()
    # the library is still usable afterwards
    small = quantized(fq, 16, 4096, 4096, 1800)
    y2 = torch.empty((16, 4096), dtype=torch.bfloat16, device=DEV)
    fq.linear_fwd_splitk_noalloc(*small, y2)
    torch.cuda.synchronize()
    assert torch.equal(y2.view(torch.int16), fq.linear_fwd_alloc(*small).view(torch.int16))
