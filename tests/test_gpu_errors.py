"""The failure path on a GPU without faulting it: a bounded wait that nothing completes
gives up, the host reads FP8Q_ERR_TIMEOUT from the device error word, and the context
stays usable. Invalid arguments are rejected before any launch."""
import ctypes

import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import fp8_block_scaled_08_b200 as f
    return f


def test_bounded_wait_reports_timeout_and_context_survives(fq, oracle_mod):
    assert fq.device_error() == fq.FP8Q_OK
    assert fq.debug_wait_timeout(50_000_000) == fq.FP8Q_OK   # 50 ms limit
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert fq._lib.fp8q_last_device_error(stream) == fq.FP8Q_ERR_TIMEOUT  # reads, keeps
    assert fq.device_error(clear=True) == fq.FP8Q_ERR_TIMEOUT
    assert fq.device_error() == fq.FP8Q_OK                    # cleared
    x = workloads.activations_bf16((64, 256), 0, 900, "cuda")
    q, s = fq.quant_act_1x128_alloc(x)
    torch.cuda.synchronize()
    rq, _ = oracle_mod.quant_act_1x128(x.cpu().view(torch.int16).numpy().view("uint16"))
    assert (q.cpu().numpy() == rq).all()


def test_invalid_arguments_raise_before_launch(fq):
    x = torch.zeros((8, 200), dtype=torch.bfloat16, device="cuda")
    q = torch.empty((8, 200), dtype=torch.uint8, device="cuda")
    s = torch.empty((2, 8), device="cuda")
    with pytest.raises(fq.Fp8qError) as e:
        fq.quant_act_1x128(x, q, s)
    assert e.value.status == fq.FP8Q_ERR_SHAPE
    qa = torch.empty((16, 128), dtype=torch.uint8, device="cuda")
    sa = torch.empty((1, 16), device="cuda")
    qw = torch.empty((200, 128), dtype=torch.uint8, device="cuda")
    sw = torch.empty((2, 1), device="cuda")
    y = torch.empty((16, 200), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fq.Fp8qError) as e:
        fq.linear_fwd(qa, sa, qw, sw, y)
    assert e.value.status == fq.FP8Q_ERR_SHAPE
    torch.cuda.synchronize()
    assert fq.device_error() == fq.FP8Q_OK
