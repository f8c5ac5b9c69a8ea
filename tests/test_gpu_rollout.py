"""The rollout weight refresh on one GPU: the packed views hold exactly the oracle's
128x128 quantization of each BF16 master (codes and scales bit for bit), the same as
separate calls of the weight quantizer, and the forward GEMM reading them gives the same
output bit for bit."""
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


def test_refresh_views_equal_separate_quantization(fq, oracle_mod):
    from fp8_block_scaled_08_b200.rollout import PackedFp8Weights, refresh
    L = workloads.LLAMA31_8B
    shapes = {lin.name: (lin.n, lin.k) for lin in L.linears}
    masters = {n: workloads.normal_bf16(s, 0.02, 0, 950 + i, DEV)
               for i, (n, s) in enumerate(shapes.items())}
    packed = PackedFp8Weights(shapes, DEV)
    refresh(packed, masters)
    torch.cuda.synchronize()
    views = packed.views()
    x = workloads.activations_bf16((512, L.hidden), 0, 960, DEV, outlier_frac=0.005,
                                   outlier_scale=50.0)
    qx, sx = fq.quant_act_1x128_alloc(x)
    for name, w in masters.items():
        # the oracle's quantization of the master, in full
        rq, rs, _ = oracle_mod.quant_weight_128x128(bits(w), want_t=False)
        assert_codes_equal(views[name][0], rq, "packed codes " + name)
        assert_scales_equal(views[name][1], rs, "packed scales " + name)
        q, s, _ = fq.quant_weight_alloc(w, want_t=False)
        torch.cuda.synchronize()
        assert torch.equal(views[name][0], q), name
        assert torch.equal(views[name][1].view(torch.int32), s.view(torch.int32)), name
        if shapes[name][1] == L.hidden:
            y1 = fq.linear_fwd_alloc(qx, sx, views[name][0], views[name][1])
            y2 = fq.linear_fwd_alloc(qx, sx, q, s)
            torch.cuda.synchronize()
            assert torch.equal(y1.view(torch.int16), y2.view(torch.int16)), name
