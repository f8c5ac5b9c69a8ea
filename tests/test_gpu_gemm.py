"""Parity of the tcgen05 FP8 GEMMs (forward, DGrad, WGrad) with the fp64 oracle:
|gpu - oracle| <= 1 BF16 ulp of the oracle value + 1e-5 * sum_k |a_k b_k|, on the tiny
layer, ragged M, N tails, single-slice K, an exact integer case, batch invariance of
the forward GEMM, and (sampled) the full Llama-3.1-8B layer."""
import numpy as np
import pytest
import torch

import workloads
from gpu_util import assert_gemm_close, bits, np_f32, np_u8

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module")
def fq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import fp8_block_scaled_08_b200 as f
    return f


def quantized_linear(fq, M, N, K, seed_id, outliers=4):
    x = workloads.activations_bf16((M, K), 0, seed_id, DEV, outlier_count=outliers,
                                   outlier_scale=30.0)
    w = workloads.normal_bf16((N, K), 0.02, 0, seed_id + 1, DEV)
    qx, sx = fq.quant_act_1x128_alloc(x)
    qw, sw, qwT = fq.quant_weight_alloc(w)
    return qx, sx, qw, sw, qwT


@pytest.mark.parametrize("M,N,K", [(256, 512, 512), (1, 256, 128), (16, 4096 // 8, 1024),
                                   (200, 384, 640), (300, 128, 256), (129, 640, 384)])
def test_fwd_matches_oracle(fq, oracle_mod, M, N, K):
    qx, sx, qw, sw, _ = quantized_linear(fq, M, N, K, 1000 + M)
    y = fq.linear_fwd_alloc(qx, sx, qw, sw)
    torch.cuda.synchronize()
    ref, ab = oracle_mod.linear_fwd(np_u8(qx), np_f32(sx), np_u8(qw), np_f32(sw))
    assert_gemm_close(y.float().cpu().numpy(), ref, ab, "fwd %dx%dx%d" % (M, N, K))


@pytest.mark.parametrize("M,N,K", [(256, 512, 512), (64, 128, 384), (130, 384, 256)])
def test_dgrad_matches_oracle(fq, oracle_mod, M, N, K):
    dy = workloads.gradients_bf16((M, N), 1e-3, 0, 1100 + M, DEV)
    w = workloads.normal_bf16((N, K), 0.02, 0, 1101 + M, DEV)
    qdy, sdy = fq.quant_act_1x128_alloc(dy)
    qw, sw, qwT = fq.quant_weight_alloc(w)
    dx = fq.linear_dgrad_alloc(qdy, sdy, qwT, sw)
    torch.cuda.synchronize()
    ref, ab = oracle_mod.linear_dgrad(np_u8(qdy), np_f32(sdy), np_u8(qw), np_f32(sw))
    assert_gemm_close(dx.float().cpu().numpy(), ref, ab, "dgrad %dx%dx%d" % (M, N, K))


@pytest.mark.parametrize("M,N,K", [(256, 512, 512), (128, 128, 128), (384, 384, 640)])
def test_wgrad_matches_oracle(fq, oracle_mod, M, N, K):
    x = workloads.activations_bf16((M, K), 0, 1200 + M, DEV, outlier_count=4, outlier_scale=30.0)
    dy = workloads.gradients_bf16((M, N), 1e-3, 0, 1201 + M, DEV)
    qx, sx = fq.quant_act_1x128_alloc(x)
    qxT, sxc = fq.transpose_quant_fp8_alloc(qx, sx)
    _, _, qdyT, sdyc = fq.transpose_quant_bf16_alloc(dy, want_row=False)
    dw = fq.linear_wgrad_alloc(qdyT, sdyc, qxT, sxc)
    torch.cuda.synchronize()
    ref, ab = oracle_mod.linear_wgrad(np_u8(qdyT), np_f32(sdyc), np_u8(qxT), np_f32(sxc))
    assert_gemm_close(dw.float().cpu().numpy(), ref, ab, "wgrad %dx%dx%d" % (M, N, K))


def test_tiny_layer_all_three(fq, oracle_mod):
    """The tiny single-layer workload: X [256,512], W [512,512], dY [256,512]."""
    x, w, dy = workloads.tiny_inputs(DEV)
    qx, sx = fq.quant_act_1x128_alloc(x)
    qw, sw, qwT = fq.quant_weight_alloc(w)
    y = fq.linear_fwd_alloc(qx, sx, qw, sw)
    qdy, sdy, qdyT, sdyc = fq.transpose_quant_bf16_alloc(dy)
    dx = fq.linear_dgrad_alloc(qdy, sdy, qwT, sw)
    qxT, sxc = fq.transpose_quant_fp8_alloc(qx, sx)
    dw = fq.linear_wgrad_alloc(qdyT, sdyc, qxT, sxc)
    torch.cuda.synchronize()
    ref, ab = oracle_mod.linear_fwd(np_u8(qx), np_f32(sx), np_u8(qw), np_f32(sw))
    assert_gemm_close(y.float().cpu().numpy(), ref, ab, "tiny fwd")
    ref, ab = oracle_mod.linear_dgrad(np_u8(qdy), np_f32(sdy), np_u8(qw), np_f32(sw))
    assert_gemm_close(dx.float().cpu().numpy(), ref, ab, "tiny dgrad")
    ref, ab = oracle_mod.linear_wgrad(np_u8(qdyT), np_f32(sdyc), np_u8(qxT), np_f32(sxc))
    assert_gemm_close(dw.float().cpu().numpy(), ref, ab, "tiny wgrad")


def test_integer_case_is_exact(fq, oracle_mod):
    """Scales 1 and codes in {-2..2}: every partial sum is a small integer, so the
    tensor-core slices and the promotion are exact and Y equals the integer product."""
    rng = np.random.default_rng(21)
    small = np.array([0xC0, 0xB8, 0x00, 0x38, 0x40], np.uint8)  # -2,-1,0,1,2
    va = rng.integers(-2, 3, (256, 512))
    vb = rng.integers(-2, 3, (256, 512))
    qa = torch.from_numpy(small[va + 2]).to(DEV)
    qb = torch.from_numpy(small[vb + 2]).to(DEV)
    sa = torch.ones((4, 256), device=DEV)
    sb = torch.ones((2, 4), device=DEV)
    y = fq.linear_fwd_alloc(qa, sa, qb, sb)
    torch.cuda.synchronize()
    exact = (va @ vb.T).astype(np.float64)
    assert np.array_equal(y.float().cpu().numpy().astype(np.float64), exact)


def test_fwd_batch_invariance(fq):
    """Row m of the forward GEMM is bit-identical whether it is computed inside a large
    token batch or in a small decode-sized batch at a different tile position
    ("Arquitectura Central": the inference graph is a subgraph of the training forward)."""
    M, N, K = 2048, 1024, 2048
    qx, sx, qw, sw, _ = quantized_linear(fq, M, N, K, 1300)
    y_big = fq.linear_fwd_alloc(qx, sx, qw, sw)
    for r0, m in ((1000, 16), (77, 64), (2040, 8), (5, 1)):
        qs = qx[r0:r0 + m].contiguous()
        ss = torch.zeros((K // 128, fq.lds_for(m)), device=DEV)
        ss[:, :m] = sx[:, r0:r0 + m]
        y_small = fq.linear_fwd_alloc(qs, ss, qw, sw)
        torch.cuda.synchronize()
        assert torch.equal(y_small.view(torch.int16), y_big[r0:r0 + m].view(torch.int16)), (r0, m)


def test_full_size_llama_layer_gemms_sampled(fq, oracle_mod):
    """Llama-3.1-8B layer, M = 8192: forward of QKV, DGrad of gate/up and WGrad of
    O at full size (the benchmark's launch configuration); the oracle checks a 128-row
    slab and 2048 random entries of each."""
    wl = workloads.LLAMA_LAYER
    M = wl.tokens
    rng = np.random.default_rng(3)
    inp = workloads.layer_inputs(wl, DEV)

    def check(gpu, slab_fn, rowA, rowB, what):
        """slab_fn((r0, 128)) -> (ref, absdot) of a 128-row slab; rowA(i) / rowB(j) ->
        the fp64 dequantized reduction vectors of output row i / column j."""
        nrows, ncols = gpu.shape
        r0 = int(rng.integers(0, nrows // 128)) * 128
        ref, ab = slab_fn((r0, 128))
        assert_gemm_close(gpu[r0:r0 + 128].float().cpu().numpy(), ref, ab, what + " slab")
        ii = rng.integers(0, nrows, 2048)
        jj = rng.integers(0, ncols, 2048)
        refs = np.empty(len(ii))
        abss = np.empty(len(ii))
        for t, (i, j) in enumerate(zip(ii, jj)):
            a, b = rowA(int(i)), rowB(int(j))
            refs[t] = a @ b
            abss[t] = np.abs(a) @ np.abs(b)
        g = gpu[torch.from_numpy(ii).to(DEV), torch.from_numpy(jj).to(DEV)]
        assert_gemm_close(g.float().cpu().numpy(), refs, abss, what + " samples")

    # forward QKV from the fused RMSNorm output
    qx, sx = fq.rmsnorm_quant_alloc(inp["x_attn"], inp["gamma1"], wl.eps)
    qw, sw, qwT = fq.quant_weight_alloc(inp["w"]["qkv"])
    y = fq.linear_fwd_alloc(qx, sx, qw, sw)
    torch.cuda.synchronize()
    qx_n, sx_n, qw_n, sw_n = np_u8(qx), np_f32(sx), np_u8(qw), np_f32(sw)
    check(y, lambda rows: oracle_mod.linear_fwd(qx_n, sx_n, qw_n, sw_n, rows),
          lambda i: oracle_mod.dequant_rows(qx_n, sx_n, i, 1)[0],
          lambda j: oracle_mod.dequant_block(qw_n, sw_n, j, 1)[0], "qkv fwd")
    del y
    # DGrad of gate/up (N = 28672, K = 4096)
    qg, sg, qgT = fq.quant_weight_alloc(inp["w"]["gate_up"])
    qdy, sdy, _, _ = fq.transpose_quant_bf16_alloc(inp["dy"]["gate_up"])
    dx = fq.linear_dgrad_alloc(qdy, sdy, qgT, sg)
    torch.cuda.synchronize()
    qdy_n, sdy_n, qg_n, sg_n = np_u8(qdy), np_f32(sdy), np_u8(qg), np_f32(sg)
    qgT_n, sgT_n = np_u8(qgT), np.ascontiguousarray(sg_n.T)
    check(dx, lambda rows: oracle_mod.linear_dgrad(qdy_n, sdy_n, qg_n, sg_n, rows),
          lambda i: oracle_mod.dequant_rows(qdy_n, sdy_n, i, 1)[0],
          lambda k: oracle_mod.dequant_block(qgT_n, sgT_n, k, 1)[0], "gate_up dgrad")
    del dx, qdy, sdy, qg, sg, qgT
    # WGrad of O (N = 4096 out features, K = 4096 in features, reduction over 8192 tokens)
    qa, sa = fq.quant_act_1x128_alloc(inp["attn_out"])
    qaT, saT = fq.transpose_quant_fp8_alloc(qa, sa)
    _, _, qdoT, sdo = fq.transpose_quant_bf16_alloc(inp["dy"]["o"], want_row=False)
    dw = fq.linear_wgrad_alloc(qdoT, sdo, qaT, saT)
    torch.cuda.synchronize()
    qdoT_n, sdo_n, qaT_n, saT_n = np_u8(qdoT), np_f32(sdo), np_u8(qaT), np_f32(saT)
    check(dw, lambda rows: oracle_mod.linear_wgrad(qdoT_n, sdo_n, qaT_n, saT_n, rows),
          lambda n: oracle_mod.dequant_cols(qdoT_n, sdo_n, n, 1)[0],
          lambda k: oracle_mod.dequant_cols(qaT_n, saT_n, k, 1)[0], "o wgrad")


@pytest.mark.parametrize("M,N,K", [(16, 4096, 4096), (1, 512, 640), (100, 4608, 3584),
                                   (128, 1024, 2048), (32, 5120, 5120), (16, 256, 27648)])
def test_splitk_matches_linear_fwd_bitwise(fq, oracle_mod, M, N, K):
    """The split-K forward writes raw slice products to its workspace and promotes them in
    order in the last CTA of each strip: the same bits as fp8q_linear_fwd, twice in a row
    on one workspace (its counters return to zero), and within the oracle's tolerance."""
    qx, sx, qw, sw, _ = quantized_linear(fq, M, N, K, 1400 + M)
    ref = fq.linear_fwd_alloc(qx, sx, qw, sw)
    ws = fq.splitk_workspace(M, N, K, DEV)
    counters = fq._lib.fp8q_linear_fwd_splitk_counter_bytes(M, N)
    for _ in range(2):
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
        fq.linear_fwd_splitk(qx, sx, qw, sw, y, ws)
        torch.cuda.synchronize()
        assert fq.device_error() == fq.FP8Q_OK
        assert torch.equal(y.view(torch.int16), ref.view(torch.int16))
        assert int(ws[:counters].count_nonzero()) == 0
    if M * N * K <= 2 ** 28:
        r, ab = oracle_mod.linear_fwd(np_u8(qx), np_f32(sx), np_u8(qw), np_f32(sw))
        assert_gemm_close(y.float().cpu().numpy(), r, ab, "split-K fwd %dx%dx%d" % (M, N, K))


def test_splitk_workspace_errors(fq):
    qx, sx, qw, sw, _ = quantized_linear(fq, 16, 4096, 4096, 1500)
    y = torch.empty((16, 4096), dtype=torch.bfloat16, device=DEV)
    small = torch.zeros(1024, dtype=torch.uint8, device=DEV)
    with pytest.raises(fq.Fp8qError) as e:
        fq.linear_fwd_splitk(qx, sx, qw, sw, y, small)
    assert e.value.status == fq.FP8Q_ERR_SHAPE
    st = fq._lib.fp8q_linear_fwd_splitk(fq._ptr(qx), fq._ptr(sx), sx.shape[1], fq._ptr(qw),
                                        fq._ptr(sw), 16, 4096, 4096, fq._ptr(y), 4096, None,
                                        0, fq._stream())
    assert st == fq.FP8Q_ERR_NULL
