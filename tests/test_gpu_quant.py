"""Parity of the quantizer kernels with the oracle: codes and scales bit-exact, on the
tiny linear layer, ragged and degenerate inputs, an exhaustive sweep of BF16 inputs
through the E4M3 conversion, and (sampled) the full Llama-3.1-8B layer sizes."""
import numpy as np
import pytest
import torch

import workloads
from gpu_util import assert_codes_equal, assert_scales_equal, bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import fp8_block_scaled_08_b200 as f
    return f


DEV = "cuda"


def run_act(fq, x):
    q, s = fq.quant_act_1x128_alloc(x)
    torch.cuda.synchronize()
    return q, s


# ---------------------------------------------------------------- a1
@pytest.mark.parametrize("M,K", [(256, 512), (1, 128), (3, 384), (200, 1280), (17, 128 * 7)])
def test_act_quant_matches_oracle(fq, oracle_mod, M, K):
    x = workloads.activations_bf16((M, K), 0, 100 + M, DEV, outlier_count=min(4, K // 64),
                                   outlier_scale=30.0)
    q, s = run_act(fq, x)
    rq, rs = oracle_mod.quant_act_1x128(bits(x))
    assert_codes_equal(q, rq, "a1 codes")
    assert_scales_equal(s, rs, "a1 scales", cols=M)


def test_act_quant_strided_input_and_lds(fq, oracle_mod):
    big = workloads.activations_bf16((64, 1024), 0, 140, DEV)
    x = big[:, 256:768]                      # row stride 1024, 512 columns
    q = torch.empty((64, 512), dtype=torch.uint8, device=DEV)
    s = torch.full((4, 72), -1.0, device=DEV)  # lds = 72 > M
    fq.quant_act_1x128(x, q, s)
    torch.cuda.synchronize()
    rq, rs = oracle_mod.quant_act_1x128(bits(x.contiguous()), lds=72)
    assert_codes_equal(q, rq, "a1 strided")
    assert_scales_equal(s, rs, "a1 strided scales", cols=64)
    assert torch.all(s[:, 64:] == -1.0)      # padding columns untouched


def test_e4m3_conversion_exhaustive_over_bf16(fq, oracle_mod):
    """Every finite BF16 value with |x| <= 448, placed in groups whose amax is exactly
    448 (so s = 1 and t = x): the kernel's codes equal the oracle's encoder."""
    pat = np.arange(65536, dtype=np.uint32)
    vals = (pat << 16).view(np.float32)
    keep = np.isfinite(vals) & (np.abs(vals) <= 448.0)
    pats = pat[keep].astype(np.uint16)
    n_per = 127
    groups = -(-len(pats) // n_per)
    arr = np.zeros((groups, 128), np.uint16)
    arr[:, 0] = 0x43E0  # BF16 448.0
    flat = np.zeros(groups * n_per, np.uint16)
    flat[: len(pats)] = pats
    arr[:, 1:] = flat.reshape(groups, n_per)
    x = torch.from_numpy(arr.view(np.int16)).view(torch.bfloat16).to(DEV)
    q, s = run_act(fq, x)
    rq, rs = oracle_mod.quant_act_1x128(arr)
    assert np.all(rs[0, :groups] == 1.0)
    assert_codes_equal(q, rq, "exhaustive e4m3")


def test_special_groups(fq, oracle_mod):
    """All-zero groups (s = 1), negative zeros (code 0x80), subnormal-range amax (an fp32
    subnormal scale), single nonzero elements and the largest BF16 magnitude."""
    x = torch.zeros((6, 256), dtype=torch.bfloat16)
    xv = x.view(torch.int16)
    xv[1, 5] = -32768            # -0.0 in a zero group
    xv[2, :128] = 0x0001         # smallest BF16 subnormal everywhere
    xv[2, 7] = -32765            # 0x8003: -3 x 2^-133
    x[3, 128] = -1e-30
    x[4, :] = torch.linspace(-3e38, 3e38, 256, dtype=torch.float64)  # finite (fp64 steps)
    x[5, 130] = 3.0
    x[5, 131] = -0.0
    q, s = run_act(fq, x.to(DEV))
    rq, rs = oracle_mod.quant_act_1x128(bits(x))
    assert_codes_equal(q, rq, "special codes")
    assert_scales_equal(s, rs, "special scales", cols=6)


def test_zero_groups_in_tile_and_row_kernels(fq, oracle_mod):
    """All-zero groups and blocks next to ordinary ones (s = 1; codes of +0 and -0) through
    a6 (rows, columns), a2 (a zero 128x128 block) and a3 on the lane-per-group path with a
    partial last round of groups (H = 3584: 28 groups) and a zero row."""
    dy = workloads.gradients_bf16((256, 384), 1e-3, 0, 901, "cpu")
    dy[:, 128:256] = 0.0                 # zero column groups and row groups
    dy[130:140] = 0.0                    # zero rows
    dyv = dy.view(torch.int16)
    dyv[131, 200] = -32768               # -0.0 inside zero groups
    dyv[5, 150] = -32768
    q_row, s_row, q_colT, s_col = fq.transpose_quant_bf16_alloc(dy.to(DEV))
    w = workloads.normal_bf16((256, 384), 0.02, 0, 902, "cpu")
    w[128:, 128:256] = 0.0               # one zero block
    w.view(torch.int16)[200, 130] = -32768
    qw, sw, qwT = fq.quant_weight_alloc(w.to(DEV))
    x = workloads.activations_bf16((1100, 3584), 0, 903, "cpu", outlier_frac=0.005,
                                   outlier_scale=50.0)
    x[17] = 0.0
    g = workloads.gamma_bf16(3584, 0, 904, "cpu")
    qn, sn = fq.rmsnorm_quant_alloc(x.to(DEV), g.to(DEV), 1e-5)
    torch.cuda.synchronize()
    rqr, rsr, rqc, rsc = oracle_mod.transpose_quant_bf16(bits(dy))
    assert_codes_equal(q_row, rqr, "a6 row codes, zero groups")
    assert_scales_equal(s_row, rsr, "a6 row scales, zero groups", cols=256)
    assert_codes_equal(q_colT, rqc, "a6 column codes, zero groups")
    assert_scales_equal(s_col, rsc, "a6 column scales, zero groups")
    rq, rs, rqT = oracle_mod.quant_weight_128x128(bits(w))
    assert_codes_equal(qw, rq, "a2 codes, zero block")
    assert_codes_equal(qwT, rqT, "a2 transposed codes, zero block")
    assert_scales_equal(sw, rs, "a2 scales, zero block")
    rqn, rsn = oracle_mod.rmsnorm_quant(bits(x), bits(g), 1e-5)
    assert_codes_equal(qn, rqn, "a3 codes, 28 groups")
    assert_scales_equal(sn, rsn, "a3 scales, 28 groups", cols=1100)


def test_quotient_dense_sweep(fq, oracle_mod):
    """Groups whose amax is a chosen BF16 value and whose other 127 elements sweep the
    BF16 values below it: the kernel's quotient path against the oracle's IEEE
    division, across every binade of amax (including fp32-subnormal scales)."""
    rng = np.random.default_rng(5)
    amax_bits = np.concatenate([rng.integers(0x0001, 0x7F80, 1500), [0x0001, 0x0080, 0x43E0, 0x7F7F]])
    rows = []
    for ab in amax_bits:
        xs = rng.integers(0, int(ab) + 1, 127 * 8).astype(np.uint16)
        xs |= (rng.integers(0, 2, xs.size) << 15).astype(np.uint16)  # random signs
        for k in range(8):
            row = np.empty(128, np.uint16)
            row[0] = ab
            row[1:] = xs[127 * k: 127 * (k + 1)]
            rows.append(row)
    arr = np.stack(rows)
    x = torch.from_numpy(arr.view(np.int16)).view(torch.bfloat16).to(DEV)
    q, s = run_act(fq, x)
    rq, rs = oracle_mod.quant_act_1x128(arr)
    assert_codes_equal(q, rq, "dense quotient sweep")
    assert_scales_equal(s, rs, "dense quotient sweep scales", cols=arr.shape[0])


def test_swiglu_exhaustive_gate(fq, oracle_mod):
    """Every BF16 gate value g with |g| <= 1e37, with up-projections u in {1, -0.5, 3.25}: SwiGLU
    depends on g only through the fixed exponential and an IEEE division, so this
    covers the kernel's whole silu path."""
    pat = np.arange(65536, dtype=np.uint32)
    vals = (pat << 16).view(np.float32)
    gates = pat[np.isfinite(vals) & (np.abs(vals) <= 1e37)].astype(np.uint16)  # h stays finite
    n = -(-len(gates) // 128) * 128
    g = np.zeros(n, np.uint16)
    g[: len(gates)] = gates
    g = g.reshape(-1, 128)
    for u in (1.0, -0.5, 3.25):
        ub = np.full_like(g, np.float32(u).view(np.uint32) >> 16)
        arr = np.concatenate([g, ub], axis=1)                     # [rows, 2I] with I = 128
        x = torch.from_numpy(arr.view(np.int16)).view(torch.bfloat16).to(DEV)
        q, s = fq.swiglu_quant_alloc(x)
        torch.cuda.synchronize()
        rq, rs = oracle_mod.swiglu_quant(arr)
        assert_codes_equal(q, rq, "swiglu exhaustive u=%g" % u)
        assert_scales_equal(s, rs, "swiglu exhaustive scales u=%g" % u, cols=arr.shape[0])


# ---------------------------------------------------------------- a2
@pytest.mark.parametrize("N,K", [(512, 512), (128, 128), (384, 256)])
def test_weight_quant_matches_oracle(fq, oracle_mod, N, K):
    w = workloads.normal_bf16((N, K), 0.02, 0, 200 + N, DEV)
    q, s, qT = fq.quant_weight_alloc(w)
    torch.cuda.synchronize()
    rq, rs, rqT = oracle_mod.quant_weight_128x128(bits(w))
    assert_codes_equal(q, rq, "a2 codes")
    assert_codes_equal(qT, rqT, "a2 transposed codes")
    assert_scales_equal(s, rs, "a2 scales")


# ---------------------------------------------------------------- a3
# batches up to 1024 rows take the CTA-per-row kernel; above, H a multiple of 128 with at
# most 64 groups takes the lane-per-group kernel (1100 x 640: 5 groups; 2050 x 4096: one
# group per lane; 1040 x 4224 and 1030 x 6144: lanes with a second group), otherwise the
# two-pass warp-per-row kernel (1025 x 16384: widest; 1060 x 4112: H not a multiple of 128)
@pytest.mark.parametrize("M,H,eps", [(256, 512, 1e-5), (5, 4096, 1e-6), (130, 3584, 1e-5),
                                     (3, 16384, 0.0), (64, 128, 1e-5), (1100, 640, 1e-5),
                                     (1030, 6144, 1e-6), (1025, 16384, 1e-5),
                                     (1040, 4224, 0.0), (2050, 4096, 1e-5), (1060, 4112, 1e-5)])
def test_rmsnorm_quant_matches_oracle(fq, oracle_mod, M, H, eps):
    x = workloads.activations_bf16((M, H), 0, 300 + M, DEV, outlier_frac=0.005,
                                   outlier_scale=50.0)
    g = workloads.gamma_bf16(H, 0, 301, DEV)
    q, s = fq.rmsnorm_quant_alloc(x, g, eps)
    torch.cuda.synchronize()
    rq, rs = oracle_mod.rmsnorm_quant(bits(x), bits(g), eps)
    assert_codes_equal(q, rq, "a3 codes")
    assert_scales_equal(s, rs, "a3 scales", cols=M)


def test_rmsnorm_zero_row(fq, oracle_mod):
    x = torch.zeros((2, 256), dtype=torch.bfloat16, device=DEV)
    x[1] = 1.0
    g = torch.ones(256, dtype=torch.bfloat16, device=DEV)
    q, s = fq.rmsnorm_quant_alloc(x, g, 1e-5)
    torch.cuda.synchronize()
    rq, rs = oracle_mod.rmsnorm_quant(bits(x), bits(g), 1e-5)
    assert_codes_equal(q, rq, "a3 zero row")
    assert_scales_equal(s, rs, "a3 zero row scales", cols=2)


# ---------------------------------------------------------------- a4
@pytest.mark.parametrize("M,I", [(256, 256), (7, 1408), (64, 128), (33, 384)])
def test_swiglu_quant_matches_oracle(fq, oracle_mod, M, I):
    gu = (workloads.normal_bf16((M, 2 * I), 1.0, 0, 400 + M, DEV).float() * 4).to(torch.bfloat16)
    q, s = fq.swiglu_quant_alloc(gu)
    torch.cuda.synchronize()
    rq, rs = oracle_mod.swiglu_quant(bits(gu))
    assert_codes_equal(q, rq, "a4 codes")
    assert_scales_equal(s, rs, "a4 scales", cols=M)


def test_swiglu_extreme_gates(fq, oracle_mod):
    """Gate values across the exp clamp (-80 / 88) and exact zeros."""
    g = torch.linspace(-120, 120, 256)
    u = torch.linspace(-2, 3, 256)
    gu = torch.cat([g, u]).reshape(1, 512).repeat(4, 1)
    gu[1, :256] = 0.0
    gu[2, :256] *= -1
    gu[3, 256:] = 0.0
    gu = gu.to(torch.bfloat16)
    q, s = fq.swiglu_quant_alloc(gu.to(DEV))
    torch.cuda.synchronize()
    rq, rs = oracle_mod.swiglu_quant(bits(gu))
    assert_codes_equal(q, rq, "a4 extremes")
    assert_scales_equal(s, rs, "a4 extremes scales", cols=4)


def test_swiglu_every_bf16_gate(fq, oracle_mod):
    """Every BF16 gate value below 2^61 in magnitude (the kernel tabulates the gate factor
    for 2^-24 <= |g| < 2^7 and computes it directly elsewhere; larger gates would make h
    overflow), each with an up value drawn from N(0, 1); 512 rows of 128 gates, so some
    groups mix table and direct gates and some hold only one kind."""
    pats = np.arange(65536, dtype=np.uint32)
    pats = pats[((pats >> 7) & 0xFF) < 127 + 61].astype(np.uint16)
    pats = np.resize(pats, 512 * 128)  # repeats the start to fill the rows
    rng = np.random.default_rng(5)
    order = rng.permutation(pats.size)
    order[: pats.size // 2] = np.sort(order[: pats.size // 2])  # half the rows in order
    g = torch.from_numpy(pats[order].view(np.int16).reshape(512, 128).copy()).view(torch.bfloat16)
    u = workloads.normal_bf16((512, 128), 1.0, 0, 77, "cpu")
    gu = torch.cat([g, u], 1).contiguous()
    q, s = fq.swiglu_quant_alloc(gu.to(DEV))
    torch.cuda.synchronize()
    rq, rs = oracle_mod.swiglu_quant(bits(gu))
    assert_codes_equal(q, rq, "a4 every gate")
    assert_scales_equal(s, rs, "a4 every gate scales", cols=512)


# ---------------------------------------------------------------- a6
@pytest.mark.parametrize("M,N", [(256, 512), (128, 128), (384, 256)])
def test_transpose_quant_bf16_matches_oracle(fq, oracle_mod, M, N):
    dy = workloads.gradients_bf16((M, N), 1e-3, 0, 500 + M, DEV, small_row_frac=0.02,
                                  small_row_scale=1e-3)
    q_row, s_row, q_colT, s_col = fq.transpose_quant_bf16_alloc(dy)
    torch.cuda.synchronize()
    rqr, rsr, rqc, rsc = oracle_mod.transpose_quant_bf16(bits(dy))
    assert_codes_equal(q_row, rqr, "a6 row codes")
    assert_scales_equal(s_row, rsr, "a6 row scales", cols=M)
    assert_codes_equal(q_colT, rqc, "a6 column codes")
    assert_scales_equal(s_col, rsc, "a6 column scales")


def test_transpose_quant_bf16_column_only(fq, oracle_mod):
    dy = workloads.gradients_bf16((256, 384), 1e-3, 0, 520, DEV)
    _, _, q_colT, s_col = fq.transpose_quant_bf16_alloc(dy, want_row=False)
    torch.cuda.synchronize()
    _, _, rqc, rsc = oracle_mod.transpose_quant_bf16(bits(dy), want_row=False)
    assert_codes_equal(q_colT, rqc, "a6 column-only codes")
    assert_scales_equal(s_col, rsc, "a6 column-only scales")


# ---------------------------------------------------------------- a8
@pytest.mark.parametrize("M,K", [(256, 512), (128, 128), (384, 640)])
def test_transpose_quant_fp8_matches_oracle(fq, oracle_mod, M, K):
    x = workloads.activations_bf16((M, K), 0, 600 + M, DEV, outlier_count=4, outlier_scale=30.0)
    q, s = fq.quant_act_1x128_alloc(x)
    qT, sT = fq.transpose_quant_fp8_alloc(q, s)
    torch.cuda.synchronize()
    rq, rs = oracle_mod.quant_act_1x128(bits(x))
    rqT, rsT = oracle_mod.transpose_quant_fp8(rq, rs)
    assert_codes_equal(qT, rqT, "a8 codes")
    assert_scales_equal(sT, rsT, "a8 scales")


# ---------------------------------------------------------------- full sizes (sampled)
def test_full_size_llama_layer_quantizers_sampled(fq, oracle_mod):
    """Llama-3.1-8B layer at M = 8192: every quantizer at full size, in the launch
    configuration the benchmark uses; rows (or 128-row blocks) sampled for the oracle."""
    wl = workloads.LLAMA_LAYER
    inp = workloads.layer_inputs(wl, DEV)
    rng = np.random.default_rng(0)
    rows = np.sort(rng.choice(wl.tokens, 48, replace=False))
    # a3 on the attention input
    q, s = fq.rmsnorm_quant_alloc(inp["x_attn"], inp["gamma1"], wl.eps)
    # a1 on the attention output
    qa, sa = fq.quant_act_1x128_alloc(inp["attn_out"])
    torch.cuda.synchronize()
    xr = bits(inp["x_attn"][rows])
    rq, rs = oracle_mod.rmsnorm_quant(xr, bits(inp["gamma1"]), wl.eps)
    assert_codes_equal(q[rows], rq, "a3 full-size sampled")
    assert np.array_equal(s.cpu().numpy()[:, rows].view(np.uint32), rs[:, :len(rows)].view(np.uint32))
    rqa, rsa = oracle_mod.quant_act_1x128(bits(inp["attn_out"][rows]))
    assert_codes_equal(qa[rows], rqa, "a1 full-size sampled")
    assert np.array_equal(sa.cpu().numpy()[:, rows].view(np.uint32), rsa[:, :len(rows)].view(np.uint32))
    # a4 on a gate/up activation of full size
    I = wl.layer.intermediate
    gu = workloads.normal_bf16((wl.tokens, 2 * I), 1.5, 0, 700, DEV)
    qh, sh = fq.swiglu_quant_alloc(gu)
    torch.cuda.synchronize()
    rqh, rsh = oracle_mod.swiglu_quant(bits(gu[rows]))
    assert_codes_equal(qh[rows], rqh, "a4 full-size sampled")
    assert np.array_equal(sh.cpu().numpy()[:, rows].view(np.uint32), rsh[:, :len(rows)].view(np.uint32))
    del gu, qh, sh
    # a2 on the gate/up weight: sampled 128-row blocks
    w = inp["w"]["gate_up"]
    qw, sw, qwT = fq.quant_weight_alloc(w)
    torch.cuda.synchronize()
    for nb in rng.choice(w.shape[0] // 128, 3, replace=False):
        r0 = int(nb) * 128
        rqw, rsw, _ = oracle_mod.quant_weight_128x128(bits(w[r0:r0 + 128]), want_t=False)
        assert_codes_equal(qw[r0:r0 + 128], rqw, "a2 full-size block")
        assert_codes_equal(qwT[:, r0:r0 + 128], np.ascontiguousarray(rqw.T), "a2 full-size qT")
        assert np.array_equal(sw[nb].cpu().numpy().view(np.uint32), rsw[0].view(np.uint32))
    del qw, sw, qwT
    # a6 on the down-projection gradient, a8 on the saved attention-input activation:
    # 128-row blocks sampled (each is a complete set of column groups)
    dy = inp["dy"]["down"]
    qr, sr, qc, sc = fq.transpose_quant_bf16_alloc(dy)
    qxT, sxT = fq.transpose_quant_fp8_alloc(q, s)
    torch.cuda.synchronize()
    for mb in rng.choice(wl.tokens // 128, 2, replace=False):
        m0 = int(mb) * 128
        rqr, rsr, rqc, rsc = oracle_mod.transpose_quant_bf16(bits(dy[m0:m0 + 128]))
        assert_codes_equal(qr[m0:m0 + 128], rqr, "a6 full-size rows")
        assert_codes_equal(qc[:, m0:m0 + 128], rqc, "a6 full-size columns")
        assert np.array_equal(sc[mb].cpu().numpy().view(np.uint32), rsc[0].view(np.uint32))
        rq8, rs8 = oracle_mod.rmsnorm_quant(bits(inp["x_attn"][m0:m0 + 128]), bits(inp["gamma1"]),
                                            wl.eps)
        rqT, rsT = oracle_mod.transpose_quant_fp8(rq8, rs8)
        assert_codes_equal(qxT[:, m0:m0 + 128], rqT, "a8 full-size")
        assert np.array_equal(sxT[mb].cpu().numpy().view(np.uint32), rsT[0].view(np.uint32))
