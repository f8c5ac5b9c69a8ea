"""The Python binding checks every operand's dtype and extents before it hands a pointer
to the C ABI: the library builds its tensor maps and stores from the sizes it is given,
so a mismatched tensor must be refused on the host, before any launch.

Runs on CPU: the tensors here live in host memory, so a call whose operands all check
out stops at the device-pointer step with "takes CUDA tensors"; a call with one wrong
operand must stop earlier, with a ValueError that names that operand."""
import pytest
import torch

import fp8_block_scaled_08_b200 as fq

M, N, K = 256, 384, 512


def u8(*s):
    return torch.zeros(s, dtype=torch.uint8)


def f32(*s):
    return torch.zeros(s, dtype=torch.float32)


def bf16(*s):
    return torch.zeros(s, dtype=torch.bfloat16)


def fwd_args():
    return dict(qa=u8(M, K), sa=f32(K // 128, M), qw=u8(N, K), sw=f32(N // 128, K // 128),
                y=bf16(M, N))


def dgrad_args():
    return dict(qdy=u8(M, N), sdy=f32(N // 128, M), qwT=u8(K, N), sw=f32(N // 128, K // 128),
                dx=bf16(M, K))


def wgrad_args(out=torch.bfloat16):
    return dict(qdyT=u8(N, M), sdy_c=f32(M // 128, N), qxT=u8(K, M), sx_c=f32(M // 128, K),
                dw=torch.zeros((N, K), dtype=out))


CASES = [
    # (binding, argument factory, operand, wrong value)
    (fq.linear_fwd, fwd_args, "qw", u8(N, K + 128)),
    (fq.linear_fwd, fwd_args, "qw", f32(N, K)),
    (fq.linear_fwd, fwd_args, "sa", f32(K // 128, M - 4)),
    (fq.linear_fwd, fwd_args, "sa", f32(K // 128 + 1, M)),
    (fq.linear_fwd, fwd_args, "sw", f32(N // 128, K // 128 + 1)),
    (fq.linear_fwd, fwd_args, "sw", f32(K // 128, N // 128)),
    (fq.linear_fwd, fwd_args, "y", bf16(M, N - 128)),
    (fq.linear_fwd, fwd_args, "y", bf16(M + 1, N)),
    (fq.linear_fwd, fwd_args, "y", f32(M, N)),
    (fq.linear_fwd, fwd_args, "qa", torch.zeros((M, K), dtype=torch.int8)),
    (fq.linear_fwd_splitk_noalloc, fwd_args, "qw", u8(N + 128, K - 128)),
    (fq.linear_fwd_splitk_noalloc, fwd_args, "sw", f32(N // 128 + 1, K // 128)),
    (fq.linear_fwd_splitk_noalloc, fwd_args, "y", bf16(M, N + 8)),
    (fq.linear_dgrad, dgrad_args, "qwT", u8(K, N + 128)),
    (fq.linear_dgrad, dgrad_args, "sw", f32(K // 128, N // 128)),
    (fq.linear_dgrad, dgrad_args, "sdy", f32(N // 128, M - 4)),
    (fq.linear_dgrad, dgrad_args, "dx", bf16(M, N)),
    (fq.linear_wgrad, wgrad_args, "qxT", u8(K, M + 128)),
    (fq.linear_wgrad, wgrad_args, "sdy_c", f32(M // 128, N + 128)),
    (fq.linear_wgrad, wgrad_args, "sx_c", f32(M // 128 + 1, K)),
    (fq.linear_wgrad, wgrad_args, "dw", bf16(K, N)),
    (fq.linear_wgrad_acc_f32, lambda: wgrad_args(torch.float32), "dw", bf16(N, K)),
    (fq.linear_wgrad_acc_f32, lambda: wgrad_args(torch.float32), "sx_c", f32(M // 128, K - 128)),
]


@pytest.mark.parametrize("fn,factory,name,wrong", CASES,
                         ids=["%s-%s-%d" % (c[0].__name__, c[2], i) for i, c in enumerate(CASES)])
def test_gemm_binding_refuses_a_mismatched_operand(fn, factory, name, wrong):
    args = factory()
    args[name] = wrong
    with pytest.raises(ValueError, match=r"\b%s\b" % name):
        fn(**args)


@pytest.mark.parametrize("fn,factory", [(fq.linear_fwd, fwd_args),
                                        (fq.linear_fwd_splitk_noalloc, fwd_args),
                                        (fq.linear_dgrad, dgrad_args),
                                        (fq.linear_wgrad, wgrad_args),
                                        (fq.linear_wgrad_acc_f32,
                                         lambda: wgrad_args(torch.float32))])
def test_gemm_binding_accepts_matching_operands(fn, factory):
    # every extent matches: the call gets as far as the device-pointer check
    with pytest.raises(ValueError, match="CUDA tensors"):
        fn(**factory())


def quant_cases():
    H, I = K, 384
    x = bf16(M, H)
    g = bf16(H)
    gu = bf16(M, 2 * I)
    return [
        (fq.quant_act_1x128, dict(x=x, q=u8(M, H), s=f32(H // 128, M)), "q", u8(M, H - 128)),
        (fq.quant_act_1x128, dict(x=x, q=u8(M, H), s=f32(H // 128, M)), "s", f32(H // 128, M - 4)),
        (fq.quant_weight_128x128, dict(w=bf16(N, K), q=u8(N, K), s=f32(N // 128, K // 128),
                                       qT=u8(K, N)), "qT", u8(N, K)),
        (fq.quant_weight_128x128, dict(w=bf16(N, K), q=u8(N, K), s=f32(N // 128, K // 128)),
         "s", f32(K // 128, N // 128)),
        (fq.rmsnorm_quant, dict(x=x, gamma=g, eps=1e-5, q=u8(M, H), s=f32(H // 128, M)),
         "gamma", bf16(H - 128)),
        (fq.rmsnorm_quant, dict(x=x, gamma=g, eps=1e-5, q=u8(M, H), s=f32(H // 128, M)),
         "q", u8(M + 128, H)),
        (fq.swiglu_quant, dict(gu=gu, q=u8(M, I), s=f32(I // 128, M)), "q", u8(M, 2 * I)),
        (fq.swiglu_quant, dict(gu=gu, q=u8(M, I), s=f32(I // 128, M)), "s", f32(2 * I // 128, M)),
        (fq.transpose_quant_bf16, dict(dy=bf16(M, N), q_row=u8(M, N), s_row=f32(N // 128, M),
                                       q_colT=u8(N, M), s_col=f32(M // 128, N)),
         "q_colT", u8(M, N)),
        (fq.transpose_quant_bf16, dict(dy=bf16(M, N), q_row=u8(M, N), s_row=f32(N // 128, M),
                                       q_colT=u8(N, M), s_col=f32(M // 128, N)),
         "s_col", f32(N // 128, M)),
        (fq.transpose_quant_fp8, dict(q=u8(M, K), s=f32(K // 128, M), qT=u8(K, M),
                                      sT=f32(M // 128, K)), "sT", f32(K // 128, M)),
        (fq.transpose_quant_fp8, dict(q=u8(M, K), s=f32(K // 128, M), qT=u8(K, M),
                                      sT=f32(M // 128, K)), "qT", u8(M, K)),
        (fq.rmsnorm_quant_dual, dict(x=x, gamma=g, eps=1e-5, q_row=u8(M, H),
                                     s_row=f32(H // 128, M), q_colT=u8(H, M),
                                     s_col=f32(M // 128, H), rstd=f32(M)), "rstd", f32(M - 1)),
        (fq.swiglu_quant_dual, dict(gu=gu, q_row=u8(M, I), s_row=f32(I // 128, M),
                                    q_colT=u8(I, M), s_col=f32(M // 128, I)),
         "q_colT", u8(2 * I, M)),
        (fq.swiglu_bwd_quant_dual, dict(gu=gu, dh=bf16(M, I), q_row=u8(M, 2 * I),
                                        s_row=f32(2 * I // 128, M), q_colT=u8(2 * I, M),
                                        s_col=f32(M // 128, 2 * I)), "q_row", u8(M, I)),
    ]


@pytest.mark.parametrize("i", range(15))
def test_quantizer_binding_refuses_a_mismatched_operand(i):
    fn, args, name, wrong = quant_cases()[i]
    good = dict(args)
    with pytest.raises(ValueError, match="CUDA tensors"):
        fn(**good)
    args[name] = wrong
    with pytest.raises(ValueError, match=r"\b%s\b" % name):
        fn(**args)
