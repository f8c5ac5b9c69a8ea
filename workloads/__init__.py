"""Seeded synthetic inputs and layer shapes for the block-scaled FP8 linear path.

This module holds no arithmetic of the method: it only draws random BF16 tensors
and names shapes. Both the CUDA path (tests, bench) and the oracle (tests, CPU
baseline) receive the same bytes from here.

Recipe (same for every tensor): draw fp32 values with a seeded ``torch.Generator``
(sub-stream seed = 1000 * seed + tensor_id), shape them as the workload says, and
round to BF16 (round to nearest even). The shapes are the model shapes the Jet-RL
pages evaluate (Llama3.1-8B, Qwen2.5-7B, Qwen3-8B, a 32B model; "Resultados
Experimentales" / "Eficiencia"); no trained weights or datasets are used.
"""
from __future__ import annotations

import dataclasses

import torch


# --------------------------------------------------------------------------
# Layer shapes
# --------------------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class Linear:
    name: str
    n: int   # output features
    k: int   # input features


@dataclasses.dataclass(frozen=True)
class LayerShape:
    name: str
    hidden: int
    intermediate: int
    q_heads: int
    kv_heads: int
    head_dim: int

    @property
    def linears(self):
        qkv = (self.q_heads + 2 * self.kv_heads) * self.head_dim
        return [
            Linear("qkv", qkv, self.hidden),
            Linear("o", self.hidden, self.q_heads * self.head_dim),
            Linear("gate_up", 2 * self.intermediate, self.hidden),
            Linear("down", self.hidden, self.intermediate),
        ]


LLAMA31_8B = LayerShape("llama3.1-8b", 4096, 14336, 32, 8, 128)
QWEN3_8B = LayerShape("qwen3-8b", 4096, 12288, 32, 8, 128)
QWEN25_7B = LayerShape("qwen2.5-7b", 3584, 18944, 28, 4, 128)
DENSE_32B = LayerShape("32b-class", 5120, 27648, 40, 8, 128)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    layer: LayerShape | None
    tokens: int
    act_outlier_frac: float = 0.0
    act_outlier_scale: float = 1.0
    act_outlier_count: int = 0
    act_heavy_tail_frac: float = 0.0
    w_std: float = 0.02
    dy_std: float = 1e-3
    dy_small_row_frac: float = 0.0
    dy_small_row_scale: float = 1.0
    eps: float = 1e-5
    seed: int = 0


# Single linear layer, tiny: X [256,512] with 4 outlier columns x30, W [512,512],
# dY [256,512].
TINY = Workload("tiny-linear-256x512x512", None, 256, act_outlier_count=4,
                act_outlier_scale=30.0, w_std=0.02, dy_std=1e-3)
# Llama-3.1-8B decoder layer, M = 8192 tokens, 0.5% outlier channels x50.
LLAMA_LAYER = Workload("llama3.1-8b-layer-m8192", LLAMA31_8B, 8192,
                       act_outlier_frac=0.005, act_outlier_scale=50.0,
                       w_std=0.02, dy_std=1e-3, eps=1e-5)
# Qwen3-8B decode shapes, M in {16, 64, 256}, forward only.
QWEN3_DECODE = [Workload("qwen3-8b-decode-m%d" % m, QWEN3_8B, m, w_std=0.02, eps=1e-6)
                for m in (16, 64, 256)]
# Qwen2.5-7B long-context layer, M = 16384; gradients N(0,1e-4) with 1% of rows x1e-3.
QWEN25_LONG = Workload("qwen2.5-7b-layer-m16384", QWEN25_7B, 16384, w_std=0.02,
                       dy_std=1e-4, dy_small_row_frac=0.01, dy_small_row_scale=1e-3,
                       eps=1e-6)
# 32B-class layer, M = 8192 training and M = 128 decode; W ~ N(0, 0.015),
# activations with 1% heavy-tailed Student-t(3) channels.
DENSE32_TRAIN = Workload("32b-layer-m8192", DENSE_32B, 8192, w_std=0.015,
                         act_heavy_tail_frac=0.01, eps=1e-5)
DENSE32_DECODE = Workload("32b-decode-m128", DENSE_32B, 128, w_std=0.015,
                          act_heavy_tail_frac=0.01, eps=1e-5)


# --------------------------------------------------------------------------
# Generators
# --------------------------------------------------------------------------

def _gen(seed: int, tensor_id: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(1000 * seed + tensor_id)
    return g


def _randn(shape, seed, tensor_id, device):
    return torch.randn(*shape, generator=_gen(seed, tensor_id, device),
                       device=device, dtype=torch.float32)


def _pick(n: int, count: int, seed: int, tensor_id: int) -> torch.Tensor:
    """`count` distinct indices in [0, n) from a seeded permutation (CPU)."""
    g = _gen(seed, tensor_id, "cpu")
    return torch.randperm(n, generator=g)[:count]


def normal_bf16(shape, std: float, seed: int, tensor_id: int, device="cpu"):
    """N(0, std) rounded to BF16."""
    return (_randn(shape, seed, tensor_id, device) * std).to(torch.bfloat16)


def activations_bf16(shape, seed: int, tensor_id: int, device="cpu",
                     outlier_count: int = 0, outlier_frac: float = 0.0,
                     outlier_scale: float = 1.0, heavy_tail_frac: float = 0.0):
    """N(0,1) activations [M, C]; chosen channels are multiplied by `outlier_scale`
    (count given directly or as a fraction of C, rounded) or replaced by
    Student-t(3) draws (Z / sqrt(chi2_3 / 3))."""
    M, C = shape
    x = _randn(shape, seed, tensor_id, device)
    n_out = outlier_count or int(round(outlier_frac * C))
    if n_out:
        cols = _pick(C, n_out, seed, tensor_id + 500).to(device)
        x[:, cols] *= outlier_scale
    n_t = int(round(heavy_tail_frac * C))
    if n_t:
        cols = _pick(C, n_t, seed, tensor_id + 600).to(device)
        z = _randn((M, n_t), seed, tensor_id + 700, device)
        chi = _randn((M, n_t, 3), seed, tensor_id + 800, device).square().sum(-1)
        x[:, cols] = z / torch.sqrt(chi / 3.0)
    return x.to(torch.bfloat16)


def gradients_bf16(shape, std: float, seed: int, tensor_id: int, device="cpu",
                   small_row_frac: float = 0.0, small_row_scale: float = 1.0):
    """N(0, std) upstream gradients [M, N]; a seeded fraction of rows is scaled by
    `small_row_scale` (an underflow probe)."""
    g = _randn(shape, seed, tensor_id, device) * std
    n_rows = int(round(small_row_frac * shape[0]))
    if n_rows:
        rows = _pick(shape[0], n_rows, seed, tensor_id + 500).to(device)
        g[rows] *= small_row_scale
    return g.to(torch.bfloat16)


def gamma_bf16(h: int, seed: int, tensor_id: int, device="cpu"):
    """RMSNorm weight 1 + 0.1 N(0,1), rounded to BF16."""
    return (1.0 + 0.1 * _randn((h,), seed, tensor_id, device)).to(torch.bfloat16)


# Tensor ids (sub-streams) used by the layer workloads.
TID_X_ATTN, TID_X_MLP, TID_ATTN_OUT = 1, 2, 3
TID_GAMMA1, TID_GAMMA2 = 4, 5
TID_W = {"qkv": 10, "o": 11, "gate_up": 12, "down": 13}
TID_DY = {"qkv": 20, "o": 21, "gate_up": 22, "down": 23}
TID_TINY_X, TID_TINY_W, TID_TINY_DY = 30, 31, 32


def tiny_inputs(device="cpu", wl: Workload = TINY):
    """X [256,512] (4 outlier columns x30), W [512,512] ~ N(0,0.02), dY [256,512] ~ N(0,1e-3)."""
    x = activations_bf16((256, 512), wl.seed, TID_TINY_X, device,
                         outlier_count=wl.act_outlier_count,
                         outlier_scale=wl.act_outlier_scale)
    w = normal_bf16((512, 512), wl.w_std, wl.seed, TID_TINY_W, device)
    dy = gradients_bf16((256, 512), wl.dy_std, wl.seed, TID_TINY_DY, device)
    return x, w, dy


def layer_inputs(wl: Workload, device="cpu", tokens: int | None = None,
                 with_grads: bool = True):
    """Every input of one decoder-layer pass of the linear path.

    Returns a dict: x_attn / x_mlp (pre-norm residual streams), attn_out (stand-in for
    the attention output that feeds the O projection), gamma1 / gamma2, w[name] (BF16
    masters), dy[name] (upstream BF16 gradients of each linear's output)."""
    L = wl.layer
    M = wl.tokens if tokens is None else tokens
    H = L.hidden
    kw = dict(outlier_frac=wl.act_outlier_frac, outlier_scale=wl.act_outlier_scale,
              heavy_tail_frac=wl.act_heavy_tail_frac)
    out = {
        "x_attn": activations_bf16((M, H), wl.seed, TID_X_ATTN, device, **kw),
        "x_mlp": activations_bf16((M, H), wl.seed, TID_X_MLP, device, **kw),
        "attn_out": activations_bf16((M, L.q_heads * L.head_dim), wl.seed,
                                     TID_ATTN_OUT, device, **kw),
        "gamma1": gamma_bf16(H, wl.seed, TID_GAMMA1, device),
        "gamma2": gamma_bf16(H, wl.seed, TID_GAMMA2, device),
        "w": {lin.name: normal_bf16((lin.n, lin.k), wl.w_std, wl.seed, TID_W[lin.name],
                                    device) for lin in L.linears},
        "dy": {},
    }
    if with_grads:
        for lin in L.linears:
            out["dy"][lin.name] = gradients_bf16(
                (M, lin.n), wl.dy_std, wl.seed, TID_DY[lin.name], device,
                small_row_frac=wl.dy_small_row_frac,
                small_row_scale=wl.dy_small_row_scale)
    return out


def layer_gemm_flops(layer: LayerShape, tokens: int, passes: int = 3) -> float:
    """2*M*N*K per linear, times `passes` (fwd, DGrad, WGrad)."""
    return float(passes) * sum(2.0 * tokens * lin.n * lin.k for lin in layer.linears)


def round_up(x: int, m: int) -> int:
    return (x + m - 1) // m * m


def lds_for(m: int) -> int:
    """Smallest legal leading dimension of a 1x128 scale array for M rows."""
    return round_up(max(m, 1), 4)

