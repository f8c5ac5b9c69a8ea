"""Benchmark: one FP8 decoder-layer pass of the linear path per step.

A step runs every operation of the block-scaled FP8 linear path once over one token
batch of the Llama-3.1-8B-shaped layer (M = 8192 tokens, hidden 4096, GQA 32/8 heads,
head_dim 128, intermediate 14336):
  weights: 128x128 quantization of the four BF16 masters (+ transposed codes)
  forward: RMSNorm+quant -> QKV GEMM; 1x128 quant of the attention output -> O GEMM;
           RMSNorm+quant -> gate/up GEMM -> SwiGLU+quant -> down GEMM
  backward, per linear: dual quantization of the BF16 dY (1x128 rows + 128x1 columns),
           DGrad, 128x1 requantization of the saved FP8 input, WGrad
That is 28 kernel launches and 10.72 TFLOP of FP8 GEMM work per step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--saved fp8|dual] [--backward a6|fused]
                    [--case NAME]

--saved dual: the producers emit both groupings of their BF16 output (no FP8
requantization). --backward fused: the SwiGLU and RMSNorm backward producers emit the
gradient codes of the preceding linears (a chained backward; only the QKV gradient,
from attention, and the gradient from the layer above enter from outside). --case runs
one kernel family once, for profiling.

With N > 1 (torchrun, one rank per GPU) every rank runs its own token batch: weak
scaling, no collective on the data path; the step time is the max over ranks.
Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

import workloads  # noqa: E402

METRIC = "FP8 linear fwd+dgrad+wgrad TFLOP/s and % of FP8 peak; quantizer HBM GB/s"
WORKLOAD = workloads.LLAMA_LAYER
# Other layer shapes of the pages, selectable with --workload (secondary measurements;
# the decode shapes run the serving forward pass only, weights quantized once up front).
WORKLOADS = {w.name: w for w in [workloads.LLAMA_LAYER, workloads.QWEN25_LONG,
                                 workloads.DENSE32_TRAIN, workloads.DENSE32_DECODE]
             + list(workloads.QWEN3_DECODE)}


def is_decode(wl) -> bool:
    """Decode-sized token batches run the forward pass only."""
    return wl.tokens < 1024

# Algorithmic bytes per element of each quantizer (reads + writes, scales included).
BYTES_PER_ELEM = {
    "quant_act_1x128": 2 + 1 + 4 / 128,          # per input element
    "rmsnorm_quant": 2 + 1 + 4 / 128,            # per element (gamma negligible)
    "swiglu_quant": 4 + 1 + 4 / 128,             # per output element
    "quant_weight_128x128": 2 + 1 + 1 + 4 / 16384,  # with the transposed copy
    "transpose_quant_bf16": 2 + 2 * (1 + 4 / 128),
    "transpose_quant_fp8": (1 + 4 / 128) * 2,
    # option B producers: read once, write both groupings (the RMSNorm variant reads x a
    # second time for its per-row reciprocal RMS; that re-read is not algorithmic)
    "rmsnorm_quant_dual": 2 + 2 * (1 + 4 / 128),
    "swiglu_quant_dual": 4 + 2 * (1 + 4 / 128),   # per output element
    "transpose_quant_bf16_act": 2 + 2 * (1 + 4 / 128),
    # backward producers with the quantizer fused: gate, up, dh in, both groupings of
    # [d_gate | d_up] out (per (token, i)); x, dy, dres in, BF16 out + both groupings
    "swiglu_bwd_quant_dual": 6 + 2 * 2 * (1 + 4 / 128),
    "rmsnorm_bwd_quant_dual": 6 + 2 + 2 * (1 + 4 / 128),
}
# kernels one call launches (the rest launch one)
KERNELS_PER_CALL = {"rmsnorm_quant_dual": 2, "rmsnorm_bwd_quant_dual": 3}


# B200 dense FP8 tensor throughput from the spec sheet (context beside the measured peak).
NOMINAL_FP8_TFLOPS = 4500.0


def read_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# --------------------------------------------------------------------------
# Multi-rank host logic (weak scaling: one independent token batch per rank)
# --------------------------------------------------------------------------

def rank_seed_offset(rank: int) -> int:
    """Each rank draws its own token batch (and weights): sub-stream seed offset."""
    return rank


def max_over_ranks(value_ms: float, dist=None, device="cpu") -> float:
    """The slowest rank's device-timed duration (all ranks take the same collective)."""
    t = torch.tensor([float(value_ms)], dtype=torch.float64, device=device)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(flops_per_rank: float, world: int, max_ms_per_step: float) -> float:
    """Units all ranks processed divided by the slowest rank's time."""
    return flops_per_rank * world / (max_ms_per_step * 1e-3) / 1e12


# --------------------------------------------------------------------------
# The layer step on the GPU
# --------------------------------------------------------------------------

class LayerStep:
    """Device buffers of one layer pass and the launch sequence (all through the C ABI)."""

    def __init__(self, fq, wl, device, seed_offset=0, forward_only=False, saved="fp8",
                 backward="a6"):
        self.fq = fq
        self.saved = saved  # "fp8": requantize the saved FP8 input for WGrad; "dual": option B
        # "a6": every linear's BF16 upstream gradient is an input, quantized by a6;
        # "fused": the SwiGLU and RMSNorm backward producers emit those codes (chained)
        self.backward = backward
        L = wl.layer
        self.M = M = wl.tokens
        self.L = L
        self.eps = wl.eps
        self.forward_only = forward_only
        wl_seeded = workloads.Workload(**{**wl.__dict__, "seed": wl.seed + seed_offset})
        self.inp = inp = workloads.layer_inputs(wl_seeded, device, with_grads=not forward_only)
        lds = fq.lds_for(M)
        H = L.hidden
        e = lambda *s, dt=torch.uint8: torch.empty(s, dtype=dt, device=device)  # noqa: E731
        f32 = torch.float32
        bf = torch.bfloat16
        self.lin = {}
        for lin in L.linears:
            N, K = lin.n, lin.k
            d = dict(N=N, K=K, qw=e(N, K), sw=e(N // 128, K // 128, dt=f32),
                     y=e(M, N, dt=bf), q_in=e(M, K), s_in=e(K // 128, lds, dt=f32))
            if not forward_only:
                d.update(qwT=e(K, N), dx=e(M, K, dt=bf), dw=e(N, K, dt=bf),
                         q_inT=e(K, M), s_inT=e(M // 128, K, dt=f32),
                         q_dy=e(M, N), s_dy=e(N // 128, lds, dt=f32),
                         q_dyT=e(N, M), s_dyc=e(M // 128, N, dt=f32))
            self.lin[lin.name] = d
        self.flops = workloads.layer_gemm_flops(L, M, passes=1 if forward_only else 3)
        if saved == "dual":
            self.rstd = {n: e(M, dt=f32) for n in ("qkv", "gate_up")}
        if backward == "fused" and not forward_only:
            # a stack of identical layers in steady state: the gradient arriving from the
            # layer above (dy["down"]) is an input; this layer's RMSNorm1 backward emits
            # the down projection's dY codes of the layer below, which the next step
            # consumes as its own (the first step's come from a6 here)
            self.d_h = e(M, H, dt=bf)
            self.d_x = e(M, H, dt=bf)
            self.dgamma = [e(H, dt=f32), e(H, dt=f32)]
            self.ws = e(fq.rmsnorm_bwd_workspace_bytes(M, H))
            dn = self.lin["down"]
            fq.transpose_quant_bf16(inp["dy"]["down"], dn["q_dy"], dn["s_dy"], dn["q_dyT"],
                                    dn["s_dyc"])
        self.launch_count = None
        if forward_only:
            # serving: the weights are quantized once (at weight sync), not per step
            for name, d in self.lin.items():
                fq.quant_weight_128x128(inp["w"][name], d["qw"], d["sw"], None)

    def _k(self, name, fn, timer):
        if self.only is not None and name not in self.only:
            return
        self._launched += KERNELS_PER_CALL.get(name, 1)
        if timer is not None:
            timer.start(name)
        fn()
        if timer is not None:
            timer.stop(name)

    only = None  # when set: launch only the kernels of these kinds (per-kind graphs)

    def run(self, timer=None, stream=None, only=None):
        self._launched = 0
        self._run(timer, stream, only)
        if only is None:
            self.launch_count = self._launched

    def _run(self, timer, stream, only):
        fq, inp, lin = self.fq, self.inp, self.lin
        self.only = only
        self.timer = timer
        k = self._k
        # weights: 128x128 quantization of the BF16 masters, with the transposed codes
        for name, d in (() if self.forward_only else lin.items()):
            k("quant_weight_128x128",
              lambda d=d, name=name: fq.quant_weight_128x128(inp["w"][name], d["qw"], d["sw"],
                                                             d["qwT"], stream), timer)
        if self.saved == "dual":
            self._forward_dual(k, stream)
        else:
            self._forward_fp8(k, stream)
        if self.forward_only:
            return
        if self.backward == "fused":
            self._backward_fused(k, stream)
        else:
            self._backward_a6(k, stream)

    def _forward_fp8(self, k, stream):
        fq, inp, lin, timer = self.fq, self.inp, self.lin, self.timer
        q, o, gu, dn = lin["qkv"], lin["o"], lin["gate_up"], lin["down"]
        # forward
        k("rmsnorm_quant", lambda: fq.rmsnorm_quant(inp["x_attn"], inp["gamma1"], self.eps,
                                                    q["q_in"], q["s_in"], stream), timer)
        k("gemm_fwd", lambda: fq.linear_fwd(q["q_in"], q["s_in"], q["qw"], q["sw"], q["y"],
                                            stream), timer)
        k("quant_act_1x128", lambda: fq.quant_act_1x128(inp["attn_out"], o["q_in"], o["s_in"],
                                                        stream), timer)
        k("gemm_fwd", lambda: fq.linear_fwd(o["q_in"], o["s_in"], o["qw"], o["sw"], o["y"],
                                            stream), timer)
        k("rmsnorm_quant", lambda: fq.rmsnorm_quant(inp["x_mlp"], inp["gamma2"], self.eps,
                                                    gu["q_in"], gu["s_in"], stream), timer)
        k("gemm_fwd", lambda: fq.linear_fwd(gu["q_in"], gu["s_in"], gu["qw"], gu["sw"], gu["y"],
                                            stream), timer)
        k("swiglu_quant", lambda: fq.swiglu_quant(gu["y"], dn["q_in"], dn["s_in"], stream), timer)
        k("gemm_fwd", lambda: fq.linear_fwd(dn["q_in"], dn["s_in"], dn["qw"], dn["sw"], dn["y"],
                                            stream), timer)

    def _wgrad(self, k, d, stream):
        """WGrad of one linear; with FP8 saved activations their 128x1 codes come from the
        requantizer a8 first."""
        fq = self.fq
        if self.saved == "fp8":
            k("transpose_quant_fp8", lambda: fq.transpose_quant_fp8(d["q_in"], d["s_in"], d["q_inT"],
                                                                    d["s_inT"], stream), self.timer)
        k("gemm_wgrad", lambda: fq.linear_wgrad(d["q_dyT"], d["s_dyc"], d["q_inT"], d["s_inT"],
                                                d["dw"], stream), self.timer)

    def _backward_a6(self, k, stream):
        """Backward of each linear from its BF16 upstream gradient (an input), quantized by
        a6."""
        fq, inp, lin = self.fq, self.inp, self.lin
        for name in ("down", "gate_up", "o", "qkv"):
            d = lin[name]
            k("transpose_quant_bf16",
              lambda d=d, name=name: fq.transpose_quant_bf16(inp["dy"][name], d["q_dy"], d["s_dy"],
                                                             d["q_dyT"], d["s_dyc"], stream),
              self.timer)
            k("gemm_dgrad", lambda d=d: fq.linear_dgrad(d["q_dy"], d["s_dy"], d["qwT"], d["sw"],
                                                        d["dx"], stream), self.timer)
            self._wgrad(k, d, stream)

    def _backward_fused(self, k, stream):
        """Chained backward: each producer's BF16 backward emits the codes of the gradient
        its preceding linear consumes. The QKV gradient comes from attention's backward
        (outside this path): an input, quantized by a6."""
        fq, inp, lin, t, eps = self.fq, self.inp, self.lin, self.timer, self.eps
        q, o, gu, dn = lin["qkv"], lin["o"], lin["gate_up"], lin["down"]
        dgrad = lambda d: k("gemm_dgrad", lambda: fq.linear_dgrad(  # noqa: E731
            d["q_dy"], d["s_dy"], d["qwT"], d["sw"], d["dx"], stream), t)
        dgrad(dn)                                  # dh = dY_down W_down
        self._wgrad(k, dn, stream)
        k("swiglu_bwd_quant_dual", lambda: fq.swiglu_bwd_quant_dual(
            gu["y"], dn["dx"], gu["q_dy"], gu["s_dy"], gu["q_dyT"], gu["s_dyc"], None, stream), t)
        dgrad(gu)                                  # gradient of the RMSNorm2 output
        self._wgrad(k, gu, stream)
        k("rmsnorm_bwd_quant_dual", lambda: fq.rmsnorm_bwd_quant_dual(
            inp["x_mlp"], inp["gamma2"], gu["dx"], inp["dy"]["down"], eps, self.d_h, o["q_dy"],
            o["s_dy"], o["q_dyT"], o["s_dyc"], self.dgamma[1], self.ws, stream), t)
        dgrad(o)                                   # gradient of the attention output
        self._wgrad(k, o, stream)
        k("transpose_quant_bf16", lambda: fq.transpose_quant_bf16(
            inp["dy"]["qkv"], q["q_dy"], q["s_dy"], q["q_dyT"], q["s_dyc"], stream), t)
        dgrad(q)                                   # gradient of the RMSNorm1 output
        self._wgrad(k, q, stream)
        k("rmsnorm_bwd_quant_dual", lambda: fq.rmsnorm_bwd_quant_dual(
            inp["x_attn"], inp["gamma1"], q["dx"], self.d_h, eps, self.d_x, dn["q_dy"], dn["s_dy"],
            dn["q_dyT"], dn["s_dyc"], self.dgamma[0], self.ws, stream), t)

    def _forward_dual(self, k, stream):
        """Option B: every producer emits the 1x128 codes for the forward GEMM and the
        transposed 128x1 codes for WGrad from its BF16 output; no FP8 requantization."""
        fq, inp, lin = self.fq, self.inp, self.lin
        q, o, gu, dn = lin["qkv"], lin["o"], lin["gate_up"], lin["down"]
        k("rmsnorm_quant_dual", lambda: fq.rmsnorm_quant_dual(
            inp["x_attn"], inp["gamma1"], self.eps, q["q_in"], q["s_in"], q["q_inT"], q["s_inT"],
            self.rstd["qkv"], stream), self.timer)
        k("gemm_fwd", lambda: fq.linear_fwd(q["q_in"], q["s_in"], q["qw"], q["sw"], q["y"], stream),
          self.timer)
        k("transpose_quant_bf16_act", lambda: fq.transpose_quant_bf16(
            inp["attn_out"], o["q_in"], o["s_in"], o["q_inT"], o["s_inT"], stream), self.timer)
        k("gemm_fwd", lambda: fq.linear_fwd(o["q_in"], o["s_in"], o["qw"], o["sw"], o["y"], stream),
          self.timer)
        k("rmsnorm_quant_dual", lambda: fq.rmsnorm_quant_dual(
            inp["x_mlp"], inp["gamma2"], self.eps, gu["q_in"], gu["s_in"], gu["q_inT"],
            gu["s_inT"], self.rstd["gate_up"], stream), self.timer)
        k("gemm_fwd", lambda: fq.linear_fwd(gu["q_in"], gu["s_in"], gu["qw"], gu["sw"], gu["y"],
                                            stream), self.timer)
        k("swiglu_quant_dual", lambda: fq.swiglu_quant_dual(
            gu["y"], dn["q_in"], dn["s_in"], dn["q_inT"], dn["s_inT"], stream), self.timer)
        k("gemm_fwd", lambda: fq.linear_fwd(dn["q_in"], dn["s_in"], dn["qw"], dn["sw"], dn["y"],
                                            stream), self.timer)

    def grad_inputs(self):
        """Upstream BF16 gradients that enter a step from outside it."""
        if self.forward_only:
            return ()
        return ("down", "qkv") if self.backward == "fused" else tuple(self.inp["dy"])

    @property
    def launches_per_step(self):
        """Kernels one full step launched (counted during the last full run)."""
        if self.launch_count is None:
            raise RuntimeError("run the step once before asking for its launch count")
        return self.launch_count

    def gemm_flops_by_kind(self):
        M = self.M
        tot = sum(2.0 * M * d["N"] * d["K"] for d in self.lin.values())
        if self.forward_only:
            return {"gemm_fwd": tot}
        return {"gemm_fwd": tot, "gemm_dgrad": tot, "gemm_wgrad": tot}

    def fwd_gemm_bytes(self):
        """Algorithmic HBM bytes of the forward GEMMs of one step: FP8 weight codes and
        128x128 scales, FP8 activation codes and 1x128 scales, BF16 outputs."""
        M = self.M
        return sum(d["N"] * d["K"] * (1 + 4 / 16384) + M * d["K"] * (1 + 4 / 128) +
                   2 * M * d["N"] for d in self.lin.values())

    def quant_bytes_by_kind(self):
        M = self.M
        L = self.L
        H, I = L.hidden, L.intermediate
        qo = L.q_heads * L.head_dim
        w_elems = sum(d["N"] * d["K"] for d in self.lin.values())
        dy_elems = sum(M * d["N"] for d in self.lin.values())
        in_elems = sum(M * d["K"] for d in self.lin.values())
        if self.saved == "dual":
            e = {
                "rmsnorm_quant_dual": 2 * M * H,
                "transpose_quant_bf16_act": M * qo,
                "swiglu_quant_dual": M * I,
            }
        else:
            e = {
                "rmsnorm_quant": 2 * M * H,
                "quant_act_1x128": M * qo,
                "swiglu_quant": M * I,
            }
        if self.forward_only:
            return {k: v * BYTES_PER_ELEM[k] for k, v in e.items()}
        e["quant_weight_128x128"] = w_elems
        if self.saved == "fp8":
            e["transpose_quant_fp8"] = in_elems
        if self.backward == "fused":
            e["transpose_quant_bf16"] = M * self.lin["qkv"]["N"]
            e["swiglu_bwd_quant_dual"] = M * I
            e["rmsnorm_bwd_quant_dual"] = 2 * M * H
        else:
            e["transpose_quant_bf16"] = dy_elems
        return {k: v * BYTES_PER_ELEM[k] for k, v in e.items()}

    # end-to-end: the per-step batch comes from pinned host memory, the results go back
    def e2e_pipeline(self):
        return E2EPipeline(self)


class E2EPipeline:
    """Each step uploads its inputs (activations and, for training, the upstream BF16
    gradients) from pinned host memory and reads its results back (the down projection's
    output and, for training, the QKV input gradient). Two device sets of inputs and of
    results let step i+1's upload and step i-1's read-back run on their own streams
    while step i computes."""

    def __init__(self, step):
        self.step = step
        inp = step.inp
        names = ["x_attn", "x_mlp", "attn_out"]
        self.keys = [(n, None) for n in names] + [("dy", n) for n in step.grad_inputs()]
        get = lambda d, k: d[k[0]] if k[1] is None else d[k[0]][k[1]]  # noqa: E731
        self.get = get
        self.host = {}
        for k in self.keys:
            t = get(inp, k)
            self.host[k] = torch.empty(t.shape, dtype=t.dtype, device="cpu").pin_memory()
            self.host[k].copy_(t)
        self.dev = [{k: get(inp, k) for k in self.keys},
                    {k: torch.empty_like(get(inp, k)) for k in self.keys}]
        self.out_slots = [("down", "y")] + ([] if step.forward_only else [("qkv", "dx")])
        self.outs = [[step.lin[a][b] for a, b in self.out_slots],
                     [torch.empty_like(step.lin[a][b]) for a, b in self.out_slots]]
        self.host_out = [[torch.empty(t.shape, dtype=t.dtype, device="cpu").pin_memory()
                          for t in self.outs[0]] for _ in range(2)]
        self.h2d_bytes = sum(t.numel() * t.element_size() for t in self.host.values())
        self.d2h_bytes = sum(t.numel() * t.element_size() for t in self.outs[0])
        self.up = torch.cuda.Stream()
        self.down = torch.cuda.Stream()
        ev = lambda: [torch.cuda.Event(), torch.cuda.Event()]  # noqa: E731
        self.ev_in, self.ev_done, self.ev_out = ev(), ev(), ev()
        self.i = 0

    def _use(self, s):
        st = self.step
        for k in self.keys:
            if k[1] is None:
                st.inp[k[0]] = self.dev[s][k]
            else:
                st.inp[k[0]][k[1]] = self.dev[s][k]
        for (a, b), t in zip(self.out_slots, self.outs[s]):
            st.lin[a][b] = t

    def run(self):
        s = self.i & 1
        cur = torch.cuda.current_stream()
        first_use = self.i < 2
        with torch.cuda.stream(self.up):
            if not first_use:
                self.up.wait_event(self.ev_done[s])  # set s's inputs were consumed
            for k in self.keys:
                self.dev[s][k].copy_(self.host[k], non_blocking=True)
            self.ev_in[s].record(self.up)
        cur.wait_event(self.ev_in[s])
        if not first_use:
            cur.wait_event(self.ev_out[s])  # set s's results were read back
        self._use(s)
        self.step.run()
        self.ev_done[s].record(cur)
        with torch.cuda.stream(self.down):
            self.down.wait_event(self.ev_done[s])
            for h, t in zip(self.host_out[s], self.outs[s]):
                h.copy_(t, non_blocking=True)
            self.ev_out[s].record(self.down)
        self.i += 1

    def finish(self):
        """Make the current stream wait for the last uploads and read-backs."""
        cur = torch.cuda.current_stream()
        for s in range(2):
            cur.wait_event(self.ev_out[s])

    def restore(self):
        self._use(0)


class KernelTimer:
    """CUDA events around every launch, on the launching (current) stream."""

    def __init__(self):
        self.pending = []
        self.cur = None

    def start(self, name):
        ev = torch.cuda.Event(enable_timing=True)
        ev.record()
        self.cur = (name, ev)

    def stop(self, name):
        ev = torch.cuda.Event(enable_timing=True)
        ev.record()
        self.pending.append((self.cur[0], self.cur[1], ev))
        self.cur = None

    def totals(self):
        out = {}
        for name, a, b in self.pending:
            ms = a.elapsed_time(b)
            t = out.setdefault(name, [0.0, 0])
            t[0] += ms
            t[1] += 1
        return out


def capture_graphs(step, reps_per_kind=10):
    """CUDA graphs of one step and, per kernel kind, of `reps_per_kind` steps' launches of
    that kind only (for device-side per-kernel times without host launch gaps)."""
    graphs = {}
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # one eager pass on the capture stream first
        step.run()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step.run()
    graphs["step"] = g
    counter = KernelTimer()
    step.run(counter)
    torch.cuda.synchronize()
    per_step = {name: n for name, (_, n) in counter.totals().items()}
    graphs["kinds"] = {}
    for name, n in per_step.items():
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(reps_per_kind):
                step.run(only={name})
        step.only = None
        graphs["kinds"][name] = (g, n, reps_per_kind)
    torch.cuda.synchronize()
    return graphs


class GraphKindTimer:
    """Per-kind device time from replays of the per-kind graphs, scaled to `steps` steps
    (same interface as KernelTimer.totals)."""

    def __init__(self, graphs, steps, replays=5):
        self.out = {}
        for name, (g, n_step, reps) in graphs["kinds"].items():
            g.replay()
            torch.cuda.synchronize()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            for _ in range(replays):
                g.replay()
            b.record()
            torch.cuda.synchronize()
            per_launch = a.elapsed_time(b) / (replays * reps * n_step)
            self.out[name] = [per_launch * n_step * steps, n_step * steps]

    def totals(self):
        return self.out


class ClockSampler:
    """Samples SM clock, power and throttle reasons through NVML while running."""

    REASONS = {
        "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80, "sync_boost": 0x10,
    }

    def __init__(self, index, period=0.02):
        self.index, self.period = index, period
        self.samples = []
        self.max_mhz = None
        self._stop = threading.Event()
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # noqa: BLE001
            self.err = repr(e)

    def _loop(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                pw = nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0
                self.samples.append((mhz, reasons, pw))
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._loop, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self.ok:
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [],
                    "samples": 0, "note": getattr(self, "err", "no samples")}
        mhz = [s[0] for s in self.samples]
        seen = 0
        for s in self.samples:
            seen |= s[1]
        reasons = [k for k, bit in self.REASONS.items() if seen & bit]
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples),
                "power_w_max": max(s[2] for s in self.samples)}


# --------------------------------------------------------------------------
# The oracle as the CPU baseline / reference arm (bounded sample of the workload)
# --------------------------------------------------------------------------

def oracle_sample_step(orc, host, wl):
    """One 128-token block of the layer through the oracle: every quantizer on the rows it
    needs, and a 128x128 output tile of each linear's forward, DGrad and WGrad.
    Returns the GEMM flops it computed."""
    import numpy as np
    L = wl.layer
    T = 128
    bits = host["bits"]
    flops = 0.0
    q1, s1 = orc.rmsnorm_quant(bits["x_attn"], bits["gamma1"], wl.eps)
    qa, sa = orc.quant_act_1x128(bits["attn_out"])
    q2, s2 = orc.rmsnorm_quant(bits["x_mlp"], bits["gamma2"], wl.eps)
    qh, sh = orc.swiglu_quant(bits["gu"])
    saved = {"qkv": (q1, s1), "o": (qa, sa), "gate_up": (q2, s2), "down": (qh, sh)}
    for lin in L.linears:
        qin, sin = saved[lin.name]
        # weight blocks for a 128-feature output tile and a 128-feature input tile
        qw_r, sw_r, _ = orc.quant_weight_128x128(bits["w_rows"][lin.name], want_t=False)
        qw_c, sw_c, _ = orc.quant_weight_128x128(bits["w_cols"][lin.name], want_t=False)
        y, _ = orc.linear_fwd(qin, sin, qw_r, sw_r)                       # [T,128] over K
        q_dy, s_dy, q_dyT, s_dyc = orc.transpose_quant_bf16(bits["dy"][lin.name])
        dx, _ = orc.linear_dgrad(q_dy, s_dy, qw_c, sw_c)                  # [T,128] over N
        qinT, sinT = orc.transpose_quant_fp8(qin, sin)
        dw, _ = orc.linear_wgrad(np.ascontiguousarray(q_dyT[:128]), np.ascontiguousarray(s_dyc[:, :128]),
                                 np.ascontiguousarray(qinT[:128]), np.ascontiguousarray(sinT[:, :128]))
        flops += 2.0 * T * 128 * (lin.k + lin.n + T)
    return flops


def oracle_host_inputs(wl):
    import numpy as np
    inp = workloads.layer_inputs(wl, "cpu", tokens=128)
    L = wl.layer

    def b(t):
        return t.contiguous().view(torch.int16).numpy().view(np.uint16)

    I = L.intermediate
    gu = workloads.normal_bf16((128, 2 * I), 1.5, wl.seed, 700, "cpu")
    bits = {"x_attn": b(inp["x_attn"]), "x_mlp": b(inp["x_mlp"]), "attn_out": b(inp["attn_out"]),
            "gamma1": b(inp["gamma1"]), "gamma2": b(inp["gamma2"]), "gu": b(gu),
            "w_rows": {n: b(w[:128]) for n, w in inp["w"].items()},
            "w_cols": {n: np.ascontiguousarray(b(w)[:, :128]) for n, w in inp["w"].items()},
            "dy": {n: b(t) for n, t in inp["dy"].items()}}
    return {"bits": bits}


def oracle_timing(wl=WORKLOAD, min_seconds=10.0, max_steps=1000):
    import oracle as orc
    orc.build()
    host = oracle_host_inputs(wl)
    oracle_sample_step(orc, host, wl)  # warm
    t0 = time.perf_counter()
    flops, steps = 0.0, 0
    while steps < max_steps:
        flops += oracle_sample_step(orc, host, wl)
        steps += 1
        if time.perf_counter() - t0 >= min_seconds:
            break
    dt = time.perf_counter() - t0
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": orc.num_threads(),
            "kind": "oracle",
            "sample": "%d repetitions of one 128-token block of the %s layer: every quantizer "
                      "on the rows it needs, a 128x128 output tile of each linear's forward, "
                      "DGrad and WGrad (fp64 dot products); %.1f s" % (steps, wl.name, dt)}


def oracle_kernel_baselines(wl=WORKLOAD):
    """The oracle, as it stands, per kernel of the step on the host cores: each quantizer
    on a full tensor of the layer (GB/s, with the algorithmic bytes per element of the GPU
    figures), and each GEMM kind on a 256-row slab of the gate/up projection (its
    TFLOP/s, and the full GEMM's time extrapolated from the slab). The inputs have the
    step's shapes and distributions (drawn on the host)."""
    import numpy as np
    import oracle as orc
    orc.build()
    L = wl.layer
    M, H, I = wl.tokens, L.hidden, L.intermediate
    lin = L.linears[2]  # gate/up: N = 2I, K = H, the largest linear
    N, K = lin.n, lin.k

    def b(t):
        return t.contiguous().view(torch.int16).numpy().view(np.uint16)

    kw = dict(outlier_frac=wl.act_outlier_frac, outlier_scale=wl.act_outlier_scale,
              heavy_tail_frac=wl.act_heavy_tail_frac)
    x = b(workloads.activations_bf16((M, H), wl.seed, workloads.TID_X_MLP, "cpu", **kw))
    g = b(workloads.gamma_bf16(H, wl.seed, workloads.TID_GAMMA2, "cpu"))
    out = {}

    def quant(name, elems, fn):
        t0 = time.perf_counter()
        r = fn()
        dt = time.perf_counter() - t0
        out[name] = {"gbs": elems * BYTES_PER_ELEM[name] / dt / 1e9, "seconds": dt,
                     "sample": "full %s tensor" % ("x".join(str(d) for d in shp[name]))}
        return r

    shp = {"quant_act_1x128": (M, H), "rmsnorm_quant": (M, H), "transpose_quant_fp8": (M, H),
           "swiglu_quant": (M, I), "quant_weight_128x128": (N, K), "transpose_quant_bf16": (M, N)}
    qx, sx = quant("quant_act_1x128", M * H, lambda: orc.quant_act_1x128(x))
    quant("rmsnorm_quant", M * H, lambda: orc.rmsnorm_quant(x, g, wl.eps))
    qxT, sxT = quant("transpose_quant_fp8", M * H, lambda: orc.transpose_quant_fp8(qx, sx))
    gu = b(workloads.normal_bf16((M, 2 * I), 1.5, wl.seed, 700, "cpu"))
    quant("swiglu_quant", M * I, lambda: orc.swiglu_quant(gu))
    del gu
    w = b(workloads.normal_bf16((N, K), wl.w_std, wl.seed, workloads.TID_W[lin.name], "cpu"))
    qw, sw, _ = quant("quant_weight_128x128", N * K, lambda: orc.quant_weight_128x128(w))
    del w
    dy = b(workloads.gradients_bf16((M, N), wl.dy_std, wl.seed, workloads.TID_DY[lin.name], "cpu",
                                    small_row_frac=wl.dy_small_row_frac,
                                    small_row_scale=wl.dy_small_row_scale))
    qdy, sdy, qdyT, sdyc = quant("transpose_quant_bf16", M * N, lambda: orc.transpose_quant_bf16(dy))
    del dy
    slab = 256
    for name, fn, full_rows in (
            ("gemm_fwd", lambda: orc.linear_fwd(qx, sx, qw, sw, rows=(0, slab)), M),
            ("gemm_dgrad", lambda: orc.linear_dgrad(qdy, sdy, qw, sw, rows=(0, slab)), M),
            ("gemm_wgrad", lambda: orc.linear_wgrad(qdyT, sdyc, qxT, sxT, rows=(0, slab)), N)):
        inner = {"gemm_fwd": K, "gemm_dgrad": N, "gemm_wgrad": M}[name]
        cols = {"gemm_fwd": N, "gemm_dgrad": K, "gemm_wgrad": K}[name]
        t0 = time.perf_counter()
        fn()
        dt = time.perf_counter() - t0
        flops = 2.0 * slab * cols * inner
        out[name] = {"tflops": flops / dt / 1e12, "seconds": dt,
                     "full_gemm_seconds_extrapolated": dt * full_rows / slab,
                     "sample": "%d of the %d output rows of the gate/up %s (%dx%dx%d), fp64 "
                               "dot products; full-GEMM time extrapolated from the slab" % (
                                   slab, full_rows, name[5:], full_rows, cols, inner)}
    return out


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    import oracle as orc
    orc.build()
    host = oracle_host_inputs(WORKLOAD)
    for _ in range(args.warmup):
        oracle_sample_step(orc, host, WORKLOAD)
    t0 = time.perf_counter()
    flops = 0.0
    for _ in range(args.steps):
        flops += oracle_sample_step(orc, host, WORKLOAD)
    dt = time.perf_counter() - t0
    value = flops / dt / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD.name, "tokens_per_step": 128,
                   "note": "the oracle (plain CPU definition) on a bounded sample per step"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": orc.num_threads(),
                         "kind": "oracle",
                         "sample": "one 128-token block per step: every quantizer on its rows, "
                                   "a 128x128 output tile of each GEMM"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------
# Single-kernel cases (for profilers): one kernel of the layer on its real shape,
# with only the buffers it needs on the device.
# --------------------------------------------------------------------------

CASES = ("gemm_fwd", "gemm_dgrad", "gemm_wgrad", "gemm_wgrad_acc", "quantizers", "gemm_decode",
         "producers")


def run_case(name, reps):
    import fp8_block_scaled_08_b200 as fq
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    wl = WORKLOAD
    M = wl.tokens
    lin = wl.layer.linears[2]  # gate/up: N = 28672, K = 4096 (the largest linear)
    N, K = lin.n, lin.k
    w = workloads.normal_bf16((N, K), wl.w_std, wl.seed, workloads.TID_W[lin.name], dev)
    if name == "gemm_fwd":
        x = workloads.activations_bf16((M, K), wl.seed, workloads.TID_X_MLP, dev,
                                       outlier_frac=wl.act_outlier_frac,
                                       outlier_scale=wl.act_outlier_scale)
        qx, sx = fq.quant_act_1x128_alloc(x)
        qw, sw, _ = fq.quant_weight_alloc(w, want_t=False)
        y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        fn = lambda: fq.linear_fwd(qx, sx, qw, sw, y)  # noqa: E731
    elif name == "gemm_dgrad":
        dy = workloads.gradients_bf16((M, N), wl.dy_std, wl.seed, workloads.TID_DY[lin.name], dev)
        qdy, sdy = fq.quant_act_1x128_alloc(dy)
        _, sw, qwT = fq.quant_weight_alloc(w)
        dx = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
        fn = lambda: fq.linear_dgrad(qdy, sdy, qwT, sw, dx)  # noqa: E731
    elif name in ("gemm_wgrad", "gemm_wgrad_acc"):
        x = workloads.activations_bf16((M, K), wl.seed, workloads.TID_X_MLP, dev)
        dy = workloads.gradients_bf16((M, N), wl.dy_std, wl.seed, workloads.TID_DY[lin.name], dev)
        qx, sx = fq.quant_act_1x128_alloc(x)
        qxT, sxT = fq.transpose_quant_fp8_alloc(qx, sx)
        _, _, qdyT, sdyc = fq.transpose_quant_bf16_alloc(dy, want_row=False)
        if name == "gemm_wgrad":
            dw = torch.empty((N, K), dtype=torch.bfloat16, device=dev)
            fn = lambda: fq.linear_wgrad(qdyT, sdyc, qxT, sxT, dw)  # noqa: E731
        else:  # fp32 dW accumulated into (read and written once per launch)
            dw = torch.zeros((N, K), dtype=torch.float32, device=dev)
            fn = lambda: fq.linear_wgrad_acc_f32(qdyT, sdyc, qxT, sxT, dw)  # noqa: E731
    elif name == "gemm_decode":
        # Qwen3-8B gate/up projection at a 16-token decode batch (skinny-M kernel)
        dwl = workloads.QWEN3_DECODE[0]
        dlin = dwl.layer.linears[2]
        Nd, Kd = dlin.n, dlin.k
        wd = workloads.normal_bf16((Nd, Kd), dwl.w_std, dwl.seed, workloads.TID_W[dlin.name], dev)
        xd = workloads.activations_bf16((dwl.tokens, Kd), dwl.seed, workloads.TID_X_MLP, dev)
        qx, sx = fq.quant_act_1x128_alloc(xd)
        qw, sw, _ = fq.quant_weight_alloc(wd, want_t=False)
        y = torch.empty((dwl.tokens, Nd), dtype=torch.bfloat16, device=dev)
        fn = lambda: fq.linear_fwd(qx, sx, qw, sw, y)  # noqa: E731
    elif name == "quantizers":
        x = workloads.activations_bf16((M, K), wl.seed, workloads.TID_X_MLP, dev)
        g = workloads.gamma_bf16(K, wl.seed, workloads.TID_GAMMA2, dev)
        dy = workloads.gradients_bf16((M, N), wl.dy_std, wl.seed, workloads.TID_DY[lin.name], dev)
        q, s = fq.quant_act_1x128_alloc(x)

        def fn():
            fq.quant_act_1x128_alloc(x)
            fq.rmsnorm_quant_alloc(x, g, wl.eps)
            fq.swiglu_quant_alloc(dy)
            fq.quant_weight_alloc(w)
            fq.transpose_quant_bf16_alloc(dy)
            fq.transpose_quant_fp8_alloc(q, s)
    elif name == "producers":
        # the kernels that quantize a value formed on the fly, at sizes above L2 but a
        # few hundred MB each: a6 on a 4096 x 28672 gradient, the option-B producers and
        # the backward producers (SwiGLU at 2048 x 14336, RMSNorm at 8192 x 4096)
        I = wl.layer.intermediate
        Ms = 2048
        dy = workloads.gradients_bf16((4096, N), wl.dy_std, wl.seed, workloads.TID_DY[lin.name],
                                      dev)
        gu = workloads.normal_bf16((Ms, 2 * I), 1.5, wl.seed, 700, dev)
        dh = workloads.gradients_bf16((Ms, I), wl.dy_std, wl.seed, 701, dev)
        x = workloads.activations_bf16((M, K), wl.seed, workloads.TID_X_MLP, dev)
        g = workloads.gamma_bf16(K, wl.seed, workloads.TID_GAMMA2, dev)
        dyk = workloads.gradients_bf16((M, K), wl.dy_std, wl.seed, 702, dev)
        dres = workloads.gradients_bf16((M, K), wl.dy_std, wl.seed, 703, dev)

        def fn():
            fq.transpose_quant_bf16_alloc(dy)
            fq.swiglu_quant_dual_alloc(gu)
            fq.rmsnorm_quant_dual_alloc(x, g, wl.eps)
            fq.swiglu_bwd_quant_dual_alloc(gu, dh)
            fq.rmsnorm_bwd_quant_dual_alloc(x, g, dyk, dres, wl.eps)
    else:
        raise SystemExit("unknown case %r (choose from %s)" % (name, ", ".join(CASES)))
    torch.cuda.synchronize()
    for _ in range(reps):
        fn()
    torch.cuda.synchronize()
    if fq.device_error() != fq.FP8Q_OK:
        raise RuntimeError("device error in case %s" % name)
    print("case %s: %d repetitions OK" % (name, reps))
    return 0


# --------------------------------------------------------------------------
# Our arm
# --------------------------------------------------------------------------

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--case", choices=CASES, default=None,
                    help="run one kernel of the layer on its real shape (for profilers)")
    ap.add_argument("--case-reps", type=int, default=3)
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default=WORKLOAD.name,
                    help="layer shape (default: the Llama-3.1-8B layer at M = 8192)")
    ap.add_argument("--backward", choices=("a6", "fused"), default="a6",
                    help="a6 = every linear's BF16 upstream gradient is an input quantized by "
                         "a6; fused = the SwiGLU / RMSNorm backward producers emit the codes "
                         "(chained, steady-state stack of identical layers)")
    ap.add_argument("--saved", choices=("fp8", "dual"), default="fp8",
                    help="saved activations for WGrad: fp8 = requantize the saved FP8 tensor "
                         "(the pages' flow, default); dual = producers emit both groupings")
    args = ap.parse_args()
    wl = WORKLOADS[args.workload]
    if args.case:
        return run_case(args.case, args.case_reps)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        return run_reference(args, rank, world)

    import fp8_block_scaled_08_b200 as fq
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
        pg = dist

    step = LayerStep(fq, wl, dev, seed_offset=rank_seed_offset(rank), forward_only=is_decode(wl),
                     saved=args.saved, backward=args.backward)
    torch.cuda.synchronize()
    for _ in range(args.warmup):
        step.run()
    torch.cuda.synchronize()
    if fq.device_error() != fq.FP8Q_OK:
        raise RuntimeError("a kernel reported a device error during warm-up")

    # ---- timed region: K steps, per-kernel events on the launching stream. Decode-sized
    # steps launch kernels faster than the host can issue them one by one, so they are
    # captured once into a CUDA graph (the same launches) and the graph is replayed.
    timer = KernelTimer()
    sampler = ClockSampler(local_rank)
    graphs = None
    if step.forward_only:
        graphs = capture_graphs(step)
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    with sampler:
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record()
        for _ in range(args.steps):
            if graphs:
                graphs["step"].replay()
            else:
                step.run(timer)
        end.record()
        torch.cuda.synchronize()
    if pg:
        pg.barrier()
    elapsed_ms = start.elapsed_time(end)
    if graphs:
        timer = GraphKindTimer(graphs, args.steps)
    if fq.device_error() != fq.FP8Q_OK:
        raise RuntimeError("a kernel reported a device error in the timed region")
    max_ms = max_over_ranks(elapsed_ms, pg, dev)
    ms_per_step = max_ms / args.steps
    value = whole_job_tflops(step.flops, world, ms_per_step)

    # ---- per-kernel breakdown (same timed steps)
    peaks = read_peaks()
    # Dense FP8 = 2x the measured BF16 GEMM rate (the nominal fp8/bf16 ratio). The timed
    # region is a fraction of a second at full clock, so the burst figure is the peak;
    # the sustained one (seconds under the power cap, lower clock) is reported beside it.
    fp8_peak = 2.0 * peaks["bf16_tflops"]
    fp8_peak_sustained = 2.0 * peaks["bf16_tflops_sustained"]
    clocks = sampler.summary()
    kt = timer.totals()
    roofline = None
    gflops = step.gemm_flops_by_kind()
    gemm_ms = sum(kt[k][0] for k in gflops)
    gemm_launches = sum(kt[k][1] for k in gflops)
    gemm_flops = sum(gflops.values()) * args.steps
    achieved = gemm_flops / (gemm_ms * 1e-3) / 1e12
    if step.forward_only:
        # below the ridge: the forward GEMMs are bound by reading the FP8 weights
        gemm_gbs = step.fwd_gemm_bytes() * args.steps / (gemm_ms * 1e-3) / 1e9
        roofline = {"bound": "hbm", "achieved": gemm_gbs, "peak": peaks["hbm_gbs"],
                    "unit": "GB/s", "frac": gemm_gbs / peaks["hbm_gbs"], "traffic": None,
                    "kernel": "gemm_fwd (decode, weight-bytes bound)",
                    "launches": gemm_launches // args.steps,
                    "bytes_per_step": step.fwd_gemm_bytes(),
                    "peak_source": "%s HBM copy bandwidth" % peaks["source"]}
    traffic = None
    prof = os.path.join(ROOT, "profiles", "gemm_traffic.json")
    if os.path.exists(prof):
        with open(prof) as f:
            traffic = json.load(f).get("bytes_per_launch")
    if roofline is None:
        roofline = {"bound": "tensor", "achieved": achieved, "peak": fp8_peak,
                    "unit": "TFLOP/s", "frac": achieved / fp8_peak, "traffic": traffic,
                    "kernel": "gemm (fwd+dgrad+wgrad launches)",
                    "launches": gemm_launches // args.steps,
                    "peak_source": "%s bf16 burst x2 (fp8/bf16 nominal ratio)" % peaks["source"],
                    "peak_sustained": fp8_peak_sustained,
                    "frac_of_sustained": achieved / fp8_peak_sustained,
                    "frac_of_nominal_fp8": achieved / NOMINAL_FP8_TFLOPS,
                    "sm_mhz_median": clocks.get("sm_mhz"),
                    "tflops_per_ghz": (achieved / (clocks["sm_mhz"] / 1000.0)
                                       if clocks.get("sm_mhz") else None)}
    kernels = {}
    for kname, fl in gflops.items():
        ms, n = kt[kname]
        if n == 0:
            continue
        kernels[kname] = {"ms_per_step": ms / args.steps, "launches_per_step": n // args.steps,
                          "tflops": fl * args.steps / (ms * 1e-3) / 1e12,
                          "frac_of_fp8_peak": fl * args.steps / (ms * 1e-3) / 1e12 / fp8_peak}
    qb = step.quant_bytes_by_kind()
    for kname, by in qb.items():
        ms, n = kt[kname]
        gbs = by * args.steps / (ms * 1e-3) / 1e9
        kernels[kname] = {"ms_per_step": ms / args.steps, "launches_per_step": n // args.steps,
                          "gbs": gbs, "frac_of_hbm": gbs / peaks["hbm_gbs"]}

    # ---- end to end through the C ABI with host buffers (uploads and read-backs inside
    # the timed region, overlapped with compute on their own streams)
    pipe = step.e2e_pipeline()
    for _ in range(2):
        pipe.run()
    pipe.finish()
    torch.cuda.synchronize()
    if pg:
        pg.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.e2e_steps):
        pipe.run()
    pipe.finish()
    e1.record()
    torch.cuda.synchronize()
    pipe.restore()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), pg, dev) / args.e2e_steps
    e2e_value = whole_job_tflops(step.flops, world, e2e_ms)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not step.forward_only:
        cpu = oracle_timing(wl, min_seconds=6.0)
        cpu["kernels"] = oracle_kernel_baselines(wl)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "fp8_e4m3", "data": "synthetic",
            "config": {"workload": wl.name, "tokens_per_gpu": wl.tokens,
                       "hidden": wl.layer.hidden,
                       "intermediate": wl.layer.intermediate,
                       "pass": "forward (serving)" if step.forward_only else "forward+backward",
                       "saved_activations": ("n/a" if step.forward_only else
                                             {"fp8": "FP8, requantized 128x1 for WGrad",
                                              "dual": "both groupings from BF16 (option B)"}[args.saved]),
                       "backward": ("n/a" if step.forward_only else
                                    {"a6": "each linear's BF16 gradient quantized by a6",
                                     "fused": "SwiGLU / RMSNorm backward producers emit the "
                                              "gradient codes (chained)"}[args.backward]),
                       "gemm_tflop_per_step_per_gpu": step.flops / 1e12,
                       "launches_per_step": step.launches_per_step,
                       "l2": "inputs larger than L2: %.1f GB touched per step" % (
                           sum(qb.values()) / 1e9),
                       "parallelism": "replicas" if world > 1 else "single"},
            "roofline": roofline,
            "kernels": kernels,
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": pipe.h2d_bytes,
                    "d2h_bytes_per_step": pipe.d2h_bytes, "ms_per_step": e2e_ms,
                    "overlap": "uploads and read-backs on their own streams, double-buffered"},
            "gpu_launches": step.launches_per_step * args.steps,
            "clocks": clocks,
        }
        print(json.dumps(line), flush=True)
    if pg:
        pg.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
