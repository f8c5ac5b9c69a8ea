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

# Algorithmic bytes per element of each quantizer (reads + writes, scales included).
BYTES_PER_ELEM = {
    "quant_act_1x128": 2 + 1 + 4 / 128,          # per input element
    "rmsnorm_quant": 2 + 1 + 4 / 128,            # per element (gamma negligible)
    "swiglu_quant": 4 + 1 + 4 / 128,             # per output element
    "quant_weight_128x128": 2 + 1 + 1 + 4 / 16384,  # with the transposed copy
    "transpose_quant_bf16": 2 + 2 * (1 + 4 / 128),
    "transpose_quant_fp8": (1 + 4 / 128) * 2,
}


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

    def __init__(self, fq, wl, device, seed_offset=0):
        self.fq = fq
        L = wl.layer
        self.M = M = wl.tokens
        self.L = L
        self.eps = wl.eps
        wl_seeded = workloads.Workload(**{**wl.__dict__, "seed": wl.seed + seed_offset})
        self.inp = inp = workloads.layer_inputs(wl_seeded, device)
        lds = fq.lds_for(M)
        H, I = L.hidden, L.intermediate
        e = lambda *s, dt=torch.uint8: torch.empty(s, dtype=dt, device=device)  # noqa: E731
        f32 = torch.float32
        bf = torch.bfloat16
        self.lin = {}
        for lin in L.linears:
            N, K = lin.n, lin.k
            self.lin[lin.name] = dict(
                N=N, K=K,
                qw=e(N, K), sw=e(N // 128, K // 128, dt=f32), qwT=e(K, N),
                y=e(M, N, dt=bf), dx=e(M, K, dt=bf), dw=e(N, K, dt=bf),
                q_in=e(M, K), s_in=e(K // 128, lds, dt=f32),
                q_inT=e(K, M), s_inT=e(M // 128, K, dt=f32),
                q_dy=e(M, N), s_dy=e(N // 128, lds, dt=f32),
                q_dyT=e(N, M), s_dyc=e(M // 128, N, dt=f32),
            )
        self.flops = workloads.layer_gemm_flops(L, M)
        self.kernel_names = []

    def _k(self, name, fn, timer):
        if timer is not None:
            timer.start(name)
        fn()
        if timer is not None:
            timer.stop(name)

    def run(self, timer=None, stream=None):
        fq, inp, lin, M = self.fq, self.inp, self.lin, self.M
        k = self._k
        # weights: 128x128 quantization of the BF16 masters, with the transposed codes
        for name, d in lin.items():
            k("quant_weight_128x128",
              lambda d=d, name=name: fq.quant_weight_128x128(inp["w"][name], d["qw"], d["sw"],
                                                             d["qwT"], stream), timer)
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
        # backward of each linear (BF16 upstream gradients)
        for name in ("down", "gate_up", "o", "qkv"):
            d = lin[name]
            k("transpose_quant_bf16",
              lambda d=d, name=name: fq.transpose_quant_bf16(inp["dy"][name], d["q_dy"], d["s_dy"],
                                                             d["q_dyT"], d["s_dyc"], stream), timer)
            k("gemm_dgrad", lambda d=d: fq.linear_dgrad(d["q_dy"], d["s_dy"], d["qwT"], d["sw"],
                                                        d["dx"], stream), timer)
            k("transpose_quant_fp8", lambda d=d: fq.transpose_quant_fp8(d["q_in"], d["s_in"],
                                                                        d["q_inT"], d["s_inT"],
                                                                        stream), timer)
            k("gemm_wgrad", lambda d=d: fq.linear_wgrad(d["q_dyT"], d["s_dyc"], d["q_inT"],
                                                        d["s_inT"], d["dw"], stream), timer)

    launches_per_step = 28

    def gemm_flops_by_kind(self):
        M = self.M
        tot = sum(2.0 * M * d["N"] * d["K"] for d in self.lin.values())
        return {"gemm_fwd": tot, "gemm_dgrad": tot, "gemm_wgrad": tot}

    def quant_bytes_by_kind(self):
        M = self.M
        L = self.L
        H, I = L.hidden, L.intermediate
        qo = L.q_heads * L.head_dim
        w_elems = sum(d["N"] * d["K"] for d in self.lin.values())
        dy_elems = sum(M * d["N"] for d in self.lin.values())
        in_elems = sum(M * d["K"] for d in self.lin.values())
        e = {
            "quant_weight_128x128": w_elems,
            "rmsnorm_quant": 2 * M * H,
            "quant_act_1x128": M * qo,
            "swiglu_quant": M * I,
            "transpose_quant_bf16": dy_elems,
            "transpose_quant_fp8": in_elems,
        }
        return {k: v * BYTES_PER_ELEM[k] for k, v in e.items()}

    # end-to-end: the per-step batch comes from pinned host memory, the results go back
    def e2e_buffers(self):
        inp = self.inp
        names = ["x_attn", "x_mlp", "attn_out"]
        host_in = {n: torch.empty_like(inp[n], device="cpu").pin_memory() for n in names}
        for n in names:
            host_in[n].copy_(inp[n])
        host_dy = {n: torch.empty_like(t, device="cpu").pin_memory() for n, t in inp["dy"].items()}
        for n, t in inp["dy"].items():
            host_dy[n].copy_(t)
        outs = [self.lin["down"]["y"], self.lin["qkv"]["dx"]]
        host_out = [torch.empty_like(t, device="cpu").pin_memory() for t in outs]
        h2d = sum(t.numel() * t.element_size() for t in host_in.values()) + \
            sum(t.numel() * t.element_size() for t in host_dy.values())
        d2h = sum(t.numel() * t.element_size() for t in host_out)
        return host_in, host_dy, outs, host_out, h2d, d2h

    def run_e2e(self, bufs, stream=None):
        host_in, host_dy, outs, host_out, _, _ = bufs
        for n, h in host_in.items():
            self.inp[n].copy_(h, non_blocking=True)
        for n, h in host_dy.items():
            self.inp["dy"][n].copy_(h, non_blocking=True)
        self.run(stream=stream)
        for h, t in zip(host_out, outs):
            h.copy_(t, non_blocking=True)


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


def oracle_timing(min_seconds=10.0, max_steps=1000):
    import oracle as orc
    orc.build()
    host = oracle_host_inputs(WORKLOAD)
    oracle_sample_step(orc, host, WORKLOAD)  # warm
    t0 = time.perf_counter()
    flops, steps = 0.0, 0
    while steps < max_steps:
        flops += oracle_sample_step(orc, host, WORKLOAD)
        steps += 1
        if time.perf_counter() - t0 >= min_seconds:
            break
    dt = time.perf_counter() - t0
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": orc.num_threads(),
            "kind": "oracle",
            "sample": "%d repetitions of one 128-token block of the %s layer: every quantizer "
                      "on the rows it needs, a 128x128 output tile of each linear's forward, "
                      "DGrad and WGrad (fp64 dot products); %.1f s" % (steps, WORKLOAD.name, dt)}


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

CASES = ("gemm_fwd", "gemm_dgrad", "gemm_wgrad", "quantizers")


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
    elif name == "gemm_wgrad":
        x = workloads.activations_bf16((M, K), wl.seed, workloads.TID_X_MLP, dev)
        dy = workloads.gradients_bf16((M, N), wl.dy_std, wl.seed, workloads.TID_DY[lin.name], dev)
        qx, sx = fq.quant_act_1x128_alloc(x)
        qxT, sxT = fq.transpose_quant_fp8_alloc(qx, sx)
        _, _, qdyT, sdyc = fq.transpose_quant_bf16_alloc(dy, want_row=False)
        dw = torch.empty((N, K), dtype=torch.bfloat16, device=dev)
        fn = lambda: fq.linear_wgrad(qdyT, sdyc, qxT, sxT, dw)  # noqa: E731
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
    args = ap.parse_args()
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

    step = LayerStep(fq, WORKLOAD, dev, seed_offset=rank_seed_offset(rank))
    torch.cuda.synchronize()
    for _ in range(args.warmup):
        step.run()
    torch.cuda.synchronize()
    if fq.device_error() != fq.FP8Q_OK:
        raise RuntimeError("a kernel reported a device error during warm-up")

    # ---- timed region: K steps, per-kernel events on the launching stream
    timer = KernelTimer()
    sampler = ClockSampler(local_rank)
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    with sampler:
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record()
        for _ in range(args.steps):
            step.run(timer)
        end.record()
        torch.cuda.synchronize()
    if pg:
        pg.barrier()
    elapsed_ms = start.elapsed_time(end)
    if fq.device_error() != fq.FP8Q_OK:
        raise RuntimeError("a kernel reported a device error in the timed region")
    max_ms = max_over_ranks(elapsed_ms, pg, dev)
    ms_per_step = max_ms / args.steps
    value = whole_job_tflops(step.flops, world, ms_per_step)

    # ---- per-kernel breakdown (same timed steps)
    peaks = read_peaks()
    fp8_peak = 2.0 * peaks["bf16_tflops_sustained"]  # fp8 dense = 2x bf16 (nominal ratio)
    kt = timer.totals()
    gflops = step.gemm_flops_by_kind()
    gemm_ms = sum(kt[k][0] for k in gflops)
    gemm_launches = sum(kt[k][1] for k in gflops)
    gemm_flops = sum(gflops.values()) * args.steps
    achieved = gemm_flops / (gemm_ms * 1e-3) / 1e12
    traffic = None
    prof = os.path.join(ROOT, "profiles", "gemm_traffic.json")
    if os.path.exists(prof):
        with open(prof) as f:
            traffic = json.load(f).get("bytes_per_launch")
    kernels = {}
    for kname, fl in gflops.items():
        ms, n = kt[kname]
        kernels[kname] = {"ms_per_step": ms / args.steps, "launches_per_step": n // args.steps,
                          "tflops": fl * args.steps / (ms * 1e-3) / 1e12,
                          "frac_of_fp8_peak": fl * args.steps / (ms * 1e-3) / 1e12 / fp8_peak}
    qb = step.quant_bytes_by_kind()
    for kname, by in qb.items():
        ms, n = kt[kname]
        gbs = by * args.steps / (ms * 1e-3) / 1e9
        kernels[kname] = {"ms_per_step": ms / args.steps, "launches_per_step": n // args.steps,
                          "gbs": gbs, "frac_of_hbm": gbs / peaks["hbm_gbs"]}

    # ---- end to end through the C ABI with host buffers
    bufs = step.e2e_buffers()
    for _ in range(2):
        step.run_e2e(bufs)
    torch.cuda.synchronize()
    if pg:
        pg.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.e2e_steps):
        step.run_e2e(bufs)
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), pg, dev) / args.e2e_steps
    e2e_value = whole_job_tflops(step.flops, world, e2e_ms)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_timing()

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "fp8_e4m3", "data": "synthetic",
            "config": {"workload": WORKLOAD.name, "tokens_per_gpu": WORKLOAD.tokens,
                       "hidden": WORKLOAD.layer.hidden,
                       "intermediate": WORKLOAD.layer.intermediate,
                       "gemm_tflop_per_step_per_gpu": step.flops / 1e12,
                       "launches_per_step": LayerStep.launches_per_step,
                       "l2": "inputs larger than L2: %.1f GB touched per step" % (
                           sum(qb.values()) / 1e9),
                       "parallelism": "replicas" if world > 1 else "single"},
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": fp8_peak,
                         "unit": "TFLOP/s", "frac": achieved / fp8_peak, "traffic": traffic,
                         "kernel": "gemm (fwd+dgrad+wgrad launches)",
                         "launches": gemm_launches // args.steps,
                         "peak_source": "%s bf16 sustained x2 (fp8/bf16 nominal ratio)" % peaks["source"]},
            "kernels": kernels,
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": bufs[4],
                    "d2h_bytes_per_step": bufs[5], "ms_per_step": e2e_ms},
            "gpu_launches": LayerStep.launches_per_step * args.steps,
            "clocks": sampler.summary(),
        }
        print(json.dumps(line), flush=True)
    if pg:
        pg.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
