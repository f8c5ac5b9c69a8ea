"""Host logic of bench.py without a GPU: the multi-rank (weak scaling) aggregation on
two gloo ranks, the per-rank input streams, and the roofline arithmetic."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import workloads


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        per_rank_ms = [12.5, 17.0][rank]          # rank 1 is the slow one
        mx = bench.max_over_ranks(per_rank_ms, dist)
        val = bench.whole_job_tflops(1e12, world, mx)
        # each rank draws its own batch: the first values differ between ranks
        x = workloads.activations_bf16((4, 256), bench.rank_seed_offset(rank), 1, "cpu")
        out[rank] = (mx, val, float(x[0, 0]))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_and_weak_scaling():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, join=True,
                       start_method="spawn")
    (m0, v0, x0), (m1, v1, x1) = out[0], out[1]
    assert m0 == m1 == 17.0                       # the max over ranks, on every rank
    assert v0 == v1 == pytest.approx(2 * 1e12 / 17e-3 / 1e12)
    assert x0 != x1                               # independent token batches


def test_flop_and_byte_accounting():
    L = workloads.LLAMA31_8B
    assert workloads.layer_gemm_flops(L, 8192) == pytest.approx(10.72e12, rel=1e-3)
    assert bench.BYTES_PER_ELEM["quant_act_1x128"] == pytest.approx(3.03125)
    assert bench.BYTES_PER_ELEM["transpose_quant_bf16"] == pytest.approx(4.0625)
    assert bench.whole_job_tflops(2e12, 4, 8.0) == pytest.approx(1000.0)


def test_peaks_reader():
    p = bench.read_peaks()
    assert p["hbm_gbs"] > 1000 and p["bf16_tflops"] > 100
    assert p["source"] in ("measured", "fallback")


class _StubBinding:
    """Records the binding calls a layer step makes (no device, no kernels)."""

    def __init__(self):
        self.calls = []

    def lds_for(self, m):
        return (m + 3) // 4 * 4

    def rmsnorm_bwd_workspace_bytes(self, M, H):
        return 16

    def __getattr__(self, name):
        def record(*args, **kwargs):
            self.calls.append(name)
        return record


@pytest.mark.parametrize("saved,backward,launches,grads", [
    ("fp8", "a6", 28, {"qkv", "o", "gate_up", "down"}),
    ("dual", "a6", 26, {"qkv", "o", "gate_up", "down"}),
    ("fp8", "fused", 32, {"down", "qkv"}),
    ("dual", "fused", 30, {"down", "qkv"})])
def test_layer_step_modes_on_a_stub(saved, backward, launches, grads):
    """The four step variants: kernel launches per step, which upstream gradients enter
    from outside, and a byte count for every quantizer kind the step times."""
    import dataclasses
    fq = _StubBinding()
    wl = dataclasses.replace(workloads.LLAMA_LAYER, tokens=256)
    step = bench.LayerStep(fq, wl, "cpu", saved=saved, backward=backward)
    fq.calls.clear()
    step.run()
    assert step.launches_per_step == launches
    assert set(step.grad_inputs()) == grads
    kinds = set(step.quant_bytes_by_kind())
    called = set(fq.calls) - {"linear_fwd", "linear_dgrad", "linear_wgrad"}
    # every quantizer entry point the step calls has its bytes accounted for (the
    # option-B attention-output quantizer is a6 under its own timing name)
    assert called - {"transpose_quant_bf16"} <= kinds
    assert ("transpose_quant_fp8" in kinds) == (saved == "fp8")
    assert ("swiglu_bwd_quant_dual" in kinds) == (backward == "fused")
    assert fq.calls.count("linear_fwd") == 4 and fq.calls.count("linear_wgrad") == 4
    assert fq.calls.count("linear_dgrad") == 4


def test_reference_arm_prints_its_line():
    """`bench.py --impl reference` (the oracle on the host cores, a bounded sample per
    step) prints one JSON line with the contract's keys; it needs no GPU."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], cwd=root, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC
    assert line["value"] > 0 and line["unit"] == "TFLOP/s" and line["higher_is_better"]
    assert line["steps"] == 1 and line["warmup"] == 3
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"]
    assert cb["value"] == line["value"]
    e2e = line["e2e"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
