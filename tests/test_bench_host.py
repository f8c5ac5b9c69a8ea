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
