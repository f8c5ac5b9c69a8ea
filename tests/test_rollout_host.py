"""Host logic of the per-step rollout weight refresh without a GPU:
the packed layout, and the distribution on two gloo ranks — rank 0 fills the buffer with
the oracle's 128x128 quantization of seeded BF16 masters (standing in for the library's
quantizer, which needs a GPU), one broadcast, and rank 1 holds exactly those codes and
scales in its views."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import workloads

SHAPES = {"qkv": (768, 512), "o": (512, 512), "gate_up": (1024, 384), "down": (384, 640)}


def _masters():
    return {n: workloads.normal_bf16(s, 0.02, 0, 900 + i, "cpu")
            for i, (n, s) in enumerate(SHAPES.items())}


def _bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _oracle_quantize(packed, masters):
    import oracle
    views = packed.views()
    for name, w in masters.items():
        q, s, _ = oracle.quant_weight_128x128(_bits(w), want_t=False)
        views[name][0].copy_(torch.from_numpy(q))
        views[name][1].copy_(torch.from_numpy(s))


def test_packed_layout():
    from fp8_block_scaled_08_b200.rollout import PackedFp8Weights
    p = PackedFp8Weights(SHAPES, "cpu")
    off = 0
    for name, (n, k) in SHAPES.items():
        _, _, q_off, s_off = p.layout[name]
        assert q_off % 16 == 0 and s_off % 16 == 0 and q_off >= off
        assert s_off >= q_off + n * k
        off = s_off + 4 * (n // 128) * (k // 128)
        qw, sw = p.views()[name]
        assert qw.shape == (n, k) and qw.dtype == torch.uint8 and qw.is_contiguous()
        assert sw.shape == (n // 128, k // 128) and sw.dtype == torch.float32
        assert sw.is_contiguous()
    assert p.nbytes >= off and p.nbytes % 16 == 0
    with pytest.raises(ValueError):
        PackedFp8Weights({"bad": (100, 128)}, "cpu")


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
        from fp8_block_scaled_08_b200.rollout import PackedFp8Weights, refresh
        packed = PackedFp8Weights(SHAPES, "cpu")
        packed.buffer.fill_(0xA5)
        refresh(packed, _masters() if rank == 0 else None, src=0, quantize=_oracle_quantize)
        out[rank] = packed.buffer.numpy().tobytes()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_receive_the_trainers_codes():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, join=True,
                       start_method="spawn")
    assert out[0] == out[1]
    # and the received bytes are the oracle's quantization of the masters
    from fp8_block_scaled_08_b200.rollout import PackedFp8Weights
    ref = PackedFp8Weights(SHAPES, "cpu")
    ref.buffer.fill_(0xA5)
    _oracle_quantize(ref, _masters())
    got = np.frombuffer(out[1], np.uint8)
    views = ref.views()
    for name, (n, k, q_off, s_off) in ref.layout.items():
        assert np.array_equal(got[q_off:q_off + n * k], views[name][0].numpy().ravel())
        nb = 4 * (n // 128) * (k // 128)
        assert np.array_equal(got[s_off:s_off + nb].view(np.float32), views[name][1].numpy().ravel())
