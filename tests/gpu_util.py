"""Shared helpers of the GPU parity tests: move tensors between the CUDA path (torch
device tensors through the C-ABI binding) and the oracle (numpy arrays)."""
import numpy as np
import torch


def bits(t: torch.Tensor) -> np.ndarray:
    """BF16 tensor (any device) -> numpy uint16 bit patterns."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def np_u8(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().numpy()


def np_f32(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().numpy()


def bf16_values(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def assert_codes_equal(gpu_q, ref_q, what=""):
    g = np_u8(gpu_q)
    if not np.array_equal(g, ref_q):
        bad = np.argwhere(g != ref_q)
        i = tuple(bad[0])
        raise AssertionError("%s: %d code mismatches, first at %s: gpu %#x oracle %#x" % (
            what, len(bad), i, g[i], ref_q[i]))


def assert_scales_equal(gpu_s, ref_s, what="", cols=None):
    g = np_f32(gpu_s)
    if cols is not None:
        g, ref_s = g[:, :cols], ref_s[:, :cols]
    if not np.array_equal(g.view(np.uint32), ref_s.view(np.uint32)):
        bad = np.argwhere(g.view(np.uint32) != ref_s.view(np.uint32))
        i = tuple(bad[0])
        raise AssertionError("%s: %d scale mismatches, first at %s: gpu %r oracle %r" % (
            what, len(bad), i, g[i], ref_s[i]))


def gemm_tolerance(ref: np.ndarray, absdot: np.ndarray) -> np.ndarray:
    """The accepted error of a BF16 GEMM output: one BF16 ulp of the fp64 oracle value
    plus 1e-5 * sum_k |a_k b_k|."""
    v = np.abs(ref)
    ulp = np.zeros_like(v)
    nz = v > 0
    ulp[nz] = np.exp2(np.floor(np.log2(v[nz])) - 7)
    return ulp + 1e-5 * absdot


def assert_gemm_close(gpu: np.ndarray, ref: np.ndarray, absdot: np.ndarray, what=""):
    gpu = np.asarray(gpu, np.float64)
    err = np.abs(gpu - ref)
    tol = gemm_tolerance(ref, absdot)
    bad = err > tol
    if bad.any():
        idx = np.argwhere(bad)
        i = tuple(idx[0])
        raise AssertionError("%s: %d/%d outside tolerance; first %s gpu %r oracle %r tol %r "
                             "(max err/tol %.3g)" % (what, len(idx), bad.size, i, gpu[i], ref[i],
                                                     tol[i], float((err / np.maximum(tol, 1e-300)).max())))
