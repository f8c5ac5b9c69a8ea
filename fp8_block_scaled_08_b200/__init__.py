"""Python binding of libfp8q (the block-scaled FP8 linear layer for B200, sm_100a).

Argument marshalling only: each function checks dtypes/shapes, allocates nothing
unless asked to (the ``*_alloc`` helpers), and calls the C entry point of the same
name with device pointers and the current CUDA stream. Every step of the path runs
in libfp8q's kernels; there is no CPU or PyTorch fallback. If libfp8q.so is missing
or stale the import fails loudly: build it with ``python fp8_block_scaled_08_b200/build.py``.

The operations follow "Resumen Técnico: Jet-RL" (gist.science, paper 2601.14243),
section "Esquema de Cuantización"; see include/fp8q.h for layouts and semantics.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfp8q.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        "libfp8q.so is not built (%s); run `python fp8_block_scaled_08_b200/build.py`" % LIB_PATH)

_lib = ctypes.CDLL(LIB_PATH)

FP8Q_OK = 0
FP8Q_ERR_NULL = 1
FP8Q_ERR_SHAPE = 2
FP8Q_ERR_ALIGN = 3
FP8Q_ERR_CUDA = 4
FP8Q_ERR_TIMEOUT = 5
FP8Q_ERR_UNSUPPORTED = 6

_P = ctypes.c_void_p
_I = ctypes.c_int64
_F = ctypes.c_float

_SIGS = {
    "fp8q_status_string": ([ctypes.c_int], ctypes.c_char_p),
    "fp8q_version": ([], ctypes.c_int),
    "fp8q_last_error_message": ([], ctypes.c_char_p),
    "fp8q_device_error": ([_P, ctypes.c_int], ctypes.c_int),
    "fp8q_last_device_error": ([_P], ctypes.c_int),
    "fp8q_quant_act_1x128": ([_P, _I, _I, _I, _P, _P, _I, _P], ctypes.c_int),
    "fp8q_quant_weight_128x128": ([_P, _I, _I, _I, _P, _P, _P, _P], ctypes.c_int),
    "fp8q_rmsnorm_quant": ([_P, _P, _I, _I, _I, _F, _P, _P, _I, _P], ctypes.c_int),
    "fp8q_swiglu_quant": ([_P, _I, _I, _I, _P, _P, _I, _P], ctypes.c_int),
    "fp8q_transpose_quant_bf16": ([_P, _I, _I, _I, _P, _P, _I, _P, _P, _P], ctypes.c_int),
    "fp8q_transpose_quant_fp8": ([_P, _P, _I, _I, _I, _P, _P, _P], ctypes.c_int),
    "fp8q_rmsnorm_quant_dual": ([_P, _P, _I, _I, _I, _F, _P, _P, _I, _P, _P, _P, _P],
                                ctypes.c_int),
    "fp8q_swiglu_quant_dual": ([_P, _I, _I, _I, _P, _P, _I, _P, _P, _P], ctypes.c_int),
    "fp8q_swiglu_bwd_quant_dual": ([_P, _P, _I, _I, _P, _P, _P, _I, _P, _P, _P], ctypes.c_int),
    "fp8q_rmsnorm_bwd_workspace_bytes": ([_I, _I], ctypes.c_int64),
    "fp8q_rmsnorm_bwd_quant_dual": ([_P, _P, _P, _P, _I, _I, _F, _P, _P, _P, _I, _P, _P, _P,
                                     _P, _I, _P], ctypes.c_int),
    "fp8q_linear_fwd": ([_P, _P, _I, _P, _P, _I, _I, _I, _P, _I, _P], ctypes.c_int),
    "fp8q_linear_fwd_splitk_workspace": ([_I, _I, _I], ctypes.c_int64),
    "fp8q_linear_fwd_splitk_counter_bytes": ([_I, _I], ctypes.c_int64),
    "fp8q_linear_fwd_splitk": ([_P, _P, _I, _P, _P, _I, _I, _I, _P, _I, _P, _I, _P],
                               ctypes.c_int),
    "fp8q_linear_fwd_splitk_noalloc": ([_P, _P, _I, _P, _P, _I, _I, _I, _P, _I, _P],
                                       ctypes.c_int),
    "fp8q_linear_dgrad": ([_P, _P, _I, _P, _P, _I, _I, _I, _P, _I, _P], ctypes.c_int),
    "fp8q_linear_wgrad": ([_P, _P, _P, _P, _I, _I, _I, _P, _I, _P], ctypes.c_int),
    "fp8q_linear_wgrad_acc_f32": ([_P, _P, _P, _P, _I, _I, _I, _P, _I, _P], ctypes.c_int),
    "fp8q_debug_wait_timeout": ([_I, _P], ctypes.c_int),
}
for _name, (_args, _res) in _SIGS.items():
    try:
        _fn = getattr(_lib, _name)
    except AttributeError as _e:
        raise ImportError("libfp8q.so is stale (no %s); rebuild it with "
                          "`python fp8_block_scaled_08_b200/build.py`" % _name) from _e
    _fn.argtypes = _args
    _fn.restype = _res

EXPORTED = tuple(_SIGS)


class Fp8qError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        detail = ""
        if status in (FP8Q_ERR_CUDA, FP8Q_ERR_UNSUPPORTED):
            detail = " [%s]" % last_error_message()
        super().__init__("%s: %s%s" % (where, status_string(status), detail))


def status_string(status: int) -> str:
    return _lib.fp8q_status_string(int(status)).decode()


def last_error_message() -> str:
    return _lib.fp8q_last_error_message().decode()


def version() -> int:
    return int(_lib.fp8q_version())


def _check(status: int, where: str) -> None:
    if status != FP8Q_OK:
        raise Fp8qError(status, where)


def _ptr(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch.Tensor")
    if not t.is_cuda:
        raise ValueError("libfp8q takes CUDA tensors (device pointers)")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _want(t, dtype, ndim, name):
    if t.dtype != dtype or t.dim() != ndim:
        raise ValueError("%s must be a %d-D %s tensor, got %s %s" % (
            name, ndim, dtype, tuple(t.shape), t.dtype))


def _rows_dense(t, name):
    if t.stride(-1) != 1:
        raise ValueError("%s must have unit column stride" % name)
    return t.stride(0)


def _dense(t, name):
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)


def _groups(n: int) -> int:
    """Number of 128-wide groups covering n elements."""
    return (int(n) + 127) // 128


def _shape(t, shape, dtype, name):
    """Operand `name` must be a `dtype` tensor of exactly `shape` (checked before any
    pointer reaches the C side, whose tensor maps and stores trust these extents)."""
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch.Tensor" % name)
    if t.dtype != dtype or tuple(t.shape) != tuple(int(d) for d in shape):
        raise ValueError("%s must be a %s tensor of shape %s, got %s %s" % (
            name, dtype, tuple(int(d) for d in shape), tuple(t.shape), t.dtype))


def _scales_1x128(s, groups, rows, name):
    """1x128 scale array: fp32 [groups, lds] with lds >= rows (a multiple of 4 is
    checked by the library)."""
    if not isinstance(s, torch.Tensor):
        raise TypeError("%s must be a torch.Tensor" % name)
    if s.dtype != torch.float32 or s.dim() != 2 or s.shape[0] != groups or s.shape[1] < rows:
        raise ValueError("%s must be a float32 tensor [%d, >=%d], got %s %s" % (
            name, groups, rows, tuple(s.shape), s.dtype))


def lds_for(m: int) -> int:
    """Smallest legal leading dimension of a 1x128 scale array for M rows."""
    return (max(m, 1) + 3) // 4 * 4


# --------------------------------------------------------------------------
# Raw entry points (caller-owned outputs)
# --------------------------------------------------------------------------

def device_error(stream=None, clear: bool = True) -> int:
    """Synchronise the stream and return (and clear) the device error status."""
    return int(_lib.fp8q_device_error(_stream(stream), 1 if clear else 0))


def quant_act_1x128(x, q, s, stream=None):
    """a1: x BF16 [M,K] -> q uint8 [M,K], s float32 [K/128, lds]."""
    _want(x, torch.bfloat16, 2, "x"); _want(q, torch.uint8, 2, "q"); _want(s, torch.float32, 2, "s")
    _dense(q, "q"); _dense(s, "s")
    M, K = x.shape
    _shape(q, (M, K), torch.uint8, "q")
    _scales_1x128(s, _groups(K), M, "s")
    _check(_lib.fp8q_quant_act_1x128(_ptr(x), M, K, _rows_dense(x, "x"), _ptr(q), _ptr(s),
                                     s.shape[1], _stream(stream)), "fp8q_quant_act_1x128")


def quant_weight_128x128(w, q, s, qT=None, stream=None):
    """a2: w BF16 [N,K] -> q [N,K], s [N/128,K/128], optional qT [K,N]."""
    _want(w, torch.bfloat16, 2, "w"); _want(q, torch.uint8, 2, "q"); _want(s, torch.float32, 2, "s")
    _dense(q, "q"); _dense(s, "s")
    if qT is not None:
        _want(qT, torch.uint8, 2, "qT"); _dense(qT, "qT")
    N, K = w.shape
    _shape(q, (N, K), torch.uint8, "q")
    _shape(s, (_groups(N), _groups(K)), torch.float32, "s")
    if qT is not None:
        _shape(qT, (K, N), torch.uint8, "qT")
    _check(_lib.fp8q_quant_weight_128x128(_ptr(w), N, K, _rows_dense(w, "w"), _ptr(q), _ptr(s),
                                          _ptr(qT), _stream(stream)), "fp8q_quant_weight_128x128")


def rmsnorm_quant(x, gamma, eps, q, s, stream=None):
    """a3: RMSNorm(x)*gamma rounded to BF16, then 1x128 quantization."""
    _want(x, torch.bfloat16, 2, "x"); _want(gamma, torch.bfloat16, 1, "gamma")
    _want(q, torch.uint8, 2, "q"); _want(s, torch.float32, 2, "s")
    _dense(gamma, "gamma"); _dense(q, "q"); _dense(s, "s")
    M, H = x.shape
    _shape(gamma, (H,), torch.bfloat16, "gamma")
    _shape(q, (M, H), torch.uint8, "q")
    _scales_1x128(s, _groups(H), M, "s")
    _check(_lib.fp8q_rmsnorm_quant(_ptr(x), _ptr(gamma), M, H, _rows_dense(x, "x"), float(eps),
                                   _ptr(q), _ptr(s), s.shape[1], _stream(stream)),
           "fp8q_rmsnorm_quant")


def swiglu_quant(gu, q, s, stream=None):
    """a4: gu BF16 [M,2I] (gate | up) -> SwiGLU BF16 -> 1x128 quantization."""
    _want(gu, torch.bfloat16, 2, "gu"); _want(q, torch.uint8, 2, "q"); _want(s, torch.float32, 2, "s")
    _dense(q, "q"); _dense(s, "s")
    M, I2 = gu.shape
    if I2 % 2:
        raise ValueError("gu must be [M, 2I] (gate | up), got %s" % (tuple(gu.shape),))
    _shape(q, (M, I2 // 2), torch.uint8, "q")
    _scales_1x128(s, _groups(I2 // 2), M, "s")
    _check(_lib.fp8q_swiglu_quant(_ptr(gu), M, I2 // 2, _rows_dense(gu, "gu"), _ptr(q), _ptr(s),
                                  s.shape[1], _stream(stream)), "fp8q_swiglu_quant")


def transpose_quant_bf16(dy, q_row, s_row, q_colT, s_col, stream=None):
    """a6: dY BF16 [M,N] -> row-wise (q_row [M,N], s_row [N/128,lds]) and column-wise
    transposed (q_colT [N,M], s_col [M/128,N]). q_row/s_row may be None."""
    _want(dy, torch.bfloat16, 2, "dy")
    _want(q_colT, torch.uint8, 2, "q_colT"); _want(s_col, torch.float32, 2, "s_col")
    _dense(q_colT, "q_colT"); _dense(s_col, "s_col")
    lds_row = 0
    if q_row is not None:
        _want(q_row, torch.uint8, 2, "q_row"); _want(s_row, torch.float32, 2, "s_row")
        _dense(q_row, "q_row"); _dense(s_row, "s_row")
        lds_row = s_row.shape[1]
    M, N = dy.shape
    if q_row is not None:
        _shape(q_row, (M, N), torch.uint8, "q_row")
        _scales_1x128(s_row, _groups(N), M, "s_row")
    _shape(q_colT, (N, M), torch.uint8, "q_colT")
    _shape(s_col, (_groups(M), N), torch.float32, "s_col")
    _check(_lib.fp8q_transpose_quant_bf16(_ptr(dy), M, N, _rows_dense(dy, "dy"), _ptr(q_row),
                                          _ptr(s_row), lds_row, _ptr(q_colT), _ptr(s_col),
                                          _stream(stream)), "fp8q_transpose_quant_bf16")


def transpose_quant_fp8(q, s, qT, sT, stream=None):
    """a8: saved FP8 (q [M,K], s [K/128,lds]) -> 128x1 requantized transposed (qT [K,M],
    sT [M/128,K])."""
    _want(q, torch.uint8, 2, "q"); _want(s, torch.float32, 2, "s")
    _want(qT, torch.uint8, 2, "qT"); _want(sT, torch.float32, 2, "sT")
    for t, n in ((q, "q"), (s, "s"), (qT, "qT"), (sT, "sT")):
        _dense(t, n)
    M, K = q.shape
    _scales_1x128(s, _groups(K), M, "s")
    _shape(qT, (K, M), torch.uint8, "qT")
    _shape(sT, (_groups(M), K), torch.float32, "sT")
    _check(_lib.fp8q_transpose_quant_fp8(_ptr(q), _ptr(s), M, K, s.shape[1], _ptr(qT), _ptr(sT),
                                         _stream(stream)), "fp8q_transpose_quant_fp8")


def rmsnorm_quant_dual(x, gamma, eps, q_row, s_row, q_colT, s_col, rstd, stream=None):
    """Option B: RMSNorm(x)*gamma in BF16, emitted 1x128 (rows) and 128x1 (transposed),
    plus the per-row reciprocal RMS."""
    _want(x, torch.bfloat16, 2, "x"); _want(gamma, torch.bfloat16, 1, "gamma")
    for t, n in ((q_row, "q_row"), (s_row, "s_row"), (q_colT, "q_colT"), (s_col, "s_col"),
                 (rstd, "rstd")):
        _dense(t, n)
    M, H = x.shape
    _shape(gamma, (H,), torch.bfloat16, "gamma")
    _shape(q_row, (M, H), torch.uint8, "q_row")
    _scales_1x128(s_row, _groups(H), M, "s_row")
    _shape(q_colT, (H, M), torch.uint8, "q_colT")
    _shape(s_col, (_groups(M), H), torch.float32, "s_col")
    _shape(rstd, (M,), torch.float32, "rstd")
    _check(_lib.fp8q_rmsnorm_quant_dual(_ptr(x), _ptr(gamma), M, H, _rows_dense(x, "x"),
                                        float(eps), _ptr(q_row), _ptr(s_row), s_row.shape[1],
                                        _ptr(q_colT), _ptr(s_col), _ptr(rstd), _stream(stream)),
           "fp8q_rmsnorm_quant_dual")


def rmsnorm_quant_dual_alloc(x, gamma, eps, stream=None):
    M, H = x.shape
    q = _empty((M, H), torch.uint8, x.device)
    s = _empty((_groups(H), lds_for(M)), torch.float32, x.device)
    qT = _empty((H, M), torch.uint8, x.device)
    sT = _empty((_groups(M), H), torch.float32, x.device)
    r = _empty((M,), torch.float32, x.device)
    rmsnorm_quant_dual(x, gamma, eps, q, s, qT, sT, r, stream)
    return q, s, qT, sT, r


def swiglu_quant_dual(gu, q_row, s_row, q_colT, s_col, stream=None):
    """Option B: SwiGLU(gate, up) in BF16, emitted 1x128 (rows) and 128x1 (transposed)."""
    _want(gu, torch.bfloat16, 2, "gu")
    for t, n in ((q_row, "q_row"), (s_row, "s_row"), (q_colT, "q_colT"), (s_col, "s_col")):
        _dense(t, n)
    M, I2 = gu.shape
    if I2 % 2:
        raise ValueError("gu must be [M, 2I] (gate | up), got %s" % (tuple(gu.shape),))
    I = I2 // 2
    _shape(q_row, (M, I), torch.uint8, "q_row")
    _scales_1x128(s_row, _groups(I), M, "s_row")
    _shape(q_colT, (I, M), torch.uint8, "q_colT")
    _shape(s_col, (_groups(M), I), torch.float32, "s_col")
    _check(_lib.fp8q_swiglu_quant_dual(_ptr(gu), M, I2 // 2, _rows_dense(gu, "gu"), _ptr(q_row),
                                       _ptr(s_row), s_row.shape[1], _ptr(q_colT), _ptr(s_col),
                                       _stream(stream)), "fp8q_swiglu_quant_dual")


def swiglu_quant_dual_alloc(gu, stream=None):
    M, I2 = gu.shape
    I = I2 // 2
    q = _empty((M, I), torch.uint8, gu.device)
    s = _empty((_groups(I), lds_for(M)), torch.float32, gu.device)
    qT = _empty((I, M), torch.uint8, gu.device)
    sT = _empty((_groups(M), I), torch.float32, gu.device)
    swiglu_quant_dual(gu, q, s, qT, sT, stream)
    return q, s, qT, sT


def swiglu_bwd_quant_dual(gu, dh, q_row, s_row, q_colT, s_col, dgu=None, stream=None):
    """SwiGLU backward in BF16 (gu [M, 2I] = [gate | up], dh [M, I]) with the gradient
    [d_gate | d_up] quantized 1x128 (rows) and 128x1 (transposed); dgu optionally receives
    the BF16 gradient."""
    _want(gu, torch.bfloat16, 2, "gu"); _want(dh, torch.bfloat16, 2, "dh")
    for t, n in ((gu, "gu"), (dh, "dh"), (q_row, "q_row"), (s_row, "s_row"),
                 (q_colT, "q_colT"), (s_col, "s_col")):
        _dense(t, n)
    if dgu is not None:
        _want(dgu, torch.bfloat16, 2, "dgu"); _dense(dgu, "dgu")
    M, I2 = gu.shape
    if dh.shape != (M, I2 // 2):
        raise ValueError("dh must be [M, I] for gu [M, 2I]")
    _shape(q_row, (M, I2), torch.uint8, "q_row")
    _scales_1x128(s_row, _groups(I2), M, "s_row")
    _shape(q_colT, (I2, M), torch.uint8, "q_colT")
    _shape(s_col, (_groups(M), I2), torch.float32, "s_col")
    if dgu is not None:
        _shape(dgu, (M, I2), torch.bfloat16, "dgu")
    _check(_lib.fp8q_swiglu_bwd_quant_dual(_ptr(gu), _ptr(dh), M, I2 // 2, _ptr(dgu), _ptr(q_row),
                                           _ptr(s_row), s_row.shape[1], _ptr(q_colT),
                                           _ptr(s_col), _stream(stream)),
           "fp8q_swiglu_bwd_quant_dual")


def swiglu_bwd_quant_dual_alloc(gu, dh, want_dgu=False, stream=None):
    M, I2 = gu.shape
    q = _empty((M, I2), torch.uint8, gu.device)
    s = _empty((_groups(I2), lds_for(M)), torch.float32, gu.device)
    qT = _empty((I2, M), torch.uint8, gu.device)
    sT = _empty((_groups(M), I2), torch.float32, gu.device)
    dgu = _empty((M, I2), torch.bfloat16, gu.device) if want_dgu else None
    swiglu_bwd_quant_dual(gu, dh, q, s, qT, sT, dgu, stream)
    return q, s, qT, sT, dgu


def rmsnorm_bwd_workspace_bytes(M: int, H: int) -> int:
    return int(_lib.fp8q_rmsnorm_bwd_workspace_bytes(int(M), int(H)))


def rmsnorm_bwd_quant_dual(x, gamma, dy, dres, eps, out, q_row, s_row, q_colT, s_col, dgamma,
                           workspace, stream=None):
    """RMSNorm backward in BF16 plus the residual gradient dres (may be None): out [M, H]
    BF16, its 1x128 and 128x1 (transposed) quantizations, dgamma [H] fp32 (may be None).
    workspace: a uint8 CUDA tensor of rmsnorm_bwd_workspace_bytes(M, H) bytes."""
    _want(x, torch.bfloat16, 2, "x"); _want(gamma, torch.bfloat16, 1, "gamma")
    _want(dy, torch.bfloat16, 2, "dy"); _want(out, torch.bfloat16, 2, "out")
    if dres is not None:
        _want(dres, torch.bfloat16, 2, "dres")
    for t, n in ((x, "x"), (dy, "dy"), (dres, "dres"), (out, "out"), (q_row, "q_row"),
                 (s_row, "s_row"), (q_colT, "q_colT"), (s_col, "s_col"), (dgamma, "dgamma"),
                 (workspace, "workspace")):
        if t is not None:
            _dense(t, n)
    M, H = x.shape
    for t, n in ((dy, "dy"), (dres, "dres"), (out, "out")):
        if t is not None and t.shape != (M, H):
            raise ValueError("%s must have the shape of x" % n)
    _shape(gamma, (H,), torch.bfloat16, "gamma")
    _shape(q_row, (M, H), torch.uint8, "q_row")
    _scales_1x128(s_row, _groups(H), M, "s_row")
    _shape(q_colT, (H, M), torch.uint8, "q_colT")
    _shape(s_col, (_groups(M), H), torch.float32, "s_col")
    if dgamma is not None:
        _shape(dgamma, (H,), torch.float32, "dgamma")
    if workspace.dtype != torch.uint8:
        raise ValueError("workspace must be a uint8 tensor")
    _check(_lib.fp8q_rmsnorm_bwd_quant_dual(
        _ptr(x), _ptr(gamma), _ptr(dy), _ptr(dres), M, H, float(eps), _ptr(out), _ptr(q_row),
        _ptr(s_row), s_row.shape[1], _ptr(q_colT), _ptr(s_col), _ptr(dgamma), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)),
        "fp8q_rmsnorm_bwd_quant_dual")


def rmsnorm_bwd_quant_dual_alloc(x, gamma, dy, dres, eps, stream=None):
    M, H = x.shape
    dev = x.device
    out = _empty((M, H), torch.bfloat16, dev)
    q = _empty((M, H), torch.uint8, dev)
    s = _empty((_groups(H), lds_for(M)), torch.float32, dev)
    qT = _empty((H, M), torch.uint8, dev)
    sT = _empty((_groups(M), H), torch.float32, dev)
    dg = _empty((H,), torch.float32, dev)
    nbytes = rmsnorm_bwd_workspace_bytes(M, H)
    ws = _empty((max(nbytes, 16),), torch.uint8, dev)
    rmsnorm_bwd_quant_dual(x, gamma, dy, dres, eps, out, q, s, qT, sT, dg, ws, stream)
    return out, q, s, qT, sT, dg


def _gemm_operands(qa, sa, qw, name_a, name_sa, name_w):
    """Extents of a block-scaled product [M, N] = qa [M, K] x qw [N, K]^T: checks the
    two code operands and the 1x128 row scales sa [K/128, >= M]; returns (M, N, K) for
    the caller to check the block scales and the output against."""
    if not isinstance(qa, torch.Tensor) or qa.dim() != 2 or qa.dtype != torch.uint8:
        raise ValueError("%s must be a 2-D uint8 tensor" % name_a)
    if not isinstance(qw, torch.Tensor) or qw.dim() != 2 or qw.dtype != torch.uint8:
        raise ValueError("%s must be a 2-D uint8 tensor" % name_w)
    M, K = qa.shape
    N = qw.shape[0]
    _shape(qw, (N, K), torch.uint8, name_w)
    _scales_1x128(sa, _groups(K), M, name_sa)
    return M, N, K


def linear_fwd(qa, sa, qw, sw, y, stream=None):
    """a5: y BF16 [M,N] = block-scaled qa [M,K] x qw [N,K]^T."""
    for t, n in ((qa, "qa"), (sa, "sa"), (qw, "qw"), (sw, "sw")):
        _dense(t, n)
    M, N, K = _gemm_operands(qa, sa, qw, "qa", "sa", "qw")
    _shape(sw, (_groups(N), _groups(K)), torch.float32, "sw")
    _shape(y, (M, N), torch.bfloat16, "y")
    _check(_lib.fp8q_linear_fwd(_ptr(qa), _ptr(sa), sa.shape[1], _ptr(qw), _ptr(sw), M, N, K,
                                _ptr(y), _rows_dense(y, "y"), _stream(stream)), "fp8q_linear_fwd")


def linear_fwd_splitk_workspace_bytes(M, N, K):
    """Bytes of workspace fp8q_linear_fwd_splitk needs for this shape (0 if unsupported)."""
    return int(_lib.fp8q_linear_fwd_splitk_workspace(M, N, K))


def splitk_workspace(M, N, K, device):
    """A workspace for fp8q_linear_fwd_splitk, zero-filled (its counters must start at
    zero; the kernel leaves them at zero)."""
    n = linear_fwd_splitk_workspace_bytes(M, N, K)
    if n <= 0:
        raise ValueError("no split-K workspace for M=%d N=%d K=%d" % (M, N, K))
    return torch.zeros(n, dtype=torch.uint8, device=device)


def linear_fwd_splitk(qa, sa, qw, sw, y, workspace, stream=None):
    """a5 at decode sizes with K split over CTAs (same bits as linear_fwd); `workspace`
    is a uint8 device tensor from splitk_workspace (not shared by concurrent calls)."""
    for t, n in ((qa, "qa"), (sa, "sa"), (qw, "qw"), (sw, "sw")):
        _dense(t, n)
    M, N, K = _gemm_operands(qa, sa, qw, "qa", "sa", "qw")
    _shape(sw, (_groups(N), _groups(K)), torch.float32, "sw")
    _shape(y, (M, N), torch.bfloat16, "y")
    _want(workspace, torch.uint8, 1, "workspace")
    _check(_lib.fp8q_linear_fwd_splitk(_ptr(qa), _ptr(sa), sa.shape[1], _ptr(qw), _ptr(sw), M, N,
                                       K, _ptr(y), _rows_dense(y, "y"), _ptr(workspace),
                                       workspace.numel(), _stream(stream)),
           "fp8q_linear_fwd_splitk")


def linear_fwd_splitk_noalloc(qa, sa, qw, sw, y, stream=None):
    """linear_fwd_splitk on the library's static workspace (no allocation; calls on one
    device must not overlap)."""
    for t, n in ((qa, "qa"), (sa, "sa"), (qw, "qw"), (sw, "sw")):
        _dense(t, n)
    M, N, K = _gemm_operands(qa, sa, qw, "qa", "sa", "qw")
    _shape(sw, (_groups(N), _groups(K)), torch.float32, "sw")
    _shape(y, (M, N), torch.bfloat16, "y")
    _check(_lib.fp8q_linear_fwd_splitk_noalloc(_ptr(qa), _ptr(sa), sa.shape[1], _ptr(qw),
                                               _ptr(sw), M, N, K, _ptr(y), _rows_dense(y, "y"),
                                               _stream(stream)),
           "fp8q_linear_fwd_splitk_noalloc")


def linear_dgrad(qdy, sdy, qwT, sw, dx, stream=None):
    """a7: dx BF16 [M,K] = block-scaled qdy [M,N] x W [N,K] (weights passed transposed,
    qwT [K,N])."""
    for t, n in ((qdy, "qdy"), (sdy, "sdy"), (qwT, "qwT"), (sw, "sw")):
        _dense(t, n)
    # dx [M, K] = qdy [M, N] x qwT [K, N]^T: the product's reduction runs over N
    M, K, N = _gemm_operands(qdy, sdy, qwT, "qdy", "sdy", "qwT")
    _shape(sw, (_groups(N), _groups(K)), torch.float32, "sw")
    _shape(dx, (M, K), torch.bfloat16, "dx")
    _check(_lib.fp8q_linear_dgrad(_ptr(qdy), _ptr(sdy), sdy.shape[1], _ptr(qwT), _ptr(sw), M, N,
                                  K, _ptr(dx), _rows_dense(dx, "dx"), _stream(stream)),
           "fp8q_linear_dgrad")


def _wgrad_operands(qdyT, sdy_c, qxT, sx_c):
    """Shapes of WGrad: qdyT [N, M] and qxT [K, M] (128x1 codes, transposed) with their
    scales sdy_c [M/128, N] and sx_c [M/128, K]. Returns (N, M, K)."""
    for t, n in ((qdyT, "qdyT"), (qxT, "qxT")):
        if not isinstance(t, torch.Tensor) or t.dim() != 2 or t.dtype != torch.uint8:
            raise ValueError("%s must be a 2-D uint8 tensor" % n)
    N, M = qdyT.shape
    K = qxT.shape[0]
    _shape(qxT, (K, M), torch.uint8, "qxT")
    _shape(sdy_c, (_groups(M), N), torch.float32, "sdy_c")
    _shape(sx_c, (_groups(M), K), torch.float32, "sx_c")
    return N, M, K


def linear_wgrad(qdyT, sdy_c, qxT, sx_c, dw, stream=None):
    """a9: dw BF16 [N,K] = sum over 128-token groups of (qdyT [N,M]) x (qxT [K,M])^T with
    the 128x1 scales sdy_c [M/128,N] and sx_c [M/128,K]."""
    for t, n in ((qdyT, "qdyT"), (sdy_c, "sdy_c"), (qxT, "qxT"), (sx_c, "sx_c")):
        _dense(t, n)
    N, M, K = _wgrad_operands(qdyT, sdy_c, qxT, sx_c)
    _shape(dw, (N, K), torch.bfloat16, "dw")
    _check(_lib.fp8q_linear_wgrad(_ptr(qdyT), _ptr(sdy_c), _ptr(qxT), _ptr(sx_c), M, N, K,
                                  _ptr(dw), _rows_dense(dw, "dw"), _stream(stream)),
           "fp8q_linear_wgrad")


def linear_wgrad_acc_f32(qdyT, sdy_c, qxT, sx_c, dw, stream=None):
    """WGrad accumulated in fp32: dw [N,K] (fp32) += the fp32 accumulator of linear_wgrad."""
    for t, n in ((qdyT, "qdyT"), (sdy_c, "sdy_c"), (qxT, "qxT"), (sx_c, "sx_c")):
        _dense(t, n)
    N, M, K = _wgrad_operands(qdyT, sdy_c, qxT, sx_c)
    _shape(dw, (N, K), torch.float32, "dw")
    _check(_lib.fp8q_linear_wgrad_acc_f32(_ptr(qdyT), _ptr(sdy_c), _ptr(qxT), _ptr(sx_c), M, N,
                                          K, _ptr(dw), _rows_dense(dw, "dw"), _stream(stream)),
           "fp8q_linear_wgrad_acc_f32")


def debug_wait_timeout(limit_ns: int, stream=None) -> int:
    """Launch the bounded-wait probe (gives up after limit_ns); returns the launch status."""
    return int(_lib.fp8q_debug_wait_timeout(int(limit_ns), _stream(stream)))


# --------------------------------------------------------------------------
# Allocating helpers (torch allocates; the kernels are the ones above)
# --------------------------------------------------------------------------

def _empty(shape, dtype, device):
    return torch.empty(shape, dtype=dtype, device=device)


def quant_act_1x128_alloc(x, stream=None):
    M, K = x.shape
    q = _empty((M, K), torch.uint8, x.device)
    s = _empty((_groups(K), lds_for(M)), torch.float32, x.device)
    quant_act_1x128(x, q, s, stream)
    return q, s


def quant_weight_alloc(w, want_t=True, stream=None):
    N, K = w.shape
    q = _empty((N, K), torch.uint8, w.device)
    s = _empty((_groups(N), _groups(K)), torch.float32, w.device)
    qT = _empty((K, N), torch.uint8, w.device) if want_t else None
    quant_weight_128x128(w, q, s, qT, stream)
    return q, s, qT


def rmsnorm_quant_alloc(x, gamma, eps, stream=None):
    M, H = x.shape
    q = _empty((M, H), torch.uint8, x.device)
    s = _empty((_groups(H), lds_for(M)), torch.float32, x.device)
    rmsnorm_quant(x, gamma, eps, q, s, stream)
    return q, s


def swiglu_quant_alloc(gu, stream=None):
    M, I2 = gu.shape
    q = _empty((M, I2 // 2), torch.uint8, gu.device)
    s = _empty((_groups(I2 // 2), lds_for(M)), torch.float32, gu.device)
    swiglu_quant(gu, q, s, stream)
    return q, s


def transpose_quant_bf16_alloc(dy, want_row=True, stream=None):
    M, N = dy.shape
    q_row = _empty((M, N), torch.uint8, dy.device) if want_row else None
    s_row = _empty((_groups(N), lds_for(M)), torch.float32, dy.device) if want_row else None
    q_colT = _empty((N, M), torch.uint8, dy.device)
    s_col = _empty((_groups(M), N), torch.float32, dy.device)
    transpose_quant_bf16(dy, q_row, s_row, q_colT, s_col, stream)
    return q_row, s_row, q_colT, s_col


def transpose_quant_fp8_alloc(q, s, stream=None):
    M, K = q.shape
    qT = _empty((K, M), torch.uint8, q.device)
    sT = _empty((_groups(M), K), torch.float32, q.device)
    transpose_quant_fp8(q, s, qT, sT, stream)
    return qT, sT


def linear_fwd_alloc(qa, sa, qw, sw, stream=None):
    y = _empty((qa.shape[0], qw.shape[0]), torch.bfloat16, qa.device)
    linear_fwd(qa, sa, qw, sw, y, stream)
    return y


def linear_dgrad_alloc(qdy, sdy, qwT, sw, stream=None):
    dx = _empty((qdy.shape[0], qwT.shape[0]), torch.bfloat16, qdy.device)
    linear_dgrad(qdy, sdy, qwT, sw, dx, stream)
    return dx


def linear_wgrad_alloc(qdyT, sdy_c, qxT, sx_c, stream=None):
    dw = _empty((qdyT.shape[0], qxT.shape[0]), torch.bfloat16, qdyT.device)
    linear_wgrad(qdyT, sdy_c, qxT, sx_c, dw, stream)
    return dw
