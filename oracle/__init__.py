"""fp8q oracle: the plain CPU definition of the block-scaled FP8 linear-layer path.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
/ reference leg of ``bench.py`` may import this package. The CUDA library and its
Python binding never import it, and it imports nothing from them.

Elementwise and group arithmetic (E4M3 encode/decode, the quantizers, RMSNorm, SwiGLU,
the transposed requantizers) lives in ``fp8q_oracle.c`` (plain C, built with gcc, no
FMA contraction, IEEE division). The GEMMs are written here: both operands are
dequantized exactly to fp64 and multiplied with numpy's fp64 matmul.

Method: "Resumen Técnico: Jet-RL" (gist.science, paper 2601.14243), section
"Esquema de Cuantización" (1x128 activation groups, 128x128 weight blocks, FP8 saved
activations, BF16 inter-operator gradients, FP8 DGrad/WGrad with 1x128 and 128x1
grouping for WGrad) and section "Implementación" (fused quantize / transpose /
activation / RMSNorm kernels next to FP8 GEMMs).

Layouts (all row-major; G(n) = ceil(n / 128) groups along a dimension of n elements,
the last one partial when n is not a multiple of 128):
  codes          uint8 [rows][cols]
  1x128 scales   float32 [G(cols)][lds]    scale of (row m, group g) at s[g, m]
  weight scales  float32 [G(N)][G(K)]
  128x1 scales   float32 [G(rows)][cols]   scale of (group mb, column c) at s[mb, c]

Partial groups (dimensions that are not multiples of 128): the group is the full group
with zeros in the missing places; its scale comes from its valid elements alone and
only the codes of the valid places exist.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fp8q_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

GCC_FLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
             "-fno-fast-math", "-fopenmp"]


def build(force: bool = False) -> str:
    """Compile fp8q_oracle.c into liboracle.so next to it (gcc)."""
    if force or not os.path.exists(_LIB_PATH) or \
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", *GCC_FLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    # FP8Q_ORACLE_LIB: load another build of fp8q_oracle.c instead (the mutation test
    # of the pins points it at copies with a deliberately planted mistake)
    other = os.environ.get("FP8Q_ORACLE_LIB")
    if other:
        lib = ctypes.CDLL(other)
    else:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
    P = ctypes.c_void_p
    I = ctypes.c_int64
    F = ctypes.c_float
    lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
    lib.oracle_e4m3_decode.restype = ctypes.c_double
    lib.oracle_e4m3_encode.argtypes = [F]
    lib.oracle_e4m3_encode.restype = ctypes.c_uint8
    lib.oracle_bf16_to_f32.argtypes = [ctypes.c_uint16]
    lib.oracle_bf16_to_f32.restype = F
    lib.oracle_f32_to_bf16.argtypes = [F]
    lib.oracle_f32_to_bf16.restype = ctypes.c_uint16
    lib.oracle_exp_cw.argtypes = [F]
    lib.oracle_exp_cw.restype = F
    lib.oracle_swiglu_one.argtypes = [ctypes.c_uint16, ctypes.c_uint16]
    lib.oracle_swiglu_one.restype = ctypes.c_uint16
    lib.oracle_rmsnorm_rstd.argtypes = [P, I, F]
    lib.oracle_rmsnorm_rstd.restype = F
    lib.oracle_quant_act_1x128.argtypes = [P, I, I, I, P, P, I]
    lib.oracle_quant_weight_128x128.argtypes = [P, I, I, I, P, P, P]
    lib.oracle_rmsnorm_quant.argtypes = [P, P, I, I, I, F, P, P, I, P]
    lib.oracle_swiglu_quant.argtypes = [P, I, I, I, P, P, I, P]
    lib.oracle_transpose_quant_bf16.argtypes = [P, I, I, I, P, P, I, P, P]
    lib.oracle_transpose_quant_fp8.argtypes = [P, P, I, I, I, P, P]
    lib.oracle_swiglu_bwd_one.argtypes = [ctypes.c_uint16, ctypes.c_uint16, ctypes.c_uint16,
                                          P, P]
    lib.oracle_swiglu_bwd.argtypes = [P, P, I, I, P]
    lib.oracle_rmsnorm_bwd.argtypes = [P, P, P, P, I, I, F, P, P, P, P]
    lib.oracle_exact_sum_f32.argtypes = [P, I, ctypes.c_int]
    lib.oracle_exact_sum_f32.restype = ctypes.c_double
    lib.oracle_dequant_rows.argtypes = [P, P, I, I, I, I, I, P]
    lib.oracle_dequant_block.argtypes = [P, P, I, I, I, I, P]
    lib.oracle_dequant_cols.argtypes = [P, P, I, I, I, I, P]
    lib.oracle_num_threads.restype = ctypes.c_int
    _lib = lib
    return lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return ctypes.c_void_p(a.ctypes.data)


def _bf16(a) -> np.ndarray:
    """Accept BF16 data as uint16 bit patterns (numpy) or a torch bfloat16 tensor."""
    if hasattr(a, "dtype") and str(getattr(a, "dtype", "")) == "torch.bfloat16":
        a = a.detach().cpu().contiguous().view(__import__("torch").int16).numpy()
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        a = a.view(np.uint16)
    return a


def num_threads() -> int:
    return int(_load().oracle_num_threads())


# --------------------------------------------------------------------------
# Scalar definitions
# --------------------------------------------------------------------------

def e4m3_decode(code: int) -> float:
    """Value of an OCP E4M3 'fn' code (exact; NaN for S.1111.111)."""
    return float(_load().oracle_e4m3_decode(int(code) & 0xFF))


def e4m3_encode(t: float) -> int:
    """Nearest E4M3 code to the fp32 value t: ties to even, saturate at 448, sign kept."""
    return int(_load().oracle_e4m3_encode(float(np.float32(t))))


def e4m3_table() -> np.ndarray:
    """fp64 value of each of the 256 codes (NaN codes are NaN)."""
    lib = _load()
    return np.array([lib.oracle_e4m3_decode(c) for c in range(256)], dtype=np.float64)


def bf16_to_f32(b: int) -> float:
    return float(_load().oracle_bf16_to_f32(int(b)))


def f32_to_bf16(x: float) -> int:
    return int(_load().oracle_f32_to_bf16(float(np.float32(x))))


def exp_cw(x: float) -> float:
    """The method's fixed fp32 exponential (Cody-Waite + degree-7 Taylor), see the C file."""
    return float(_load().oracle_exp_cw(float(np.float32(x))))


def swiglu_one(gate_bits: int, up_bits: int) -> int:
    return int(_load().oracle_swiglu_one(int(gate_bits), int(up_bits)))


def rmsnorm_rstd(xrow_bits: np.ndarray, eps: float) -> float:
    x = _bf16(xrow_bits)
    return float(_load().oracle_rmsnorm_rstd(_p(x), x.shape[-1], float(eps)))


# --------------------------------------------------------------------------
# Quantizers (all outputs are fresh numpy arrays)
# --------------------------------------------------------------------------

def groups(n: int) -> int:
    """Number of 128-element groups along a dimension of n elements (the last one
    partial when n is not a multiple of 128)."""
    return (int(n) + 127) // 128


def _lds_for(M: int) -> int:
    return (M + 3) // 4 * 4


def quant_act_1x128(x, lds: int | None = None):
    """a1: x BF16 [M,K] -> (q uint8 [M,K], s float32 [K/128, lds])."""
    x = _bf16(x)
    M, K = x.shape
    lds = _lds_for(M) if lds is None else lds
    q = np.zeros((M, K), np.uint8)
    s = np.zeros((groups(K), lds), np.float32)
    _load().oracle_quant_act_1x128(_p(x), M, K, K, _p(q), _p(s), lds)
    return q, s


def quant_weight_128x128(w, want_t: bool = True):
    """a2: w BF16 [N,K] -> (q [N,K], s [N/128,K/128], qT [K,N] or None)."""
    w = _bf16(w)
    N, K = w.shape
    q = np.zeros((N, K), np.uint8)
    s = np.zeros((groups(N), groups(K)), np.float32)
    qT = np.zeros((K, N), np.uint8) if want_t else None
    _load().oracle_quant_weight_128x128(_p(w), N, K, K, _p(q), _p(s),
                                        _p(qT) if want_t else None)
    return q, s, qT


def rmsnorm_quant(x, gamma, eps: float, lds: int | None = None, want_y: bool = False):
    """a3: RMSNorm (BF16 output) fused with 1x128 quantization."""
    x = _bf16(x)
    g = _bf16(gamma)
    M, H = x.shape
    assert g.shape == (H,)
    lds = _lds_for(M) if lds is None else lds
    q = np.zeros((M, H), np.uint8)
    s = np.zeros((groups(H), lds), np.float32)
    y = np.zeros((M, H), np.uint16) if want_y else None
    _load().oracle_rmsnorm_quant(_p(x), _p(g), M, H, H, float(eps), _p(q), _p(s), lds,
                                 _p(y) if want_y else None)
    return (q, s, y) if want_y else (q, s)


def swiglu_quant(gu, lds: int | None = None, want_h: bool = False):
    """a4: gu BF16 [M, 2I] (gate | up) -> SwiGLU BF16 h [M,I] -> 1x128 quantization."""
    gu = _bf16(gu)
    M, I2 = gu.shape
    I = I2 // 2
    assert I2 % 2 == 0
    lds = _lds_for(M) if lds is None else lds
    q = np.zeros((M, I), np.uint8)
    s = np.zeros((groups(I), lds), np.float32)
    h = np.zeros((M, I), np.uint16) if want_h else None
    _load().oracle_swiglu_quant(_p(gu), M, I, I2, _p(q), _p(s), lds,
                                _p(h) if want_h else None)
    return (q, s, h) if want_h else (q, s)


def transpose_quant_bf16(dy, lds_row: int | None = None, want_row: bool = True):
    """a6: dY BF16 [M,N] -> row-wise 1x128 (q_row [M,N], s_row [N/128, lds_row]) and
    column-wise 128x1 transposed (q_colT [N,M], s_col [M/128, N])."""
    dy = _bf16(dy)
    M, N = dy.shape
    lds_row = _lds_for(M) if lds_row is None else lds_row
    q_row = np.zeros((M, N), np.uint8) if want_row else None
    s_row = np.zeros((groups(N), lds_row), np.float32) if want_row else None
    q_colT = np.zeros((N, M), np.uint8)
    s_col = np.zeros((groups(M), N), np.float32)
    _load().oracle_transpose_quant_bf16(
        _p(dy), M, N, N, _p(q_row) if want_row else None,
        _p(s_row) if want_row else None, lds_row, _p(q_colT), _p(s_col))
    return q_row, s_row, q_colT, s_col


def rmsnorm_quant_dual(x, gamma, eps: float, lds_row: int | None = None):
    """Saved activations in both groupings from BF16 ("option B" for the RMSNorm producer:
    no FP8 requantization): y = RMSNorm(x) * gamma rounded to BF16 as in rmsnorm_quant, then y
    quantized 1x128 along rows (forward) and 128x1 along columns, stored transposed
    (WGrad), plus the per-row reciprocal RMS r. Returns (q_row, s_row, q_colT, s_col, r)."""
    x = _bf16(x)
    q, s, y = rmsnorm_quant(x, gamma, eps, lds_row, want_y=True)
    _, _, qT, sT = transpose_quant_bf16(y, want_row=False)
    r = np.array([rmsnorm_rstd(row, eps) for row in x], np.float32)
    return q, s, qT, sT, r


def swiglu_quant_dual(gu, lds_row: int | None = None):
    """Option B for the SwiGLU producer: h = SwiGLU(gate, up) in BF16 as in swiglu_quant,
    then h quantized 1x128 along rows and 128x1 along columns (transposed).
    Returns (q_row, s_row, q_colT, s_col)."""
    q, s, h = swiglu_quant(gu, lds_row, want_h=True)
    _, _, qT, sT = transpose_quant_bf16(h, want_row=False)
    return q, s, qT, sT


def swiglu_bwd_one(gate_bits: int, up_bits: int, dh_bits: int) -> tuple[int, int]:
    """Backward of one SwiGLU element: (d_gate, d_up) BF16 bits."""
    dg, du = ctypes.c_uint16(0), ctypes.c_uint16(0)
    _load().oracle_swiglu_bwd_one(int(gate_bits), int(up_bits), int(dh_bits),
                                  ctypes.byref(dg), ctypes.byref(du))
    return int(dg.value), int(du.value)


def swiglu_bwd(gu, dh) -> np.ndarray:
    """SwiGLU backward in BF16: gu [M, 2I] (gate | up), dh [M, I] -> dgu [M, 2I]
    (d_gate | d_up), the rounding sequence of oracle_swiglu_bwd_one."""
    gu, dh = _bf16(gu), _bf16(dh)
    M, I2 = gu.shape
    I = I2 // 2
    assert I2 % 2 == 0 and dh.shape == (M, I)
    dgu = np.zeros((M, I2), np.uint16)
    _load().oracle_swiglu_bwd(_p(gu), _p(dh), M, I, _p(dgu))
    return dgu


def swiglu_bwd_dual(gu, dh, lds_row: int | None = None):
    """The SwiGLU backward with the gradient quantizer a6 fused behind it: dgu (BF16)
    quantized 1x128 along rows (DGrad of the gate/up projection) and 128x1 along columns,
    stored transposed (its WGrad). Returns (q_row, s_row, q_colT, s_col, dgu)."""
    dgu = swiglu_bwd(gu, dh)
    q, s, qT, sT = transpose_quant_bf16(dgu, lds_row)
    return q, s, qT, sT, dgu


def exact_sum_f32(t, to_f32: bool = False) -> float:
    """The exact sum of the fp32 values t, rounded once: to the nearest double, or (to_f32)
    to the nearest fp32 (returned as a Python float). The reductions of rmsnorm_bwd."""
    a = np.ascontiguousarray(np.asarray(t, dtype=np.float32))
    return float(_load().oracle_exact_sum_f32(_p(a), a.size, 1 if to_f32 else 0))


def rmsnorm_bwd(x, gamma, dy, dres, eps: float):
    """RMSNorm backward in BF16 plus the residual gradient: x, dy, dres [M, H] BF16
    (dres may be None), gamma [H]. Returns (out [M, H] BF16 bits, dgamma [H] fp32,
    r [M] fp32, k [M] fp32) with the rounding sequence of oracle_rmsnorm_bwd."""
    x, dy, g = _bf16(x), _bf16(dy), _bf16(gamma)
    M, H = x.shape
    assert dy.shape == (M, H) and g.shape == (H,)
    dr = None if dres is None else _bf16(dres)
    assert dr is None or dr.shape == (M, H)
    out = np.zeros((M, H), np.uint16)
    dgamma = np.zeros(H, np.float32)
    r = np.zeros(M, np.float32)
    k = np.zeros(M, np.float32)
    _load().oracle_rmsnorm_bwd(_p(x), _p(g), _p(dy), None if dr is None else _p(dr), M, H,
                               float(eps), _p(out), _p(dgamma), _p(r), _p(k))
    return out, dgamma, r, k


def rmsnorm_bwd_dual(x, gamma, dy, dres, eps: float, lds_row: int | None = None):
    """The RMSNorm backward (+ residual gradient) with a6 fused behind it: out (BF16)
    and its 1x128 row codes and 128x1 transposed column codes. Returns
    (out, q_row, s_row, q_colT, s_col, dgamma)."""
    out, dgamma, _, _ = rmsnorm_bwd(x, gamma, dy, dres, eps)
    q, s, qT, sT = transpose_quant_bf16(out, lds_row)
    return out, q, s, qT, sT, dgamma


def transpose_quant_fp8(q, s):
    """a8: saved FP8 activation (q [M,K], s [K/128, lds]) -> 128x1 requantized,
    transposed (qT [K,M], sT [M/128, K])."""
    q = np.ascontiguousarray(q, dtype=np.uint8)
    s = np.ascontiguousarray(s, dtype=np.float32)
    M, K = q.shape
    assert s.shape[0] == groups(K)
    qT = np.zeros((K, M), np.uint8)
    sT = np.zeros((groups(M), K), np.float32)
    _load().oracle_transpose_quant_fp8(_p(q), _p(s), M, K, s.shape[1], _p(qT), _p(sT))
    return qT, sT


# --------------------------------------------------------------------------
# Exact dequantization and the fp64 GEMMs
# --------------------------------------------------------------------------

def dequant_rows(q, s, r0: int = 0, nr: int | None = None) -> np.ndarray:
    """Rows scaled per 1x128 group: out[i,k] = s[k//128, r0+i] * dec(q[r0+i,k]) (fp64)."""
    q = np.ascontiguousarray(q, dtype=np.uint8)
    s = np.ascontiguousarray(s, dtype=np.float32)
    R, K = q.shape
    nr = R - r0 if nr is None else nr
    out = np.empty((nr, K), np.float64)
    _load().oracle_dequant_rows(_p(q), _p(s), R, K, s.shape[1], r0, nr, _p(out))
    return out


def dequant_block(q, s, r0: int = 0, nr: int | None = None) -> np.ndarray:
    """128x128 blocks: out[i,k] = s[(r0+i)//128, k//128] * dec(q[r0+i,k]) (fp64)."""
    q = np.ascontiguousarray(q, dtype=np.uint8)
    s = np.ascontiguousarray(s, dtype=np.float32)
    N, K = q.shape
    nr = N - r0 if nr is None else nr
    out = np.empty((nr, K), np.float64)
    _load().oracle_dequant_block(_p(q), _p(s), N, K, r0, nr, _p(out))
    return out


def dequant_cols(qT, sT, c0: int = 0, nc: int | None = None) -> np.ndarray:
    """128x1 groups stored transposed (qT [C,R], sT [R/128, C]):
    out[i,r] = sT[r//128, c0+i] * dec(qT[c0+i, r]) (fp64)."""
    qT = np.ascontiguousarray(qT, dtype=np.uint8)
    sT = np.ascontiguousarray(sT, dtype=np.float32)
    C, R = qT.shape
    nc = C - c0 if nc is None else nc
    out = np.empty((nc, R), np.float64)
    _load().oracle_dequant_cols(_p(qT), _p(sT), C, R, c0, nc, _p(out))
    return out


def gemm_nt(a: np.ndarray, b: np.ndarray):
    """out[i,j] = sum_k a[i,k] * b[j,k] in fp64, and the magnitude sum_k |a b|."""
    return a @ b.T, np.abs(a) @ np.abs(b).T


def linear_fwd(qa, sa, qw, sw, rows=None):
    """a5: Y[m,n] = sum_k sa*sw * qa[m,k]*qw[n,k], exact operands, fp64 dot.
    "Arquitectura Central": the training forward and the rollout share this GEMM.
    rows: optional (r0, nr) slab of output rows."""
    r0, nr = (0, qa.shape[0]) if rows is None else rows
    A = dequant_rows(qa, sa, r0, nr)
    B = dequant_block(qw, sw)
    return gemm_nt(A, B)


def linear_dgrad(qdy, sdy, qw, sw, rows=None):
    """a7: dX[m,k] = sum_n sdy*sw * qdy[m,n]*qw[n,k] ("Esquema de Cuantización",
    DGrad in FP8). Uses W in its stored [N,K] orientation."""
    r0, nr = (0, qdy.shape[0]) if rows is None else rows
    A = dequant_rows(qdy, sdy, r0, nr)          # [nr, N]
    W = dequant_block(qw, sw)                   # [N, K]
    return A @ W, np.abs(A) @ np.abs(W)


def linear_wgrad(qdyT, sdy_c, qxT, sx_c, rows=None):
    """a9: dW[n,k] = sum_m sdy_c[m/128,n]*sx_c[m/128,k] * qdyT[n,m]*qxT[k,m]
    ("Esquema de Cuantización": WGrad in FP8 with 1x128 / 128x1 grouping; both
    operands grouped along the reduction dimension M)."""
    r0, nr = (0, qdyT.shape[0]) if rows is None else rows
    A = dequant_cols(qdyT, sdy_c, r0, nr)       # [nr, M]
    B = dequant_cols(qxT, sx_c)                 # [K, M]
    return gemm_nt(A, B)


def bf16_ulp(v: np.ndarray) -> np.ndarray:
    """One BF16 ulp at |v|: 2^(floor(log2|v|) - 7); 0 where v == 0."""
    v = np.abs(np.asarray(v, np.float64))
    out = np.zeros_like(v)
    nz = v > 0
    out[nz] = np.exp2(np.floor(np.log2(v[nz])) - 7)
    return out
