"""The C-ABI library builds, loads and exports every entry point include/fp8q.h declares;
argument validation happens on the host, before any CUDA call (no GPU needed)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", fn)).read()
            txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
            names += re.findall(r"\b(fp8q_[a-z0-9_]+)\s*\(", txt)
    return sorted(set(names))


def build_module():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "fp8q_build", os.path.join(ROOT, "fp8_block_scaled_08_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.fixture(scope="module", autouse=True)
def lib():
    path = build_module().build()
    return ctypes.CDLL(path)


def test_header_declares_the_hot_path():
    names = header_functions()
    for n in ["fp8q_quant_act_1x128", "fp8q_quant_weight_128x128", "fp8q_rmsnorm_quant",
              "fp8q_swiglu_quant", "fp8q_transpose_quant_bf16", "fp8q_transpose_quant_fp8",
              "fp8q_linear_fwd", "fp8q_linear_dgrad", "fp8q_linear_wgrad"]:
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", build_module().LIB], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (fp8q_[a-z0-9_]+)$", out, flags=re.M))
    missing = [n for n in header_functions() if n not in exported]
    assert not missing, missing
    for n in header_functions():
        getattr(lib, n)


def test_binding_covers_every_symbol():
    import fp8_block_scaled_08_b200 as f
    assert set(header_functions()) == set(f.EXPORTED)


def test_status_strings_and_version():
    import fp8_block_scaled_08_b200 as f
    assert f.version() >= 10000
    for code in range(7):
        assert f.status_string(code).startswith("FP8Q_")
    assert "UNKNOWN" in f.status_string(99)


# Host-side validation: fake (never dereferenced) device addresses, 16-byte aligned.
A = ctypes.c_void_p(0x10000)
B = ctypes.c_void_p(0x20000)
C = ctypes.c_void_p(0x30000)
D = ctypes.c_void_p(0x40000)
E = ctypes.c_void_p(0x50000)
ODD = ctypes.c_void_p(0x10008)
NUL = None


def call(name, *args):
    import fp8_block_scaled_08_b200 as f
    return getattr(f._lib, name)(*args)


def test_validation_act_quant():
    f = "fp8q_quant_act_1x128"
    assert call(f, NUL, 8, 128, 128, B, C, 8, NUL) == 1
    assert call(f, A, 8, 100, 128, B, C, 8, NUL) == 2        # K % 16
    assert call(f, A, 0, 128, 128, B, C, 8, NUL) == 2        # M <= 0
    assert call(f, A, 8, 128, 128, B, C, 6, NUL) == 2        # lds % 4
    assert call(f, A, 8, 128, 128, B, C, 4, NUL) == 2        # lds < M
    assert call(f, A, 8, 256, 128, B, C, 8, NUL) == 2        # ldx < K
    assert call(f, ODD, 8, 128, 128, B, C, 8, NUL) == 3      # misaligned
    assert call(f, A, 8, 128, 132, B, C, 8, NUL) == 3        # ldx % 8


def test_validation_gemms():
    assert call("fp8q_linear_fwd", A, B, 16, C, D, 16, 200, 128, E, 256, NUL) == 2   # N % 16
    assert call("fp8q_linear_fwd", A, B, 16, C, D, 16, 256, 100, E, 256, NUL) == 2   # K % 16
    assert call("fp8q_linear_fwd", A, B, 8, C, D, 16, 256, 128, E, 256, NUL) == 2    # ldsa < M
    assert call("fp8q_linear_fwd", A, B, 16, C, D, 16, 256, 128, E, 250, NUL) == 2   # ldy < N
    assert call("fp8q_linear_fwd", A, B, 16, C, D, 16, 256, 128, E, 260, NUL) == 3   # ldy % 8
    assert call("fp8q_linear_fwd", A, NUL, 16, C, D, 16, 256, 128, E, 256, NUL) == 1
    assert call("fp8q_linear_dgrad", A, B, 16, C, D, 16, 256, 200, E, 256, NUL) == 2
    assert call("fp8q_linear_wgrad", A, B, C, D, 100, 256, 256, E, 256, NUL) == 2    # M % 16
    assert call("fp8q_linear_wgrad", A, B, C, D, 128, 256, 256, ODD, 256, NUL) == 3


def test_validation_splitk():
    f = "fp8q_linear_fwd_splitk"
    W = ctypes.c_void_p(0x10000)
    assert call(f, A, B, 16, C, D, 200, 256, 128, E, 256, W, 1 << 20, NUL) == 2    # M > 128
    assert call(f, A, B, 16, C, D, 16, 200, 128, E, 256, W, 1 << 20, NUL) == 2    # N % 128
    assert call(f, A, B, 16, C, D, 16, 256, 100, E, 256, W, 1 << 20, NUL) == 2    # K % 128
    assert call(f, A, B, 16, C, D, 16, 256, 128, E, 260, W, 1 << 20, NUL) == 3    # ldy % 8
    assert call(f, NUL, B, 16, C, D, 16, 256, 128, E, 256, W, 1 << 20, NUL) == 1


def test_splitk_workspace_sizes():
    import fp8_block_scaled_08_b200 as f
    # counters: one word per 64-column strip, padded to 256 bytes; partials: one fp32 per
    # (output column, K slice, token row)
    assert f._lib.fp8q_linear_fwd_splitk_counter_bytes(16, 4096) == 256
    assert f._lib.fp8q_linear_fwd_splitk_counter_bytes(16, 24576) == 1536
    assert f._lib.fp8q_linear_fwd_splitk_workspace(16, 4096, 4096) == 256 + 4096 * 32 * 16 * 4
    assert f.linear_fwd_splitk_workspace_bytes(1, 128, 256) == 256 + 128 * 2 * 1 * 4
    assert f._lib.fp8q_linear_fwd_splitk_workspace(129, 4096, 4096) == 0
    assert f._lib.fp8q_linear_fwd_splitk_workspace(16, 100, 4096) == 0


def test_validation_tile_quantizers():
    assert call("fp8q_transpose_quant_bf16", A, 100, 128, 128, B, C, 128, D, E, NUL) == 2
    assert call("fp8q_transpose_quant_bf16", A, 128, 128, 128, B, NUL, 128, D, E, NUL) == 1
    assert call("fp8q_transpose_quant_fp8", A, B, 128, 100, 128, C, D, NUL) == 2
    assert call("fp8q_quant_weight_128x128", A, 100, 128, 128, B, C, NUL, NUL) == 2
    assert call("fp8q_rmsnorm_quant", A, B, 4, 128, 128, ctypes.c_float(-1.0), C, D, 4, NUL) == 2
    assert call("fp8q_rmsnorm_quant", A, B, 4, 32768, 32768, ctypes.c_float(1e-5), C, D, 4, NUL) == 2
    assert call("fp8q_swiglu_quant", A, 4, 128, 200, B, C, 4, NUL) == 2   # ldgu < 2I
    assert call("fp8q_debug_wait_timeout", 0, NUL) == 2


def test_validation_backward_producers():
    W = ctypes.c_void_p(0x10000)
    F = ctypes.c_float
    f = "fp8q_swiglu_bwd_quant_dual"
    assert call(f, A, B, 100, 128, NUL, C, D, 128, E, A, NUL) == 2               # M % 128
    assert call(f, A, B, 128, 100, NUL, C, D, 128, E, A, NUL) == 2               # I % 128
    assert call(f, A, B, 128, 128, NUL, C, D, 126, E, A, NUL) == 2               # lds_row < M
    assert call(f, NUL, B, 128, 128, NUL, C, D, 128, E, A, NUL) == 1
    assert call(f, A, B, 128, 128, ctypes.c_void_p(0x10008), C, D, 128, E, A, NUL) == 3
    g = "fp8q_rmsnorm_bwd_quant_dual"
    need = call("fp8q_rmsnorm_bwd_workspace_bytes", 256, 512)
    assert need == 2048 + 512 * 16 * 8                                  # r, k, dgamma's bins
    assert call("fp8q_rmsnorm_bwd_workspace_bytes", 100, 512) == -1
    assert call("fp8q_rmsnorm_bwd_workspace_bytes", (1 << 23) + 128, 512) == -1   # M too large
    assert call("fp8q_rmsnorm_bwd_workspace_bytes", 256, (1 << 19) + 128) == -1   # H too large
    assert call("fp8q_rmsnorm_bwd_workspace_bytes", 256, 1 << 19) > 0
    ok = (A, B, C, NUL, 256, 512, F(1e-5), D, E, A, 256, B, C, NUL, W)
    assert call(g, *ok, need - 1, NUL) == 2                                        # workspace
    assert call(g, A, B, C, NUL, 256, 512, F(-1.0), D, E, A, 256, B, C, NUL, W, need, NUL) == 2
    assert call(g, A, B, C, NUL, 256, 500, F(1e-5), D, E, A, 256, B, C, NUL, W, need, NUL) == 2
    assert call(g, A, B, C, NUL, 256, 512, F(1e-5), NUL, E, A, 256, B, C, NUL, W, need, NUL) == 1
    assert call(g, A, B, C, ctypes.c_void_p(0x10004), 256, 512, F(1e-5), D, E, A, 256, B, C, NUL,
                W, need, NUL) == 3                                                 # dres align


def test_validation_wgrad_acc_f32():
    f = "fp8q_linear_wgrad_acc_f32"
    assert call(f, A, B, C, D, 100, 128, 128, E, 128, NUL) == 2       # M % 16
    assert call(f, A, B, C, D, 128, 128, 100, E, 128, NUL) == 2       # K % 16
    assert call(f, A, B, C, D, 128, 128, 128, E, 126, NUL) == 2       # lddw < K
    assert call(f, A, B, C, D, 128, 128, 256, E, 258, NUL) == 3       # lddw % 4
    assert call(f, A, B, C, NUL, 128, 128, 128, E, 128, NUL) == 1


def test_binding_fails_loudly_without_the_library(tmp_path):
    """No fallback: a copy of the package without libfp8q.so refuses to import."""
    import shutil
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    pkg = os.path.join(root, "fp8_block_scaled_08_b200")
    dst = tmp_path / "fp8_block_scaled_08_b200"
    dst.mkdir()
    for name in os.listdir(pkg):
        if name.endswith(".py"):
            shutil.copy(os.path.join(pkg, name), dst / name)
    r = subprocess.run([sys.executable, "-c", "import fp8_block_scaled_08_b200"],
                       cwd=str(tmp_path), capture_output=True, text=True, timeout=300)
    assert r.returncode != 0
    assert "ImportError" in r.stderr and "libfp8q.so is not built" in r.stderr
