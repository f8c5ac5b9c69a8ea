"""Mutation check of the oracle's pins. Each case copies oracle/fp8q_oracle.c, plants one
plausible mistake (a dropped term or factor, a wrong constant, sign, index or rounding
rule, a swapped operand), builds the copy with the oracle's own flags, and runs the pin
files that cover that function in a subprocess whose oracle loader uses the copy
(FP8Q_ORACLE_LIB): at least one pin must fail. An unaltered copy, built and run the
same way, must pass them all — so a failure is the mistake's doing, not the harness's."""
import os
import subprocess
import sys

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "fp8q_oracle.c")

E4M3, QUANT = "tests/test_oracle_e4m3.py", "tests/test_oracle_quant.py"
NORM, BWD = "tests/test_oracle_norm_swiglu.py", "tests/test_oracle_backward.py"
GEMM = "tests/test_oracle_gemm.py"
TAILS = "tests/test_oracle_tails.py"

# (name, exact text in fp8q_oracle.c, replacement, pin files that must catch it)
MUTANTS = [
    ("e4m3 ties round up",
     "else pick = (lo & 1) ? up : lo; /* tie: even mantissa",
     "else pick = up; /* tie: even mantissa", [E4M3]),
    ("scale = amax / 240",
     "volatile float s = amax / 448.0f;", "volatile float s = amax / 240.0f;", [QUANT]),
    ("rmsnorm without eps",
     "double r = 1.0 / sqrt(ms + (double)eps);", "double r = 1.0 / sqrt(ms);", [NORM]),
    ("rmsnorm without gamma",
     "volatile float t2 = t1 * oracle_bf16_to_f32(gamma[c]);", "volatile float t2 = t1;", [NORM]),
    ("swiglu gate and up swapped",
     "oracle_swiglu_one(gu[m * ldgu + c], gu[m * ldgu + I + c])",
     "oracle_swiglu_one(gu[m * ldgu + I + c], gu[m * ldgu + c])", [NORM]),
    ("exp: 1/6 coefficient rounded",
     "const float C3 = 0x1.555556p-3f;", "const float C3 = 0x1.5p-3f;", [NORM]),
    ("swiglu backward without 1 + g(1 - sig)",
     "volatile float t3 = 1.0f + t2;", "volatile float t3 = 1.0f;", [BWD]),
    ("swiglu backward sig = g / d",
     "volatile float sig = 1.0f / d;", "volatile float sig = g / d;", [BWD]),
    ("rmsnorm backward k with r^2",
     "    kd = kd * (double)r;\n    kd = kd * (double)r;\n", "    kd = kd * (double)r;\n", [BWD]),
    ("rmsnorm backward without the residual",
     "oracle_bf16_to_f32(dxb) + oracle_bf16_to_f32(dres[m * H + j]);",
     "oracle_bf16_to_f32(dxb);", [BWD]),
    ("dgamma without r",
     "volatile float xr = oracle_bf16_to_f32(x[m * H + j]) * rr[m];",
     "volatile float xr = oracle_bf16_to_f32(x[m * H + j]);", [BWD]),
    ("exact sum without the carry between words",
     "uint64_t v = (uint64_t)a->w[i] + term[i] + c;", "uint64_t v = (uint64_t)a->w[i] + term[i];",
     [BWD]),
    ("exact sum loses its sticky bits",
     "for (int i = p - 54; i >= 0; --i) sticky |= xacc_bit(mag, i);",
     "for (int i = p - 54; i >= 0 && 0; --i) sticky |= xacc_bit(mag, i);", [BWD]),
    ("fp32 reduction rounded through a double",
     "{ return (float)xacc_round(a, 1); }", "{ return (float)xacc_round(a, 0); }", [BWD]),
    ("partial group drops its last element",
     "static int gwidth(i64 n, i64 g) { return n - g * 128 < 128 ? (int)(n - g * 128) : 128; }",
     "static int gwidth(i64 n, i64 g) { return n - g * 128 < 128 ? (int)(n - g * 128) - 1 : 128; }",
     [TAILS]),
    ("partial group count rounded down",
     "static i64 ngroups(i64 n) { return (n + 127) / 128; }",
     "static i64 ngroups(i64 n) { return n / 128; }", [TAILS]),
    ("128x1 column group rows mis-indexed",
     "dy[(mb * 128 + i) * lddy + n]", "dy[(mb + i) * lddy + n]", [QUANT]),
    ("requantizer drops the row scale",
     "volatile float v = s[(k / 128) * lds + m] * dec;", "volatile float v = dec;", [QUANT]),
    ("weight block scale transposed",
     "s[((r0 + i) / 128) * KB + k / 128]", "s[(k / 128) * KB + (r0 + i) / 128]", [GEMM]),
]

# The same for the definitions in oracle/__init__.py (the numpy GEMMs and the dual /
# backward compositions): the module's source, with the mistake, is executed again in
# the module's own namespace before the pins run.
PY_SRC = os.path.join(ROOT, "oracle", "__init__.py")
PY_MUTANTS = [
    ("forward without the activation scale",
     "A = dequant_rows(qa, sa, r0, nr)", "A = dequant_rows(qa, np.ones_like(sa), r0, nr)", [GEMM]),
    ("DGrad against the reversed weight rows",
     "return A @ W, np.abs(A) @ np.abs(W)", "return A @ W[::-1], np.abs(A) @ np.abs(W)", [GEMM]),
    ("WGrad with the X operand's scales doubled",
     "B = dequant_cols(qxT, sx_c)                 # [K, M]",
     "B = dequant_cols(qxT, sx_c * 2)             # [K, M]", [GEMM]),
    ("GEMM without the transposed operand",
     "return a @ b.T, np.abs(a) @ np.abs(b).T", "return a @ b[::-1].T, np.abs(a) @ np.abs(b).T",
     [GEMM]),
    ("RMSNorm dual emission quantizes x instead of y",
     "_, _, qT, sT = transpose_quant_bf16(y, want_row=False)",
     "_, _, qT, sT = transpose_quant_bf16(x, want_row=False)", [NORM]),
    ("SwiGLU dual emission quantizes the gate instead of h",
     "_, _, qT, sT = transpose_quant_bf16(h, want_row=False)",
     "_, _, qT, sT = transpose_quant_bf16(_bf16(gu)[:, :h.shape[1]], want_row=False)", [NORM]),
    ("SwiGLU backward quantizes gu instead of its gradient",
     "q, s, qT, sT = transpose_quant_bf16(dgu, lds_row)",
     "q, s, qT, sT = transpose_quant_bf16(_bf16(gu), lds_row)", [BWD]),
    ("RMSNorm backward quantizes dy instead of its output",
     "q, s, qT, sT = transpose_quant_bf16(out, lds_row)",
     "q, s, qT, sT = transpose_quant_bf16(_bf16(dy), lds_row)", [BWD]),
]

_PY_RUNNER = """
import sys
sys.path.insert(0, {root!r})
import numpy as np
import pytest
import oracle
src = open({src!r}).read()
assert src.count({old!r}) == 1, "mutation site not unique"
oracle._lib = None
exec(compile(src.replace({old!r}, {new!r}), {src!r}, "exec"), oracle.__dict__)
sys.exit(pytest.main({files!r} + ["-x", "-q", "-m", "not gpu", "-p", "no:cacheprovider"]))
"""


_JOBS = 8                       # subprocesses at a time
_ENV = dict(os.environ, OMP_NUM_THREADS="2")


def _build_copy(tmp_path, name, text):
    src = tmp_path / (name + ".c")
    src.write_text(text)
    lib = tmp_path / (name + ".so")
    subprocess.check_call(["gcc", *oracle.GCC_FLAGS, str(src), "-o", str(lib), "-lm"])
    return str(lib)


def _run_pins(lib, files):
    env = dict(_ENV, FP8Q_ORACLE_LIB=lib)
    r = subprocess.run([sys.executable, "-m", "pytest", *files, "-x", "-q", "-m", "not gpu",
                        "-p", "no:cacheprovider"], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=600)
    return r.returncode, r.stdout[-2000:]


@pytest.fixture(scope="module")
def c_results(tmp_path_factory):
    """Builds the unaltered copy and every C mutant, runs their pin files concurrently:
    {name: (return code, output tail)} ("" is the unaltered copy)."""
    from concurrent.futures import ThreadPoolExecutor
    tmp = tmp_path_factory.mktemp("c_mutants")
    with open(SRC) as f:
        text = f.read()
    jobs = {"": (text, [E4M3, QUANT, NORM, BWD])}
    for i, (name, old, new, files) in enumerate(MUTANTS):
        assert text.count(old) == 1, "mutation site not unique: %r" % old
        jobs[name] = (text.replace(old, new), files)

    def run(item):
        name, (src, files) = item
        lib = _build_copy(tmp, "m%d" % abs(hash(name)), src)
        return name, _run_pins(lib, files)

    with ThreadPoolExecutor(_JOBS) as ex:
        return dict(ex.map(run, jobs.items()))


def test_unaltered_copy_passes_every_pin_file(c_results):
    code, out = c_results[""]
    assert code == 0, out


@pytest.mark.parametrize("name", [m[0] for m in MUTANTS])
def test_planted_mistake_fails_a_pin(c_results, name):
    code, out = c_results[name]
    assert code != 0, "no pin caught the mistake %r:\n%s" % (name, out)


def _run_py(old, new, files):
    code = _PY_RUNNER.format(root=ROOT, src=PY_SRC, old=old, new=new, files=files)
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True,
                       timeout=600, env=_ENV)
    return r.returncode, r.stdout[-2000:] + r.stderr[-1000:]


@pytest.fixture(scope="module")
def py_results():
    """Runs the unaltered module (a no-op replacement) and every Python mutant
    concurrently: {name: (return code, output tail)}."""
    from concurrent.futures import ThreadPoolExecutor
    jobs = {"": ("def gemm_nt(", "def gemm_nt(", [GEMM, NORM, BWD])}
    for name, old, new, files in PY_MUTANTS:
        jobs[name] = (old, new, files)
    with ThreadPoolExecutor(_JOBS) as ex:
        return dict(ex.map(lambda kv: (kv[0], _run_py(*kv[1])), jobs.items()))


def test_unaltered_module_passes_the_pins(py_results):
    code, out = py_results[""]
    assert code == 0, out


@pytest.mark.parametrize("name", [m[0] for m in PY_MUTANTS])
def test_planted_python_mistake_fails_a_pin(py_results, name):
    code, out = py_results[name]
    assert code != 0, "no pin caught the mistake %r:\n%s" % (name, out)
