"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of oracle/fp8_oracle.c (a dropped term,
a wrong sign, a swapped index, a transposed operand, a wrong rounding rule),
builds the copy with gcc into a temporary library, and runs pin checks of the
kind tests/test_oracle_*.py use against it: at least one check must fail.  The
unmutated source must pass the same checks, so the harness itself is sound.
CPU only; nothing here touches the CUDA library."""
import ctypes
import math
import os
import subprocess
import tempfile
from fractions import Fraction

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "fp8_oracle.c")


def _build(source, tmpdir, name):
    c = os.path.join(tmpdir, name + ".c")
    so = os.path.join(tmpdir, name + ".so")
    with open(c, "w") as f:
        f.write(source)
    subprocess.run(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-fno-fast-math", c, "-o", so,
                    "-lm"], check=True)
    L = ctypes.CDLL(so)
    L.oracle_fp8_decode.restype = ctypes.c_double
    L.oracle_fp8_decode.argtypes = [ctypes.c_uint8, ctypes.c_int]
    L.oracle_fp8_encode.restype = ctypes.c_uint8
    L.oracle_fp8_encode.argtypes = [ctypes.c_double, ctypes.c_int, ctypes.c_int]
    L.oracle_compute_bias.restype = ctypes.c_int32
    L.oracle_compute_bias.argtypes = [ctypes.c_float, ctypes.c_int, ctypes.c_int]
    L.oracle_amax_f32.restype = ctypes.c_float
    L.oracle_amax_f32.argtypes = [ctypes.c_void_p, ctypes.c_size_t]
    L.oracle_linear_full.restype = None
    L.oracle_linear_full.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_int, ctypes.c_int32,
                                     ctypes.c_void_p, ctypes.c_int, ctypes.c_int32, ctypes.c_int64,
                                     ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
                                     ctypes.c_void_p]
    return L


# --- pin checks (independent restatements, as in the pin tests) -------------

def _decode_ref(code, fmt):
    """The OCP definitions, written out again for the check."""
    s = -1.0 if code & 0x80 else 1.0
    if fmt == 0:
        e, m = (code >> 3) & 0xF, code & 7
        if e == 15 and m == 7:
            return math.nan
        return s * (m / 8 * 2.0 ** -6 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7))
    e, m = (code >> 2) & 0x1F, code & 3
    if e == 31:
        return s * math.inf if m == 0 else math.nan
    return s * (m / 4 * 2.0 ** -14 if e == 0 else (1 + m / 4) * 2.0 ** (e - 15))


def _pins_codec(L):
    for fmt in (0, 1):
        for c in range(256):
            want = _decode_ref(c, fmt)
            got = L.oracle_fp8_decode(c, fmt)
            if math.isnan(want) != math.isnan(got) or (not math.isnan(want) and want != got):
                return False
        # round trip of finite codes, ties to even, saturation
        for c in range(256):
            v = _decode_ref(c, fmt)
            if math.isfinite(v) and L.oracle_fp8_encode(v, fmt, 1) != c:
                return False
    if L.oracle_fp8_encode(2.0 ** -10, 0, 1) != 0 or L.oracle_fp8_encode(3 * 2.0 ** -10, 0, 1) != 2:
        return False
    if L.oracle_fp8_encode(1e6, 0, 1) != 0x7E or L.oracle_fp8_encode(-1e6, 1, 1) != 0xFB:
        return False
    return True


def _pins_bias(L):
    rng = np.random.default_rng(0)
    for fmt, fm in ((0, 448), (1, 57344)):
        for bits in rng.integers(1, 0x7F800000, 300, dtype=np.uint32):
            a = float(np.array([bits], np.uint32).view(np.float32)[0])
            for margin in (0, 3):
                want = max(b for b in range(-300, 301) if Fraction(a) * Fraction(2) ** b <= fm)
                if L.oracle_compute_bias(a, fmt, margin) != want - margin:
                    return False
        if L.oracle_compute_bias(0.0, fmt, 3) != 0:
            return False
    return True


def _pins_amax(L):
    x = np.array([1.0, -7.5, np.nan, 3.0], dtype=np.float32)
    if not math.isnan(L.oracle_amax_f32(x.ctypes.data, 4)):
        return False
    x = np.array([1.0, -7.5, 3.0], dtype=np.float32)
    return L.oracle_amax_f32(x.ctypes.data, 3) == 7.5


def _pins_gemm(L):
    rng = np.random.default_rng(1)
    T, In, Out = 3, 5, 4
    fin = lambda fmt: np.array([c for c in range(256) if math.isfinite(_decode_ref(c, fmt))],
                               dtype=np.uint8)
    X = rng.choice(fin(0), (T, In))
    W = rng.choice(fin(0), (Out, In))
    dY = rng.choice(fin(1), (T, Out))
    d = lambda c, f: Fraction(_decode_ref(int(c), f))
    cases = [(0, X, 0, W, 0, (T, Out), lambda r, c: sum(d(X[r, i], 0) * d(W[c, i], 0) for i in range(In))),
             (1, dY, 1, W, 0, (T, In), lambda r, c: sum(d(dY[r, o], 1) * d(W[o, c], 0) for o in range(Out))),
             (2, dY, 1, X, 0, (Out, In), lambda r, c: sum(d(dY[t, r], 1) * d(X[t, c], 0) for t in range(T)))]
    for p, A, fa, B, fb, shape, f in cases:
        A = np.ascontiguousarray(A, np.uint8)
        B = np.ascontiguousarray(B, np.uint8)
        val = np.empty(shape, np.float64)
        L.oracle_linear_full(p, A.ctypes.data, fa, 3, B.ctypes.data, fb, -1, T, In, Out,
                             val.ctypes.data, None)
        for r in range(shape[0]):
            for c in range(shape[1]):
                if Fraction(val[r, c]) != f(r, c) * Fraction(2) ** -2:
                    return False
    return True


def _all_pins(L):
    return _pins_codec(L) and _pins_bias(L) and _pins_amax(L) and _pins_gemm(L)


MUTATIONS = {
    "bias_round_instead_of_floor": ("(int32_t)floor(log2(ratio))", "(int32_t)round(log2(ratio))"),
    "bias_margin_added": ("floor(log2(ratio)) - margin", "floor(log2(ratio)) + margin"),
    "bias_zero_amax_keeps_margin": ("if (!(amax > 0.0f) || isinf(amax)) return 0;",
                                    "if (isnan(amax) || isinf(amax)) return 0;\n    if (amax == 0.0f) return -margin;"),
    "encode_ties_to_odd": ("code = (lo % 2 == 0) ? lo : lo + 1;", "code = (lo % 2 == 1) ? lo : lo + 1;"),
    "encode_ties_down": ("code = (lo % 2 == 0) ? lo : lo + 1;", "code = lo;"),
    "encode_no_saturation": ("if (saturate) return (uint8_t)(sign | max_finite_code(fmt));",
                             "if (0) return 0;"),
    "decode_e4m3_bias_8": ("int ebias = (fmt == FMT_E4M3) ? 7 : 15;", "int ebias = (fmt == FMT_E4M3) ? 8 : 15;"),
    "decode_no_subnormals": ("mag = ldexp((double)mfield, 1 - ebias - mbits);", "mag = 0.0;"),
    "amax_ignores_nan": ("return saw_nan ? NAN : m;\n}\n\nfloat oracle_amax_bf16",
                         "return m;\n}\n\nfloat oracle_amax_bf16"),
    "gemm_unscale_sign": ("int32_t e = -(bias_a + bias_b);\n    #pragma omp parallel for schedule(dynamic, 1)",
                          "int32_t e = (bias_a + bias_b);\n    #pragma omp parallel for schedule(dynamic, 1)"),
    "gemm_dropped_bias_b": ("int32_t e = -(bias_a + bias_b);\n    #pragma omp parallel for schedule(dynamic, 1)",
                            "int32_t e = -(bias_a);\n    #pragma omp parallel for schedule(dynamic, 1)"),
    "gemm_dgrad_transposed_w": ("dot_fp8(A + r * out, 1, fa, B + c, in, fb, out, e, v, av);",
                                "dot_fp8(A + r * out, 1, fa, B + c * in, 1, fb, out, e, v, av);"),
    "gemm_wgrad_swapped_index": ("dot_fp8(A + r, out, fa, B + c, in, fb, T, e, v, av);",
                                 "dot_fp8(A + c, out, fa, B + r, in, fb, T, e, v, av);"),
    "gemm_dropped_last_term": ("for (int64_t k = 0; k < K; ++k) {", "for (int64_t k = 0; k + 1 < K; ++k) {"),
}


@pytest.fixture(scope="module")
def source():
    with open(SRC) as f:
        return f.read()


def test_unmutated_oracle_passes_the_checks(source, tmp_path):
    assert _all_pins(_build(source, str(tmp_path), "clean"))


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(source, tmp_path, name):
    old, new = MUTATIONS[name]
    assert source.count(old) == 1, "mutation site not found: %s" % name
    L = _build(source.replace(old, new), str(tmp_path), name)
    assert not _all_pins(L), "pins did not catch: %s" % name
