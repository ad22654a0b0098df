"""CPU oracle for the FP8-AMAX scaled linear layer — TEST INFRASTRUCTURE ONLY.

Only tests/, ``__graft_entry__.smoke()`` and the CPU-baseline / reference leg of
``bench.py`` may import this package.  It wraps ``fp8_oracle.c`` (plain C,
compiled by ``oracle/build.py``) with numpy marshalling and holds no arithmetic
of its own.  It never imports the CUDA library and the CUDA library never
imports it.

Functions (each cites its source in fp8_oracle.c):
  fp8_decode(codes, fmt)            exact value of each FP8 code (float64)
  fp8_encode(values, fmt, saturate) nearest FP8 code, ties to even
  amax(x)                           NaN-propagating max |x| (fp32 result)
  compute_bias(amax, fmt, margin)   floor(log2(fmt_max/amax)) - margin
  cast_scaled(x, bias, fmt)         FP8 codes of x * 2^bias
  linear(pass_, A, fa, ba, B, fb, bb, T, in_, out)          full fp64 output
  linear_entries(pass_, ..., rows, cols)                     sampled entries
"""
import ctypes
import os

import numpy as np

from . import build as _build

E4M3, E5M2 = 0, 1
FWD, DGRAD, WGRAD = 0, 1, 2

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        c = ctypes
        L.oracle_fp8_decode.restype = c.c_double
        L.oracle_fp8_decode.argtypes = [c.c_uint8, c.c_int]
        L.oracle_fp8_encode.restype = c.c_uint8
        L.oracle_fp8_encode.argtypes = [c.c_double, c.c_int, c.c_int]
        L.oracle_fmt_max.restype = c.c_double
        L.oracle_fmt_max.argtypes = [c.c_int]
        L.oracle_amax_f32.restype = c.c_float
        L.oracle_amax_f32.argtypes = [c.c_void_p, c.c_size_t]
        L.oracle_amax_bf16.restype = c.c_float
        L.oracle_amax_bf16.argtypes = [c.c_void_p, c.c_size_t]
        L.oracle_compute_bias.restype = c.c_int32
        L.oracle_compute_bias.argtypes = [c.c_float, c.c_int, c.c_int]
        L.oracle_cast_scaled_f32.restype = None
        L.oracle_cast_scaled_f32.argtypes = [c.c_void_p, c.c_size_t, c.c_int32, c.c_int, c.c_void_p]
        L.oracle_cast_scaled_bf16.restype = None
        L.oracle_cast_scaled_bf16.argtypes = [c.c_void_p, c.c_size_t, c.c_int32, c.c_int, c.c_void_p]
        L.oracle_encode_f32_bits.restype = None
        L.oracle_encode_f32_bits.argtypes = [c.c_void_p, c.c_size_t, c.c_int, c.c_int, c.c_void_p]
        L.oracle_linear_entries.restype = None
        L.oracle_linear_entries.argtypes = [
            c.c_int, c.c_void_p, c.c_int, c.c_int32, c.c_void_p, c.c_int, c.c_int32,
            c.c_int64, c.c_int64, c.c_int64, c.c_void_p, c.c_void_p, c.c_int64,
            c.c_void_p, c.c_void_p]
        L.oracle_linear_full.restype = None
        L.oracle_linear_full.argtypes = [
            c.c_int, c.c_void_p, c.c_int, c.c_int32, c.c_void_p, c.c_int, c.c_int32,
            c.c_int64, c.c_int64, c.c_int64, c.c_void_p, c.c_void_p]
        L.oracle_num_threads.restype = c.c_int
        L.oracle_num_threads.argtypes = []
        _lib = L
    return _lib


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _as_bits(x):
    """Accept numpy float32 / uint16 (bf16 bits) arrays, or torch CPU tensors."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().contiguous().cpu()
            if x.dtype == torch.bfloat16:
                return x.view(torch.int16).numpy().view(np.uint16), "bf16"
            if x.dtype == torch.float32:
                return x.numpy(), "f32"
            raise TypeError("oracle takes bf16 or fp32 tensors, got %s" % x.dtype)
    except ImportError:
        pass
    x = np.ascontiguousarray(x)
    if x.dtype == np.float32:
        return x, "f32"
    if x.dtype == np.uint16:
        return x, "bf16"
    raise TypeError("oracle takes float32 or uint16 (bf16 bits), got %s" % x.dtype)


def num_threads():
    return lib().oracle_num_threads()


def fmt_max(fmt):
    return lib().oracle_fmt_max(fmt)


def fp8_decode(codes, fmt):
    codes = np.asarray(codes, dtype=np.uint8)
    f = lib().oracle_fp8_decode
    return np.array([f(int(c), fmt) for c in codes.ravel()], dtype=np.float64).reshape(codes.shape)


def fp8_decode_table(fmt):
    return fp8_decode(np.arange(256, dtype=np.uint8), fmt)


def fp8_encode(values, fmt, saturate=True):
    values = np.asarray(values, dtype=np.float64)
    f = lib().oracle_fp8_encode
    return np.array([f(float(v), fmt, int(bool(saturate))) for v in values.ravel()],
                    dtype=np.uint8).reshape(values.shape)


def encode_f32_bits(bits, fmt, saturate=True):
    bits = np.ascontiguousarray(bits, dtype=np.uint32)
    out = np.empty(bits.shape, dtype=np.uint8)
    lib().oracle_encode_f32_bits(_ptr(bits), bits.size, fmt, int(bool(saturate)), _ptr(out))
    return out


def amax(x):
    a, kind = _as_bits(x)
    if kind == "f32":
        return np.float32(lib().oracle_amax_f32(_ptr(a), a.size))
    return np.float32(lib().oracle_amax_bf16(_ptr(a), a.size))


def compute_bias(amax_value, fmt, margin):
    return int(lib().oracle_compute_bias(float(np.float32(amax_value)), fmt, int(margin)))


def cast_scaled(x, bias, fmt):
    a, kind = _as_bits(x)
    out = np.empty(a.shape, dtype=np.uint8)
    fn = lib().oracle_cast_scaled_f32 if kind == "f32" else lib().oracle_cast_scaled_bf16
    fn(_ptr(a), a.size, int(bias), fmt, _ptr(out))
    return out


def quantize(x, fmt, margin):
    """amax -> compute_bias -> cast, the whole per-tensor FP8-AMAX step."""
    m = amax(x)
    b = compute_bias(m, fmt, margin)
    return m, b, cast_scaled(x, b, fmt)


def _codes(a):
    try:
        import torch
        if isinstance(a, torch.Tensor):
            a = a.detach().contiguous().cpu().view(torch.uint8).numpy()
    except ImportError:
        pass
    return np.ascontiguousarray(a, dtype=np.uint8)


def _out_shape(pass_, T, in_, out):
    return {FWD: (T, out), DGRAD: (T, in_), WGRAD: (out, in_)}[pass_]


def linear(pass_, A, fa, ba, B, fb, bb, T, in_, out, with_abs=True):
    """Whole output of one pass in fp64 (and the matching sum of |products|)."""
    A = _codes(A)
    B = _codes(B)
    shape = _out_shape(pass_, T, in_, out)
    val = np.empty(shape, dtype=np.float64)
    av = np.empty(shape, dtype=np.float64) if with_abs else None
    lib().oracle_linear_full(pass_, _ptr(A), fa, int(ba), _ptr(B), fb, int(bb),
                             T, in_, out, _ptr(val), _ptr(av) if with_abs else None)
    return (val, av) if with_abs else val


def linear_entries(pass_, A, fa, ba, B, fb, bb, T, in_, out, rows, cols):
    """Selected output entries (rows[e], cols[e]) of one pass, fp64."""
    A = _codes(A)
    B = _codes(B)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    cols = np.ascontiguousarray(cols, dtype=np.int64)
    n = rows.size
    val = np.empty(n, dtype=np.float64)
    av = np.empty(n, dtype=np.float64)
    lib().oracle_linear_entries(pass_, _ptr(A), fa, int(ba), _ptr(B), fb, int(bb),
                                T, in_, out, _ptr(rows), _ptr(cols), n, _ptr(val), _ptr(av))
    return val, av
