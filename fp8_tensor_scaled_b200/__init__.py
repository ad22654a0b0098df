"""fp8_tensor_scaled_b200 — B200 (sm_100a) FP8-AMAX scaled linear layer.

A thin Python binding over the C ABI in ``include/fp8amax.h`` (library
``libfp8amax.so`` built in-tree by ``python -m fp8_tensor_scaled_b200.build``).
Every function here only marshals torch CUDA tensors into pointers and sizes
and calls the entry point of the same name; all arithmetic runs in the
library's kernels on the tensor's stream.  There is no CPU path: without the
built library, or without an sm_100 device, every call raises.

Method: review page "Training and inference of large language models using
8-bit floating point" (Perez, Zhang et al.), section "Proposed method":
per-tensor amax -> compute_bias (log2 of fmt_max / amax, less a margin) ->
scale by 2^bias and cast to FP8 (E4M3 for weights and activations, E5M2 for
gradients) -> FP8 matmul -> unscale by 2^-(biasA + biasB).
"""
import ctypes
import os
import re

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfp8amax.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "fp8amax.h")

E4M3, E5M2 = 0, 1
BF16, FP32 = 0, 1
FMT_MAX = {E4M3: 448.0, E5M2: 57344.0}
STATUS = {0: "FP8_OK", 1: "FP8_ERR_INVALID_ARGUMENT", 2: "FP8_ERR_UNSUPPORTED",
          3: "FP8_ERR_MISALIGNED", 4: "FP8_ERR_CUDA", 5: "FP8_ERR_TIMEOUT", 6: "FP8_ERR_NO_DEVICE"}


class Fp8Error(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__("%s failed: %s" % (fn, STATUS.get(status, str(status))))


_lib = None


def lib():
    """The loaded C library (ctypes), with argument types declared."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError("libfp8amax.so is not built (%s); run `python -m "
                          "fp8_tensor_scaled_b200.build` (nvcc, sm_100a)" % LIB_PATH)
    L = ctypes.CDLL(LIB_PATH)
    c = ctypes
    vp, i32, i64, sz, u64 = c.c_void_p, c.c_int32, c.c_int64, c.c_size_t, c.c_uint64
    sigs = {
        "fp8_amax": [vp, c.c_int, sz, vp, vp],
        "fp8_compute_bias": [vp, c.c_int, i32, vp, vp],
        "fp8_cast_scaled": [vp, c.c_int, sz, vp, c.c_int, vp, vp],
        "fp8_quantize": [vp, c.c_int, sz, c.c_int, i32, vp, vp, vp, vp],
        "fp8_linear_fwd": [vp, c.c_int, vp, vp, c.c_int, vp, i64, i64, i64, vp, c.c_int, vp],
        "fp8_linear_bwd_dgrad": [vp, c.c_int, vp, vp, c.c_int, vp, i64, i64, i64, vp, c.c_int, vp],
        "fp8_linear_bwd_wgrad": [vp, c.c_int, vp, vp, c.c_int, vp, i64, i64, i64, vp, c.c_int, vp],
        "fp8_linear_fwd_amax": [vp, c.c_int, vp, vp, c.c_int, vp, i64, i64, i64, vp, c.c_int, vp,
                                vp],
        "fp8_linear_bwd_dgrad_amax": [vp, c.c_int, vp, vp, c.c_int, vp, i64, i64, i64, vp, c.c_int,
                                      vp, vp],
        "fp8_linear_fwd_ws": [vp, c.c_int, vp, vp, c.c_int, vp, i64, i64, i64, vp, c.c_int, vp,
                              sz, vp],
        "fp8_linear_bwd_wgrad_ws": [vp, c.c_int, vp, vp, c.c_int, vp, i64, i64, i64, vp, c.c_int,
                                    vp, sz, vp],
        "fp8_device_error": [c.c_int, vp],
        "fp8_selftest_bounded_wait": [u64],
        "fp8_abi_version": [],
    }
    for name, args in sigs.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = c.c_int
    L.fp8_status_string.argtypes = [c.c_int]
    L.fp8_status_string.restype = c.c_char_p
    L.fp8_linear_fwd_workspace_size.argtypes = [i64, i64, i64]
    L.fp8_linear_fwd_workspace_size.restype = sz
    L.fp8_linear_bwd_wgrad_workspace_size.argtypes = [i64, i64, i64]
    L.fp8_linear_bwd_wgrad_workspace_size.restype = sz
    _lib = L
    return L


def declared_entry_points():
    """Names of the functions include/fp8amax.h declares."""
    with open(HEADER_PATH) as f:
        text = f.read()
    return sorted(set(re.findall(r"\b(fp8_[a-z0-9_]+)\s*\(", text)))


def _check(fn, status):
    if status != 0:
        raise Fp8Error(fn, status)


def _stream_ptr(t):
    return torch.cuda.current_stream(t.device).cuda_stream


def _dtype_code(t):
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return FP32
    raise TypeError("expected a bfloat16 or float32 tensor, got %s" % t.dtype)


def _need_cuda(*ts):
    for t in ts:
        if t is not None and (not isinstance(t, torch.Tensor) or not t.is_cuda):
            raise TypeError("fp8_tensor_scaled_b200 takes CUDA tensors only")
        if t is not None and not t.is_contiguous():
            raise ValueError("tensors must be contiguous (row-major)")


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None and t.numel() > 0 else ctypes.c_void_p(0)


def fp8_status_string(status: int) -> str:
    return lib().fp8_status_string(int(status)).decode()


def fp8_amax(x: torch.Tensor, out: torch.Tensor = None) -> torch.Tensor:
    """max |x| of the whole tensor, as a float32 [1] tensor on x's device."""
    _need_cuda(x)
    if out is None:
        out = torch.empty(1, dtype=torch.float32, device=x.device)
    _check("fp8_amax", lib().fp8_amax(_ptr(x), _dtype_code(x), x.numel(), _ptr(out),
                                      ctypes.c_void_p(_stream_ptr(x))))
    return out


def fp8_compute_bias(amax: torch.Tensor, fmt: int, margin: int = 0,
                     out: torch.Tensor = None) -> torch.Tensor:
    """floor(log2(fmt_max / amax)) - margin as an int32 [1] tensor (0 for amax 0/inf/NaN)."""
    _need_cuda(amax)
    if out is None:
        out = torch.empty(1, dtype=torch.int32, device=amax.device)
    _check("fp8_compute_bias", lib().fp8_compute_bias(_ptr(amax), int(fmt), int(margin), _ptr(out),
                                                      ctypes.c_void_p(_stream_ptr(amax))))
    return out


def fp8_cast_scaled(x: torch.Tensor, bias: torch.Tensor, fmt: int,
                    out: torch.Tensor = None) -> torch.Tensor:
    """FP8 codes (uint8, same shape as x) of x * 2^bias, RNE, satfinite."""
    _need_cuda(x, bias)
    if out is None:
        out = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    _check("fp8_cast_scaled", lib().fp8_cast_scaled(_ptr(x), _dtype_code(x), x.numel(), _ptr(bias),
                                                    int(fmt), _ptr(out),
                                                    ctypes.c_void_p(_stream_ptr(x))))
    return out


def fp8_quantize(x: torch.Tensor, fmt: int, margin: int = 0, amax: torch.Tensor = None,
                 bias: torch.Tensor = None, out: torch.Tensor = None):
    """amax -> bias -> cast in one call; returns (amax [1] f32, bias [1] i32, codes u8)."""
    _need_cuda(x)
    dev = x.device
    if amax is None:
        amax = torch.empty(1, dtype=torch.float32, device=dev)
    if bias is None:
        bias = torch.empty(1, dtype=torch.int32, device=dev)
    if out is None:
        out = torch.empty(x.shape, dtype=torch.uint8, device=dev)
    _check("fp8_quantize", lib().fp8_quantize(_ptr(x), _dtype_code(x), x.numel(), int(fmt),
                                              int(margin), _ptr(amax), _ptr(bias), _ptr(out),
                                              ctypes.c_void_p(_stream_ptr(x))))
    return amax, bias, out


_OUT = {torch.bfloat16: BF16, torch.float32: FP32}


def _linear(name, a, fa, ba, b, fb, bb, T, in_, out_, shape, out, out_dtype, amax=False):
    _need_cuda(a, ba, b, bb, out)
    dev = ba.device
    if out is None:
        out = torch.empty(shape, dtype=out_dtype, device=dev)
    if tuple(out.shape) != tuple(shape) or out.dtype not in _OUT:
        raise ValueError("output must be %s of bfloat16/float32" % (shape,))
    args = [_ptr(a), int(fa), _ptr(ba), _ptr(b), int(fb), _ptr(bb), int(T), int(in_), int(out_),
            _ptr(out), _OUT[out.dtype]]
    if amax is not False:
        if amax is None or amax is True:
            amax = torch.empty(1, dtype=torch.float32, device=dev)
        _need_cuda(amax)
        name = name + "_amax"
        args.append(_ptr(amax))
    f = getattr(lib(), name)
    _check(name, f(*args, ctypes.c_void_p(_stream_ptr(ba))))
    return out if amax is False else (out, amax)


def fp8_linear_fwd(x8, fx, bias_x, w8, fw, bias_w, out=None, out_dtype=torch.bfloat16,
                   amax=False):
    """Y [T,out] = (X8 [T,in] . W8 [out,in]^T) * 2^-(bias_x + bias_w).

    amax=True (or a float32 [1] device tensor) calls fp8_linear_fwd_amax and
    returns (Y, max|Y|) with the amax taken in the GEMM epilogue."""
    T, in_ = x8.shape
    out_ = w8.shape[0]
    assert w8.shape[1] == in_
    return _linear("fp8_linear_fwd", x8, fx, bias_x, w8, fw, bias_w, T, in_, out_, (T, out_),
                   out, out_dtype, amax)


def fp8_linear_fwd_workspace_size(T, in_, out_):
    """Bytes of workspace fp8_linear_fwd_ws splits K with (0: no split)."""
    return int(lib().fp8_linear_fwd_workspace_size(int(T), int(in_), int(out_)))


def fp8_linear_fwd_ws(x8, fx, bias_x, w8, fw, bias_w, out=None, out_dtype=torch.bfloat16,
                      workspace=None):
    """fp8_linear_fwd for few tokens with a split-K workspace (allocated here
    through torch when not given)."""
    T, in_ = x8.shape
    out_ = w8.shape[0]
    assert w8.shape[1] == in_
    _need_cuda(x8, bias_x, w8, bias_w, out, workspace)
    dev = bias_x.device
    if out is None:
        out = torch.empty((T, out_), dtype=out_dtype, device=dev)
    need = fp8_linear_fwd_workspace_size(T, in_, out_)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    nbytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("fp8_linear_fwd_ws", lib().fp8_linear_fwd_ws(
        _ptr(x8), int(fx), _ptr(bias_x), _ptr(w8), int(fw), _ptr(bias_w), int(T), int(in_),
        int(out_), _ptr(out), _OUT[out.dtype], _ptr(workspace), nbytes,
        ctypes.c_void_p(_stream_ptr(bias_x))))
    return out


def fp8_linear_fwd_noalloc(x8, fx, bias_x, w8, fw, bias_w, out, stream=None):
    """fp8_linear_fwd_ws without a workspace or any allocation: for callers
    that may not allocate device memory when they run a forward.  `out` must
    be given; the split-K scratch is the library's own 16 MiB array per GPU
    (calls that overlap on the GPU must be serialised by the caller)."""
    L = lib()
    f = L.fp8_linear_fwd_noalloc
    if f.argtypes is None:
        c = ctypes
        f.argtypes = [c.c_void_p, c.c_int, c.c_void_p, c.c_void_p, c.c_int, c.c_void_p,
                      c.c_int64, c.c_int64, c.c_int64, c.c_void_p, c.c_int, c.c_void_p]
        f.restype = c.c_int
    T, in_ = x8.shape
    out_ = w8.shape[0]
    _need_cuda(x8, bias_x, w8, bias_w, out)
    if tuple(out.shape) != (T, out_) or out.dtype not in _OUT:
        raise ValueError("output must be [T, out] of bfloat16/float32")
    s = stream if stream is not None else _stream_ptr(bias_x)
    _check("fp8_linear_fwd_noalloc", f(_ptr(x8), int(fx), _ptr(bias_x), _ptr(w8), int(fw),
                                       _ptr(bias_w), int(T), int(in_), int(out_), _ptr(out),
                                       _OUT[out.dtype], ctypes.c_void_p(s)))
    return out


def fp8_linear_bwd_dgrad(dy8, fdy, bias_dy, w8, fw, bias_w, out=None, out_dtype=torch.bfloat16,
                         amax=False):
    """dX [T,in] = (dY8 [T,out] . W8 [out,in]) * 2^-(bias_dy + bias_w).

    amax=True (or a float32 [1] device tensor) calls fp8_linear_bwd_dgrad_amax
    and returns (dX, max|dX|)."""
    T, out_ = dy8.shape
    in_ = w8.shape[1]
    assert w8.shape[0] == out_
    return _linear("fp8_linear_bwd_dgrad", dy8, fdy, bias_dy, w8, fw, bias_w, T, in_, out_,
                   (T, in_), out, out_dtype, amax)


FWD, DGRAD, WGRAD = 0, 1, 2


class _Plan(ctypes.Structure):
    _fields_ = [("tile_m", ctypes.c_int32), ("tile_n", ctypes.c_int32),
                ("ctas_per_tile", ctypes.c_int32), ("k_splits", ctypes.c_int32)]


def fp8_linear_plan(pass_, T, in_, out_, with_workspace=False):
    """The launch plan of one pass on the current device:
    {"tile_m", "tile_n", "ctas_per_tile", "k_splits"}."""
    L = lib()
    f = L.fp8_linear_plan
    f.argtypes = [ctypes.c_int, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int,
                  ctypes.POINTER(_Plan)]
    f.restype = ctypes.c_int
    p = _Plan()
    _check("fp8_linear_plan", f(int(pass_), int(T), int(in_), int(out_), int(bool(with_workspace)),
                                ctypes.byref(p)))
    return {k: int(getattr(p, k)) for k, _ in _Plan._fields_}


def fp8_linear_bwd_wgrad_workspace_size(T, in_, out_):
    """Bytes of workspace fp8_linear_bwd_wgrad_ws splits K with (0: no split)."""
    return int(lib().fp8_linear_bwd_wgrad_workspace_size(int(T), int(in_), int(out_)))


def fp8_linear_bwd_wgrad_ws(dy8, fdy, bias_dy, x8, fx, bias_x, out=None,
                            out_dtype=torch.bfloat16, workspace=None):
    """fp8_linear_bwd_wgrad with a split-K workspace (allocated here through
    torch when not given) for small weight gradients over many tokens."""
    T, out_ = dy8.shape
    in_ = x8.shape[1]
    assert x8.shape[0] == T
    _need_cuda(dy8, bias_dy, x8, bias_x, out, workspace)
    dev = bias_dy.device
    if out is None:
        out = torch.empty((out_, in_), dtype=out_dtype, device=dev)
    need = fp8_linear_bwd_wgrad_workspace_size(T, in_, out_)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    nbytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("fp8_linear_bwd_wgrad_ws", lib().fp8_linear_bwd_wgrad_ws(
        _ptr(dy8), int(fdy), _ptr(bias_dy), _ptr(x8), int(fx), _ptr(bias_x), int(T), int(in_),
        int(out_), _ptr(out), _OUT[out.dtype], _ptr(workspace), nbytes,
        ctypes.c_void_p(_stream_ptr(bias_dy))))
    return out


def fp8_linear_bwd_wgrad(dy8, fdy, bias_dy, x8, fx, bias_x, out=None, out_dtype=torch.bfloat16):
    """dW [out,in] = (dY8 [T,out]^T . X8 [T,in]) * 2^-(bias_dy + bias_x)."""
    T, out_ = dy8.shape
    in_ = x8.shape[1]
    assert x8.shape[0] == T
    return _linear("fp8_linear_bwd_wgrad", dy8, fdy, bias_dy, x8, fx, bias_x, T, in_, out_,
                   (out_, in_), out, out_dtype)


def fp8_device_error(clear: bool = True):
    """(status, site) of the device error word that bounded kernel waits write."""
    where = ctypes.c_int32(0)
    st = lib().fp8_device_error(int(bool(clear)), ctypes.byref(where))
    return st, where.value


def fp8_selftest_bounded_wait(timeout_ns: int = 50_000_000) -> int:
    """Status of a kernel wait on a barrier nothing completes (FP8_ERR_TIMEOUT expected)."""
    return lib().fp8_selftest_bounded_wait(int(timeout_ns))


from .layer import Fp8AmaxLinear  # noqa: E402  (convenience: one linear's fwd+bwd step)

__all__ = [
    "E4M3", "E5M2", "BF16", "FP32", "FMT_MAX", "Fp8Error", "lib", "declared_entry_points",
    "fp8_status_string", "fp8_amax", "fp8_compute_bias", "fp8_cast_scaled", "fp8_quantize",
    "fp8_linear_fwd", "fp8_linear_bwd_dgrad", "fp8_linear_bwd_wgrad", "fp8_device_error",
    "fp8_linear_fwd_ws", "fp8_linear_fwd_workspace_size", "fp8_linear_fwd_noalloc",
    "fp8_linear_bwd_wgrad_ws", "fp8_linear_bwd_wgrad_workspace_size", "fp8_linear_plan",
    "fp8_selftest_bounded_wait", "Fp8AmaxLinear",
]
