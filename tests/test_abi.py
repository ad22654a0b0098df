"""The C-ABI library: it loads, exports every entry point the header declares,
and rejects bad arguments with status codes (no GPU needed: argument checks
run before any device work, and without a device a valid call reports
FP8_ERR_NO_DEVICE instead of falling back to anything)."""
import ctypes

import pytest
import torch

import fp8_tensor_scaled_b200 as fp8
from fp8_tensor_scaled_b200 import build as fp8_build

OK, INVALID, UNSUPPORTED, MISALIGNED, CUDA_ERR, TIMEOUT, NO_DEVICE = range(7)


@pytest.fixture(scope="module")
def L():
    fp8_build.build()
    return fp8.lib()


def test_exports_every_declared_symbol(L):
    names = fp8.declared_entry_points()
    required = {"fp8_amax", "fp8_compute_bias", "fp8_cast_scaled", "fp8_linear_fwd",
                "fp8_linear_bwd_dgrad", "fp8_linear_bwd_wgrad", "fp8_status_string"}
    assert required <= set(names)
    for n in names:
        assert hasattr(L, n), n


def test_status_strings(L):
    for code, name in fp8.STATUS.items():
        assert fp8.fp8_status_string(code) == name
    assert fp8.fp8_status_string(99) == "FP8_ERR_UNKNOWN"
    assert L.fp8_abi_version() == 1


P = ctypes.c_void_p
A16 = P(0x10000)          # a fake 16-byte aligned "device" address (never dereferenced)
A4 = P(0x10004)


def test_argument_validation(L):
    # null pointers / bad enums -> INVALID; misalignment -> MISALIGNED
    assert L.fp8_amax(P(0), 0, 10, A16, P(0)) == INVALID
    assert L.fp8_amax(A16, 7, 10, A16, P(0)) == INVALID
    assert L.fp8_amax(A16, 0, 10, P(0), P(0)) == INVALID
    assert L.fp8_amax(P(0x10008), 0, 10, A16, P(0)) == MISALIGNED
    assert L.fp8_compute_bias(A16, 2, 0, A16, P(0)) == INVALID
    assert L.fp8_compute_bias(A16, 0, 0, P(0x10002), P(0)) == MISALIGNED
    assert L.fp8_cast_scaled(A16, 0, 10, P(0), 0, A16, P(0)) == INVALID
    assert L.fp8_cast_scaled(A16, 0, 10, A16, 0, P(0x10001), P(0)) == MISALIGNED
    assert L.fp8_quantize(A16, 0, 10, 0, 0, A16, A16, P(0x10008), P(0)) == MISALIGNED
    # linear shapes: in/out multiples of 16, T >= 0
    args = lambda T, i, o, y=A16, x=A16: (x, 0, A16, A16, 0, A16, T, i, o, y, 0, P(0))
    assert L.fp8_linear_fwd(*args(128, 17, 32)) == UNSUPPORTED
    assert L.fp8_linear_fwd(*args(128, 32, 40)) == UNSUPPORTED
    assert L.fp8_linear_fwd(*args(-1, 32, 32)) == INVALID
    assert L.fp8_linear_fwd(*args(128, 0, 32)) == INVALID
    assert L.fp8_linear_fwd(*args(128, 32, 32, y=P(0x10008))) == MISALIGNED
    assert L.fp8_linear_bwd_dgrad(*args(128, 32, 32, x=P(0))) == INVALID
    assert L.fp8_linear_bwd_wgrad(*args(128, 32, 32, y=P(0))) == INVALID
    assert L.fp8_linear_fwd(A16, 0, A4, A16, 3, A16, 8, 16, 16, A16, 0, P(0)) == INVALID
    assert L.fp8_selftest_bounded_wait(10) == INVALID


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device behaviour")
def test_valid_calls_without_a_device_fail_loudly(L):
    # a valid call must not fall back to any CPU path: it reports NO_DEVICE
    assert L.fp8_amax(A16, 0, 10, A16, P(0)) == NO_DEVICE
    assert L.fp8_linear_fwd(A16, 0, A16, A16, 0, A16, 128, 32, 32, A16, 0, P(0)) == NO_DEVICE
    with pytest.raises(TypeError):
        fp8.fp8_amax(torch.zeros(4))            # CPU tensors are refused by the binding


def test_empty_token_count_is_valid_shape(L):
    # T == 0 passes argument checks with null token-sized tensors (then needs a device)
    r = L.fp8_linear_fwd(P(0), 0, A16, A16, 0, A16, 0, 32, 32, P(0), 0, P(0))
    assert r in (OK, NO_DEVICE)


def test_workspace_and_plan_entry_points(L):
    """Argument checks of the workspace, no-allocation and plan entry points
    run before any device work."""
    i64, sz = ctypes.c_int64, ctypes.c_size_t
    ws = lambda wptr, wbytes, y=A16: (A16, 0, A16, A16, 0, A16, i64(128), i64(32), i64(32), y, 0,
                                      wptr, sz(wbytes), P(0))
    # a workspace must be 256-byte aligned, and non-null when bytes are given
    assert L.fp8_linear_fwd_ws(*ws(P(0x10010), 1024)) == MISALIGNED
    assert L.fp8_linear_fwd_ws(*ws(P(0), 1024)) == INVALID
    assert L.fp8_linear_fwd_ws(*ws(P(0x10000), 1024, y=P(0x10008))) == MISALIGNED
    assert L.fp8_linear_bwd_wgrad_ws(*ws(P(0x10010), 1024)) == MISALIGNED
    assert L.fp8_linear_bwd_wgrad_ws(*ws(P(0), 1024)) == INVALID
    f = L.fp8_linear_fwd_noalloc
    f.argtypes = [P, ctypes.c_int, P, P, ctypes.c_int, P, i64, i64, i64, P, ctypes.c_int, P]
    f.restype = ctypes.c_int
    assert f(A16, 0, A16, A16, 0, A16, 128, 17, 32, A16, 0, P(0)) == UNSUPPORTED
    assert f(A16, 0, A16, A16, 0, A16, 128, 32, 32, P(0x10008), 0, P(0)) == MISALIGNED
    # the size queries report 0 without a device (nothing to plan on)
    if not torch.cuda.is_available():
        assert L.fp8_linear_fwd_workspace_size(16, 12288, 512) == 0
        assert L.fp8_linear_bwd_wgrad_workspace_size(8192, 768, 768) == 0
    # the plan query: null plan, unknown pass, negative sizes -> INVALID
    g = L.fp8_linear_plan
    g.argtypes = [ctypes.c_int, i64, i64, i64, ctypes.c_int, P]
    g.restype = ctypes.c_int
    plan = (ctypes.c_int32 * 4)()
    assert g(0, 16, 16, 16, 0, P(0)) == INVALID
    assert g(3, 16, 16, 16, 0, ctypes.cast(plan, P)) == INVALID
    assert g(0, -1, 16, 16, 0, ctypes.cast(plan, P)) == INVALID
    if not torch.cuda.is_available():
        assert g(0, 16, 16, 16, 0, ctypes.cast(plan, P)) == NO_DEVICE
