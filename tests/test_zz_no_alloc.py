"""fp8_linear_fwd_noalloc: the forward entry point for callers that cannot
allocate device memory where they run it (a locked allocator, a fixed memory
pool, a serving loop that forbids allocation, a C program with no device
allocator).  It takes the split-K scratch from an array inside the library
instead of a caller workspace.

Checked here through the C ABI, two calls in a row, against the
workspace entry point (fp8_linear_fwd_ws) within the GEMM tolerance the other
tests use, on a shape that uses the scratch and on one that does not.  The
file sorts last so that a run stopping at its first failure has run every
other test before it; it also passes alone in a fresh process, where its
first call does the library's one-time look-up of the array's address."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from parity import assert_gemm_close, to_f64

pytestmark = pytest.mark.gpu

fp8 = pytest.importorskip("fp8_tensor_scaled_b200")
DEV = "cuda"
E4 = fp8.E4M3


def _quantized(T, In, Out, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(T, In, generator=g).to(torch.bfloat16)
    w = (torch.randn(Out, In, generator=g) * 0.02).to(torch.bfloat16)
    _, bx, qx = fp8.fp8_quantize(x.to(DEV), E4, 0)
    _, bw, qw = fp8.fp8_quantize(w.to(DEV), E4, 0)
    return qx, bx, qw, bw


def _call_noalloc(qx, bx, qw, bw, y):
    L = fp8.lib()
    f = L.fp8_linear_fwd_noalloc
    c = ctypes
    f.argtypes = [c.c_void_p, c.c_int, c.c_void_p, c.c_void_p, c.c_int, c.c_void_p,
                  c.c_int64, c.c_int64, c.c_int64, c.c_void_p, c.c_int, c.c_void_p]
    f.restype = c.c_int
    T, In = qx.shape
    Out = qw.shape[0]
    stream = torch.cuda.current_stream().cuda_stream
    return f(qx.data_ptr(), E4, bx.data_ptr(), qw.data_ptr(), E4, bw.data_ptr(), T, In, Out,
             y.data_ptr(), fp8.BF16 if y.dtype == torch.bfloat16 else fp8.FP32, c.c_void_p(stream))


# (16, 12288, 512): 128-row tiles split K; (1024, 8192, 256): CTA-pair tiles
# split K within the scratch; (2048, 2048, 1024): a pair split would need more
# than the scratch holds, so the forward runs unsplit; (200, 512, 384): no split
@pytest.mark.parametrize("T,In,Out,splits", [(16, 12288, 512, True), (1024, 8192, 256, True),
                                             (2048, 2048, 1024, True), (200, 512, 384, False)])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_noalloc_matches_workspace_entry_point(T, In, Out, splits, out_dtype):
    assert (fp8.fp8_linear_fwd_workspace_size(T, In, Out) > 0) == splits
    qx, bx, qw, bw = _quantized(T, In, Out, seed=T + In)
    ref = fp8.fp8_linear_fwd_ws(qx, E4, bx, qw, E4, bw, out_dtype=out_dtype)
    # the tolerance of the other GEMM tests: 1e-3 * sum|a*b| + 1 BF16 ulp,
    # with sum|a*b| from the oracle
    _, absref = oracle.linear(oracle.FWD, qx.cpu().numpy(), E4, int(bx.item()),
                              qw.cpu().numpy(), E4, int(bw.item()), T, In, Out)
    for call in range(2):                        # two calls in a row share the scratch
        y = torch.full((T, Out), float("nan"), dtype=out_dtype, device=DEV)
        assert _call_noalloc(qx, bx, qw, bw, y) == 0
        torch.cuda.synchronize()
        assert_gemm_close(to_f64(y), to_f64(ref), absref, "noalloc call %d" % call)
    st, where = fp8.fp8_device_error(clear=False)
    assert st == 0, where
