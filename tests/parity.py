"""Comparison helpers shared by the GPU parity tests (no method arithmetic).

GEMM tolerance, per output element (fp64 reference r, sum of |products| s, both
already multiplied by 2^-(biasA + biasB)):

    |gpu - r| <= 1e-3 * s + ulp_bf16(r)

ulp_bf16(r) = 2^(floor(log2|r|) - 7) for normal r, and never less than 2^-133
(the spacing of BF16 subnormals, which is also its value at r = 0).  The FP8
products are exact in fp32, so the only differences allowed are the order of
the fp32 accumulation and the one final rounding to the output type; the same
bound is used for BF16 and FP32 outputs.
"""
import numpy as np
import torch


def ulp_bf16(r):
    a = np.abs(r)
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    u = np.ldexp(1.0, (e - 7).astype(np.int64))
    return np.maximum(np.where(a > 0, u, 0.0), 2.0 ** -133)


def gemm_tolerance(ref, absref):
    return 1e-3 * absref + ulp_bf16(ref)


def assert_gemm_close(gpu, ref, absref, what=""):
    g = np.asarray(gpu, dtype=np.float64)
    assert g.shape == ref.shape, (g.shape, ref.shape)
    assert np.all(np.isfinite(g)), "%s: non-finite output" % what
    err = np.abs(g - ref)
    tol = gemm_tolerance(ref, absref)
    bad = err > tol
    if bad.any():
        idx = np.argwhere(bad)[:5]
        raise AssertionError("%s: %d / %d elements out of tolerance, e.g. %s: gpu=%s ref=%s tol=%s"
                             % (what, int(bad.sum()), bad.size, idx.tolist(),
                                g[tuple(idx.T)], ref[tuple(idx.T)], tol[tuple(idx.T)]))
    return float((err / np.maximum(tol, 1e-300)).max()) if err.size else 0.0


def to_f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def f32_bits(x):
    return np.array([x], dtype=np.float32).view(np.uint32)[0]


def codes_equal_nan_aware(a, b, fmt):
    """FP8 code arrays equal, treating any two NaN codes of the format as equal."""
    a = np.asarray(a, dtype=np.uint8)
    b = np.asarray(b, dtype=np.uint8)
    low_a, low_b = a & 0x7F, b & 0x7F
    if fmt == 0:
        nan_a, nan_b = low_a == 0x7F, low_b == 0x7F
    else:
        nan_a, nan_b = low_a > 0x7C, low_b > 0x7C
    return bool(np.array_equal(nan_a, nan_b) and np.array_equal(a[~nan_a], b[~nan_b]))


def u8(t):
    return t.detach().cpu().view(torch.uint8).numpy()
