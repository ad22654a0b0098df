"""GPU parity of the memory-bound steps — amax, compute_bias, scaled cast and
the fused quantize — against the CPU oracle, bit for bit, through the C ABI.

Inputs follow the amax + bias + cast sweep: BF16 and FP32 tensors, N(0, sigma)
with sigma in {1e-6, 1, 1e3}, all-zero, a single spike, values exactly
fmt_max / 2^k; both formats; margins {0, 3}; sizes with ragged tails from 0 to
2^24 elements, one 2^30 tensor per dtype, and every fp32 bit pattern through
the cast."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import codes_equal_nan_aware, f32_bits, u8

pytestmark = pytest.mark.gpu

fp8 = pytest.importorskip("fp8_tensor_scaled_b200")
DEV = "cuda"
DTYPES = [torch.bfloat16, torch.float32]
FMTS = [fp8.E4M3, fp8.E5M2]
SIZES = [0, 1, 7, 8, 9, 15, 16, 17, 31, 33, 4095, 65536, 65537, (1 << 20) + 3, 1 << 24]


def _check_amax(x_cpu, got):
    ref = oracle.amax(x_cpu)
    g = got.cpu().numpy()[0]
    if np.isnan(ref):
        assert np.isnan(g)
    else:
        assert f32_bits(g) == f32_bits(ref), (g, ref)
    return ref


def _check_all(x_cpu, fmt, margin):
    x = x_cpu.to(DEV)
    # separate calls
    amax = fp8.fp8_amax(x)
    bias = fp8.fp8_compute_bias(amax, fmt, margin)
    q = fp8.fp8_cast_scaled(x, bias, fmt)
    # fused
    amax2, bias2, q2 = fp8.fp8_quantize(x, fmt, margin)
    torch.cuda.synchronize()
    ref_amax = _check_amax(x_cpu, amax)
    _check_amax(x_cpu, amax2)
    ref_bias = oracle.compute_bias(ref_amax, fmt, margin)
    assert int(bias.item()) == ref_bias
    assert int(bias2.item()) == ref_bias
    ref_q = oracle.cast_scaled(x_cpu, ref_bias, fmt).reshape(x_cpu.shape)
    assert codes_equal_nan_aware(u8(q), ref_q, fmt)
    assert np.array_equal(u8(q2), u8(q))


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("n", SIZES)
def test_sizes_normal(dtype, n):
    x = workloads.sweep_tensor(n, dtype, "normal", 1.0, seed=4000 + n)
    for fmt in FMTS:
        _check_all(x, fmt, 0)


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("kind", ["normal", "zeros", "spike_zeros", "spike_normal", "exact_pow2"])
@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("margin", [0, 3])
def test_sweep_kinds(dtype, kind, fmt, margin):
    n = (1 << 18) + 5
    sigmas = workloads.SWEEP_SIGMAS if kind == "normal" else (1.0,)
    for sigma in sigmas:
        x = workloads.sweep_tensor(n, dtype, kind, sigma, seed=4100 + margin,
                                   fmt_max=fp8.FMT_MAX[fmt])
        _check_all(x, fmt, margin)


@pytest.mark.parametrize("dtype", DTYPES)
def test_full_size_2_30(dtype):
    n = 1 << 30
    xd = workloads.sweep_tensor(n, dtype, "normal", 1.0, seed=4999, device=DEV)
    x_cpu = xd.cpu()
    amax, bias, q = fp8.fp8_quantize(xd, fp8.E4M3, 0)
    torch.cuda.synchronize()
    ref_amax = _check_amax(x_cpu, amax)
    ref_bias = oracle.compute_bias(ref_amax, fp8.E4M3, 0)
    assert int(bias.item()) == ref_bias
    assert np.array_equal(u8(q), oracle.cast_scaled(x_cpu, ref_bias, fp8.E4M3))


def test_special_values():
    vals = [0.0, -0.0, 1.0, -1.0, 448.0, 464.0, 480.0, 1e6, float("inf"), float("-inf"),
            57344.0, 61440.0, 2.0 ** -10, -(2.0 ** -10), 3 * 2.0 ** -10, 2.0 ** -149, 1e-40,
            -1e-40, float("nan")]
    x = torch.tensor(vals * 3, dtype=torch.float32)
    for fmt in FMTS:
        for bias in (0, 5, -3):
            b = torch.tensor([bias], dtype=torch.int32, device=DEV)
            q = fp8.fp8_cast_scaled(x.to(DEV), b, fmt)
            assert codes_equal_nan_aware(u8(q), oracle.cast_scaled(x, bias, fmt), fmt)
    # amax: NaN wins, then inf
    xd = torch.tensor([1.0, float("-inf"), 3.0], device=DEV)
    assert fp8.fp8_amax(xd).item() == float("inf")
    xd = torch.tensor([1.0, float("nan"), float("inf")], device=DEV, dtype=torch.bfloat16)
    assert np.isnan(fp8.fp8_amax(xd).item())


@pytest.mark.parametrize("dtype", DTYPES)
def test_extreme_biases(dtype):
    g = torch.Generator().manual_seed(77)
    # magnitudes across the whole fp32 range, subnormals included
    e = torch.randint(-149, 127, (200003,), generator=g).to(torch.float64)
    x = (torch.randn(200003, generator=g, dtype=torch.float64) * torch.exp2(e)).to(dtype)
    xd = x.to(DEV)
    for fmt in FMTS:
        for bias in (-1000, -300, -200, -140, -127, -126, -1, 0, 1, 127, 128, 150, 164, 200, 300,
                     1000):
            b = torch.tensor([bias], dtype=torch.int32, device=DEV)
            q = fp8.fp8_cast_scaled(xd, b, fmt)
            assert codes_equal_nan_aware(u8(q), oracle.cast_scaled(x, bias, fmt), fmt), bias


def _bias_amax_values():
    rng = np.random.default_rng(5)
    bits = rng.integers(1, 0x7F800000, size=300, dtype=np.uint32)
    vals = list(bits.view(np.float32))
    vals += [np.float32(v) for v in (1.0, 1.75, 2.0, 448.0, 449.0, 57344.0, 0.001, 1e-4, 2.0 ** -149,
                                     2.0 ** -126, 3.4028234663852886e38, 0.0, np.inf, np.nan)]
    vals.append(np.nextafter(np.float32(1.75), np.float32(2)))
    return vals


def test_compute_bias_values():
    vals = _bias_amax_values()
    amax = torch.tensor(np.array(vals, dtype=np.float32), device=DEV)
    out = torch.empty(1, dtype=torch.int32, device=DEV)
    for fmt in FMTS:
        for margin in (0, 1, 3, -2):
            got = []
            for i in range(len(vals)):
                fp8.fp8_compute_bias(amax[i:i + 1], fmt, margin, out=out)
                got.append(int(out.item()))
            ref = [oracle.compute_bias(v, fmt, margin) for v in vals]
            assert got == ref, (fmt, margin)


@pytest.mark.parametrize("fmt", FMTS)
def test_cast_every_fp32_bit_pattern(fmt):
    """All 2^32 fp32 inputs through the device cast (bias 0) vs the oracle codec."""
    chunk = 1 << 28
    zero = torch.zeros(1, dtype=torch.int32, device=DEV)
    out = torch.empty(chunk, dtype=torch.uint8, device=DEV)
    for start in range(0, 1 << 32, chunk):
        bits = torch.arange(start, start + chunk, dtype=torch.int64, device=DEV).to(torch.int32)
        fp8.fp8_cast_scaled(bits.view(torch.float32), zero, fmt, out=out)
        got = out.cpu().numpy()
        host_bits = np.arange(start, start + chunk, dtype=np.uint64).astype(np.uint32)
        ref = oracle.encode_f32_bits(host_bits, fmt, True)
        assert codes_equal_nan_aware(got, ref, fmt), start


@pytest.mark.parametrize("fmt", FMTS)
def test_cast_every_bf16_pattern_many_biases(fmt):
    x = torch.arange(65536, dtype=torch.int32).to(torch.int16).view(torch.bfloat16)
    xd = x.to(DEV)
    for bias in range(-140, 141, 7):
        b = torch.tensor([bias], dtype=torch.int32, device=DEV)
        q = fp8.fp8_cast_scaled(xd, b, fmt)
        assert codes_equal_nan_aware(u8(q), oracle.cast_scaled(x, bias, fmt), fmt), bias


def test_no_device_error_recorded():
    st, where = fp8.fp8_device_error(clear=False)
    assert st == 0 and where == 0
