"""Pins for the oracle's scaled cast q = FP8(x * 2^bias).

  * power-of-two scaling of values that are representable is lossless;
  * for every tensor, max |dec(q)| never exceeds fmt_max (with the bias from
    compute_bias, any margin >= 0);
  * values exactly fmt_max / 2^k give bias k - margin, and with margin 0 the
    largest element encodes to the max finite code;
  * the cast equals the codec applied to the exactly scaled value, checked
    against torch's float8 conversion of x*2^bias (exact in fp64) below the
    overflow threshold.
"""
import numpy as np
import pytest
import torch

import oracle

TDT = {oracle.E4M3: torch.float8_e4m3fn, oracle.E5M2: torch.float8_e5m2}
MAXCODE = {oracle.E4M3: 0x7E, oracle.E5M2: 0x7B}


@pytest.mark.parametrize("fmt", [oracle.E4M3, oracle.E5M2])
def test_power_of_two_scaling_is_lossless(fmt):
    table = oracle.fp8_decode_table(fmt)
    ebits, mbits = (4, 3) if fmt == oracle.E4M3 else (5, 2)
    n_checked = 0
    for c in range(256):
        v = table[c]
        if not np.isfinite(v) or v == 0:
            continue
        for k in range(-20, 21):
            target = v * 2.0 ** k
            # the target is representable iff some code decodes to it
            hits = np.nonzero(table == target)[0]
            if hits.size == 0:
                continue
            x = np.array([v], dtype=np.float32)
            q = oracle.cast_scaled(x, k, fmt)[0]
            assert table[q] == target, (hex(c), k)
            n_checked += 1
    assert n_checked > 1000


@pytest.mark.parametrize("fmt", [oracle.E4M3, oracle.E5M2])
@pytest.mark.parametrize("margin", [0, 1, 3])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_scaled_amax_never_exceeds_fmt_max(fmt, margin, dtype):
    g = torch.Generator().manual_seed(11 + fmt + 3 * margin)
    table = oracle.fp8_decode_table(fmt)
    for sigma in (1e-6, 1.0, 1e3, 1e30):
        x = (torch.randn(4097, generator=g) * sigma).to(dtype)
        m, b, q = oracle.quantize(x, fmt, margin)
        deq = table[q]
        assert np.all(np.isfinite(deq))
        assert np.max(np.abs(deq)) <= oracle.fmt_max(fmt)
        if margin == 0:
            # the largest element lands in the top binade: at least fmt_max/2
            # up to the rounding of one ulp
            assert np.max(np.abs(deq)) >= oracle.fmt_max(fmt) / 2 * (1 - 2.0 ** -2)


@pytest.mark.parametrize("fmt", [oracle.E4M3, oracle.E5M2])
@pytest.mark.parametrize("margin", [0, 3])
def test_adversarial_exact_fmt_max_over_power_of_two(fmt, margin):
    rng = np.random.default_rng(3 + fmt)
    fm = oracle.fmt_max(fmt)
    for k in rng.integers(0, 21, size=8):
        x = np.array([fm / 2.0 ** k, -fm / 2.0 ** (k + 1), 0.0, fm / 2.0 ** (k + 5)], dtype=np.float32)
        m, b, q = oracle.quantize(x, fmt, margin)
        assert b == k - margin
        if margin == 0:
            assert q[0] == MAXCODE[fmt]
        assert oracle.fp8_decode(q[:1], fmt)[0] == fm / 2.0 ** margin


@pytest.mark.parametrize("fmt", [oracle.E4M3, oracle.E5M2])
def test_all_zero_and_single_spike(fmt):
    z = np.zeros(1000, dtype=np.float32)
    z[::7] = -0.0
    m, b, q = oracle.quantize(z, fmt, 3)
    assert m == 0 and b == 0
    assert np.all((q == 0x00) | (q == 0x80))
    assert np.array_equal(q == 0x80, np.signbit(z))
    s = np.zeros(1000, dtype=np.float32)
    s[123] = 1e4
    m, b, q = oracle.quantize(s, fmt, 0)
    assert m == np.float32(1e4)
    assert oracle.fp8_decode(q[123:124], fmt)[0] <= oracle.fmt_max(fmt)
    assert np.count_nonzero(q) == 1


@pytest.mark.parametrize("fmt", [oracle.E4M3, oracle.E5M2])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_cast_matches_torch_on_exactly_scaled_values(fmt, dtype):
    g = torch.Generator().manual_seed(21 + fmt)
    x = (torch.randn(100003, generator=g) * 0.37).to(dtype)
    for bias in (-5, 0, 3, 9, 20):
        q = oracle.cast_scaled(x, bias, fmt)
        scaled = x.to(torch.float64) * (2.0 ** bias)         # exact
        ok = scaled.abs() < oracle.fmt_max(fmt)
        ref = scaled.to(torch.float32).to(TDT[fmt]).view(torch.uint8).numpy()
        assert np.array_equal(q[ok.numpy()], ref[ok.numpy()]), bias
        sat = q[~ok.numpy()] & 0x7F
        assert np.all(sat == MAXCODE[fmt])
