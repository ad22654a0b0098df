"""Pins for the oracle's amax and compute_bias.

compute_bias (review page "Training and inference of large language models
using 8-bit floating point", section "Proposed method") is pinned by
  * a hand-worked table (tests/golden/compute_bias_table.txt);
  * a brute-force search: floor(log2(fmt_max/amax)) is the largest integer b
    with amax * 2^b <= fmt_max, found here with exact rational arithmetic;
  * its invariants: amax*2^bias <= fmt_max, and tight (the next power of two
    overflows) when margin = 0.
amax is pinned against numpy's max(|x|) and against hand cases (NaN, inf, -0).
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle


def _load_table(golden_dir):
    rows = []
    with open(os.path.join(golden_dir, "compute_bias_table.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            fmt, amax, margin, bias = line.split()
            a = float.fromhex(amax) if amax.startswith("0x") else float(amax)
            rows.append((oracle.E4M3 if fmt == "E4M3" else oracle.E5M2, a, int(margin), int(bias)))
    return rows


def test_compute_bias_hand_table(golden_dir):
    rows = _load_table(golden_dir)
    assert len(rows) >= 30
    for fmt, a, margin, bias in rows:
        assert float(np.float32(a)) == a or a == 0.001 or a == 0.0001, a
        assert oracle.compute_bias(a, fmt, margin) == bias, (fmt, a, margin)


def _brute_force_bias(amax, fmt, margin):
    """max{b in Z : amax * 2^b <= fmt_max} - margin, by exact rationals."""
    a = Fraction(float(np.float32(amax)))
    fm = Fraction(oracle.fmt_max(fmt))
    best = None
    for b in range(-300, 301):
        if a * (Fraction(2) ** b) <= fm:
            best = b
    return best - margin


def _fp32_samples(n, seed):
    rng = np.random.default_rng(seed)
    bits = rng.integers(1, 0x7F800000, size=n, dtype=np.uint32)    # positive finite, incl. subnormal
    x = bits.view(np.float32)
    extra = np.array([1.0, 1.75, 2.0, 448.0, 57344.0, 3.5, 7.0, 0.875,
                      np.nextafter(np.float32(1.75), np.float32(2)),
                      np.nextafter(np.float32(1.75), np.float32(0)),
                      np.float32(2.0 ** -149), np.float32(2.0 ** -126),
                      np.finfo(np.float32).max], dtype=np.float32)
    pw = np.float32(2.0) ** np.arange(-149, 128, dtype=np.float64)
    return np.concatenate([x, extra, pw.astype(np.float32),
                           (pw * 1.75).astype(np.float32)[np.isfinite(pw * 1.75)]])


@pytest.mark.parametrize("fmt", [oracle.E4M3, oracle.E5M2])
@pytest.mark.parametrize("margin", [0, 1, 3])
def test_compute_bias_brute_force(fmt, margin):
    for a in _fp32_samples(300, 7 + fmt * 10 + margin):
        if not np.isfinite(a):
            continue
        assert oracle.compute_bias(a, fmt, margin) == _brute_force_bias(a, fmt, margin), float(a)


@pytest.mark.parametrize("fmt", [oracle.E4M3, oracle.E5M2])
def test_compute_bias_invariants(fmt):
    fm = Fraction(oracle.fmt_max(fmt))
    for a in _fp32_samples(2000, 99 + fmt):
        b0 = oracle.compute_bias(a, fmt, 0)
        A = Fraction(float(a))
        assert A * Fraction(2) ** b0 <= fm                  # never overflows
        assert A * Fraction(2) ** (b0 + 1) > fm             # and is tight with margin 0
        for m in (1, 3):
            assert oracle.compute_bias(a, fmt, m) == b0 - m  # margin subtracts


def test_compute_bias_special_amax():
    for fmt in (oracle.E4M3, oracle.E5M2):
        for m in (0, 1, 3):
            assert oracle.compute_bias(0.0, fmt, m) == 0
            assert oracle.compute_bias(float("nan"), fmt, m) == 0
            assert oracle.compute_bias(float("inf"), fmt, m) == 0
    # bias range reachable from fp32 inputs
    assert oracle.compute_bias(2.0 ** -149, oracle.E4M3, 0) == 157
    assert oracle.compute_bias(2.0 ** -149, oracle.E5M2, 0) == 164
    assert oracle.compute_bias(float(np.finfo(np.float32).max), oracle.E4M3, 0) == -120
    assert oracle.compute_bias(float(np.finfo(np.float32).max), oracle.E5M2, 0) == -113


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_amax_matches_numpy(dtype):
    g = torch.Generator().manual_seed(5)
    for n in (1, 7, 1000, 65537):
        x = (torch.randn(n, generator=g) * 3).to(dtype)
        ref = np.float32(np.max(np.abs(x.float().numpy())))
        assert oracle.amax(x) == ref


def test_amax_special_cases():
    f = lambda v, dt=torch.float32: oracle.amax(torch.tensor(v, dtype=dt))
    assert f([0.0, -0.0]) == 0.0
    assert f([-5.0, 3.0]) == 5.0
    assert f([1.0, float("-inf"), 2.0]) == np.inf
    assert np.isnan(f([1.0, float("nan"), float("inf")]))
    assert np.isnan(f([float("nan"), 2.0], torch.bfloat16))
    assert f([-2.0 ** -149]) == np.float32(2.0 ** -149)
    assert f([-7.5, 1.0], torch.bfloat16) == 7.5
    assert oracle.amax(np.zeros(0, dtype=np.float32)) == 0.0
