"""Pins for the oracle's FP8 codec (decode / RNE-satfinite encode).

The oracle encoder is a nearest-value search over the format's sorted finite
values.  It is pinned here against things that are not itself:
  * hand-written values of the OCP E4M3 / E5M2 definitions (tests/golden);
  * torch's and ml_dtypes' float8 conversions (independent library code),
    exhaustively over all 2^32 fp32 bit patterns;
  * an exhaustive distance-minimisation over all 256 codes (numpy);
  * the round trip of all 256 codes.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle

FMTS = [(oracle.E4M3, "E4M3", torch.float8_e4m3fn), (oracle.E5M2, "E5M2", torch.float8_e5m2)]


def _golden(golden_dir):
    rows = []
    with open(os.path.join(golden_dir, "fp8_format_values.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            fmt, code, val = line.split()
            rows.append((oracle.E4M3 if fmt == "E4M3" else oracle.E5M2, int(code, 16), float(val)))
    return rows


def test_decode_hand_values(golden_dir):
    rows = _golden(golden_dir)
    assert len(rows) >= 20
    for fmt, code, val in rows:
        got = oracle.fp8_decode([code], fmt)[0]
        if math.isnan(val):
            assert math.isnan(got), (fmt, hex(code))
        else:
            assert got == val, (fmt, hex(code), got, val)
            assert math.copysign(1.0, got) == math.copysign(1.0, val), (fmt, hex(code))


@pytest.mark.parametrize("fmt,name,tdt", FMTS)
def test_decode_matches_torch_all_codes(fmt, name, tdt):
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(tdt).to(torch.float64).numpy()
    got = oracle.fp8_decode_table(fmt)
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert np.array_equal(ref[~nan], got[~nan])
    assert np.array_equal(np.signbit(ref[~nan]), np.signbit(got[~nan]))


@pytest.mark.parametrize("fmt,name", [(oracle.E4M3, "float8_e4m3fn"), (oracle.E5M2, "float8_e5m2")])
def test_decode_matches_ml_dtypes_all_codes(fmt, name):
    ml = pytest.importorskip("ml_dtypes")
    ref = np.arange(256, dtype=np.uint8).view(getattr(ml, name)).astype(np.float64)
    got = oracle.fp8_decode_table(fmt)
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert np.array_equal(ref[~nan], got[~nan])


def test_fmt_max_is_largest_finite_code():
    for fmt in (oracle.E4M3, oracle.E5M2):
        t = oracle.fp8_decode_table(fmt)
        assert np.nanmax(t[np.isfinite(t)]) == oracle.fmt_max(fmt)
    assert oracle.fmt_max(oracle.E4M3) == 448.0
    assert oracle.fmt_max(oracle.E5M2) == 57344.0


@pytest.mark.parametrize("fmt,name,tdt", FMTS)
def test_all_256_codes_round_trip(fmt, name, tdt):
    table = oracle.fp8_decode_table(fmt)
    for c in range(256):
        v = table[c]
        if math.isnan(v):
            assert math.isnan(oracle.fp8_decode(oracle.fp8_encode([v], fmt), fmt)[0])
        elif math.isinf(v):
            # infinity exists only in E5M2; it round-trips without saturation,
            # and saturates to +-57344 with it
            assert oracle.fp8_encode([v], fmt, saturate=False)[0] == c
            assert oracle.fp8_encode([v], fmt, saturate=True)[0] == (c & 0x80) | 0x7B
        else:
            assert oracle.fp8_encode([v], fmt, saturate=True)[0] == c, hex(c)
            assert oracle.fp8_encode([v], fmt, saturate=False)[0] == c, hex(c)


def _brute_force_nearest(values, fmt):
    """Exhaustive nearest-of-all-finite-codes search with ties to an even mantissa
    LSB and saturation; written independently of the oracle's binary search."""
    table = oracle.fp8_decode_table(fmt)
    pos = np.array([c for c in range(128) if np.isfinite(table[c])])
    pv = table[pos]
    a = np.abs(values)[:, None]
    d = np.abs(a - pv[None, :])
    best = d.min(axis=1, keepdims=True)
    cand = d == best
    # among tied candidates prefer an even code (= even mantissa LSB)
    score = np.where(cand, np.where(pos[None, :] % 2 == 0, 2, 1), 0)
    pick = pos[np.argmax(score, axis=1)]
    pick = np.where(np.abs(values) > pv.max(), pos[np.argmax(pv)], pick)
    return (pick | np.where(np.signbit(values), 0x80, 0)).astype(np.uint8)


@pytest.mark.parametrize("fmt", [oracle.E4M3, oracle.E5M2])
def test_encoder_matches_brute_force_nearest(fmt):
    table = oracle.fp8_decode_table(fmt)
    fin = np.sort(np.unique(np.abs(table[np.isfinite(table)])))
    mids = (fin[:-1] + fin[1:]) / 2                         # exact ties
    rng = np.random.default_rng(1234)
    # every bf16 bit pattern (as fp32) scaled into the format's range
    bf = (np.arange(65536, dtype=np.uint32) << 16).view(np.float32)
    bf = bf[np.isfinite(bf)].astype(np.float64)
    vals = [fin, -fin, mids, -mids, np.nextafter(mids, 0), np.nextafter(mids, np.inf),
            bf * 2.0 ** -100, bf, rng.standard_normal(20000) * oracle.fmt_max(fmt) / 4,
            rng.standard_normal(20000) * 1e-3, np.array([0.0, -0.0, 1e30, -1e30])]
    v = np.concatenate(vals)
    v = v[np.isfinite(v)]
    v32 = v.astype(np.float32)                               # the oracle codec reads fp32 bits
    ref = _brute_force_nearest(v32.astype(np.float64), fmt)
    for lo in range(0, v32.size, 1 << 16):
        chunk = v32[lo:lo + (1 << 16)]
        got = oracle.encode_f32_bits(chunk.view(np.uint32), fmt, True)
        bad = np.nonzero(got != ref[lo:lo + chunk.size])[0]
        assert bad.size == 0, (chunk[bad[:5]], got[bad[:5]], ref[lo + bad[:5]])


def _is_nan_code(codes, fmt):
    low = codes & 0x7F
    return (low == 0x7F) if fmt == oracle.E4M3 else (low > 0x7C)


@pytest.mark.parametrize("fmt,name,tdt", FMTS)
def test_encoder_matches_torch_exhaustive_fp32(fmt, name, tdt):
    """All 2^32 fp32 bit patterns: the non-saturating oracle mode equals torch's
    RNE conversion byte for byte (NaN compared as NaN).  On every 8th chunk the
    saturating mode is checked too: it differs only where torch overflows (or
    the input is infinite), and there it gives +-fmt_max."""
    chunk = 1 << 26
    max_code = 0x7E if fmt == oracle.E4M3 else 0x7B
    for i, start in enumerate(range(0, 1 << 32, chunk)):
        bits_t = torch.arange(start, start + chunk, dtype=torch.int64).to(torch.int32)
        ref = bits_t.view(torch.float32).to(tdt).view(torch.uint8)
        bits = bits_t.numpy().view(np.uint32)
        got = torch.from_numpy(oracle.encode_f32_bits(bits, fmt, False))
        ref_nan = _is_nan_code(ref, fmt)
        assert torch.equal(ref_nan, _is_nan_code(got, fmt)), start
        ok = (ref == got) | ref_nan
        assert bool(ok.all()), (start, torch.nonzero(~ok)[:5])
        if i % 8 == 0:
            sat = torch.from_numpy(oracle.encode_f32_bits(bits, fmt, True))
            x = bits_t.view(torch.float32)
            ref_inf = (fmt == oracle.E5M2) & ((ref & 0x7F) == 0x7C)
            overflow = (~torch.isnan(x)) & ((ref_nan & ~torch.isnan(x)) | ref_inf)
            want = torch.where(overflow, torch.where(torch.signbit(x), 0x80 | max_code, max_code)
                               .to(torch.uint8), got)
            assert torch.equal(sat, want), start


def test_satfinite_and_special_cases():
    E4, E5 = oracle.E4M3, oracle.E5M2
    enc = lambda v, f: int(oracle.fp8_encode([v], f, True)[0])
    assert enc(448.0, E4) == 0x7E
    assert enc(463.99, E4) == 0x7E
    assert enc(464.0, E4) == 0x7E          # tie between 448 (even) and the NaN slot
    assert enc(1e6, E4) == 0x7E and enc(-1e6, E4) == 0xFE
    assert enc(float("inf"), E4) == 0x7E and enc(float("-inf"), E4) == 0xFE
    assert enc(61440.0, E5) == 0x7B and enc(float("inf"), E5) == 0x7B
    assert enc(-0.0, E4) == 0x80 and enc(0.0, E4) == 0x00
    assert enc(2.0 ** -10, E4) == 0x00     # tie between 0 and 2^-9 -> even (0)
    assert enc(-(2.0 ** -10), E4) == 0x80
    assert enc(3 * 2.0 ** -10, E4) == 0x02  # tie between 1 and 2 (x 2^-9) -> even (2)
    assert enc(2.0 ** -17, E5) == 0x00 and enc(3 * 2.0 ** -17, E5) == 0x02
    assert math.isnan(oracle.fp8_decode(oracle.fp8_encode([float("nan")], E4), E4)[0])
    assert math.isnan(oracle.fp8_decode(oracle.fp8_encode([float("nan")], E5), E5)[0])
