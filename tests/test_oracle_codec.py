"""Pins of the oracle's E4M3 codec and BF16 rounding against the number
formats' own definitions and against independent implementations
(ml_dtypes, torch), never against the oracle itself."""
import math
import os
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle


def _golden_points(golden_dir):
    rows = []
    with open(os.path.join(golden_dir, "e4m3_points.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            expr, byte = line.split()[:2]
            rows.append((float(eval(expr)), int(byte, 16), line))
    return rows


def test_golden_points(golden_dir):
    pts = _golden_points(golden_dir)
    assert len(pts) >= 25
    vals = np.array([p[0] for p in pts], dtype=np.float32)
    got = oracle.e4m3_encode(vals)
    for (v, want, line), g in zip(pts, got):
        assert int(g) == want, f"{line}: got {int(g):#04x}"


def test_decode_all_patterns_match_ml_dtypes():
    table = oracle.e4m3_decode_table()
    ref = np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    nan = np.isnan(ref)
    assert list(np.nonzero(nan)[0]) == [0x7F, 0xFF]
    assert np.array_equal(np.isnan(table), nan)
    assert np.array_equal(table[~nan], ref[~nan])
    # sign of zero
    assert math.copysign(1.0, table[0x80]) == -1.0


def test_decode_closed_forms():
    t = oracle.e4m3_decode_table()
    for b in range(256):
        s, e, m = b >> 7, (b >> 3) & 15, b & 7
        if e == 15 and m == 7:
            continue
        mag = Fraction(m, 8) * Fraction(2) ** -6 if e == 0 else (1 + Fraction(m, 8)) * Fraction(2) ** (e - 7)
        assert Fraction(t[b]) == (-mag if s else mag)
    assert t[0x7E] == 448.0 and t[0x01] == 2.0 ** -9 and t[0x08] == 2.0 ** -6


def test_roundtrip_all_finite_patterns():
    codes = np.array([b for b in range(256) if b not in (0x7F, 0xFF)], dtype=np.uint8)
    vals = oracle.e4m3_decode(codes).astype(np.float32)
    back = oracle.e4m3_encode(vals)
    assert np.array_equal(back, codes)
    nan_codes = oracle.e4m3_encode(np.array([np.nan, -np.nan], dtype=np.float32))
    assert set(int(c) & 0x7F for c in nan_codes) == {0x7F}


def test_monotone_over_finite_codes():
    t = oracle.e4m3_decode_table()
    pos = t[0x00:0x7F]
    assert np.all(np.diff(pos) > 0)
    neg = t[0x80:0xFF]
    assert np.all(np.diff(neg) < 0)


def _sweep_values():
    rng = np.random.default_rng(123)
    grid = oracle.e4m3_decode_table()[0:0x7F]
    mids = (grid[:-1] + grid[1:]) / 2.0
    vals = [grid, mids]
    # one binary32 ulp either side of every value and every midpoint
    g32 = np.concatenate([grid, mids]).astype(np.float32)
    vals.append(np.nextafter(g32, np.float32(np.inf)))
    vals.append(np.nextafter(g32, np.float32(0)))
    # random binary32 values over the whole finite range, log-uniform
    vals.append(np.exp2(rng.uniform(-14, np.log2(448.0), 200_000)))
    v = np.concatenate([np.asarray(a, dtype=np.float64) for a in vals]).astype(np.float32)
    v = v[(v <= 448.0) & (v >= 0)]
    return np.concatenate([v, -v])


def test_encode_matches_ml_dtypes_in_range():
    """In range (|v| <= 448) the saturating and the non-saturating casts agree,
    so ml_dtypes' RNE cast is an independent reference."""
    v = _sweep_values()
    got = oracle.e4m3_encode(v)
    ref = v.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, [(float(v[i]), hex(got[i]), hex(ref[i])) for i in bad[:10]]


def test_encode_matches_torch_in_range():
    v = _sweep_values()
    got = oracle.e4m3_encode(v)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got, ref)


def test_saturation():
    big = np.array([448.0, 448.0001, 463.9, 464.0, 464.1, 480.0, 1e6, 3.4e38, np.inf],
                   dtype=np.float32)
    assert np.all(oracle.e4m3_encode(big) == 0x7E)
    assert np.all(oracle.e4m3_encode(-big) == 0xFE)


def _bf16_exact(v: Fraction) -> int:
    """Nearest-even BF16 bits of an exact rational (test-side, independent)."""
    if v == 0:
        return 0
    sign = 0x8000 if v < 0 else 0
    a = abs(v)
    E = math.floor(math.log2(a))
    while Fraction(2) ** E > a:
        E -= 1
    while Fraction(2) ** (E + 1) <= a:
        E += 1
    E = max(E, -126)
    q = Fraction(2) ** (E - 7)
    r = a / q
    fl = r.numerator // r.denominator
    d = r - fl
    n = fl + 1 if (d > Fraction(1, 2) or (d == Fraction(1, 2) and fl % 2 == 1)) else fl
    res = n * q
    if res >= Fraction(2) ** 128:
        return sign | 0x7F80
    f = np.float32(float(res))
    assert Fraction(float(f)) == res
    return sign | int(f.view(np.uint32) >> 16)


def test_bf16_rounding_of_float32_matches_torch():
    rng = np.random.default_rng(5)
    v = np.concatenate([
        rng.standard_normal(100_000).astype(np.float32),
        np.exp2(rng.uniform(-133, 127, 50_000)).astype(np.float32),
        # exact ties: 8 significant bits plus a half
        (np.arange(1, 2000, dtype=np.float32) * 2 + 1) * np.float32(2.0 ** -9) + 1,
    ])
    got = oracle.bf16_from_double(v.astype(np.float64))
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, ref)


def test_bf16_rounding_is_single_from_double():
    """A value just above a BF16 tie that binary32 would round onto the tie:
    rounding once from the double must go up, double rounding would go down."""
    v = 1.0 + 2.0 ** -8 + 2.0 ** -30
    assert int(oracle.bf16_from_double(np.array([v]))[0]) == 0x3F81
    rng = np.random.default_rng(9)
    vals = rng.standard_normal(3000) * np.exp2(rng.integers(-40, 40, 3000))
    got = oracle.bf16_from_double(vals)
    for x, g in zip(vals, got):
        assert int(g) == _bf16_exact(Fraction(float(x)))
    # subnormal and overflow edges
    assert int(oracle.bf16_from_double(np.array([2.0 ** -133]))[0]) == 0x0001
    assert int(oracle.bf16_from_double(np.array([2.0 ** -134]))[0]) == 0x0000  # tie to even
    assert int(oracle.bf16_from_double(np.array([3.0 * 2.0 ** -135]))[0]) == 0x0001
    assert int(oracle.bf16_from_double(np.array([2.0 ** 128 * (1 - 2.0 ** -9)]))[0]) == 0x7F80
    assert int(oracle.bf16_from_double(np.array([2.0 ** 127 * (2 - 2.0 ** -7)]))[0]) == 0x7F7F


@pytest.mark.parametrize("mistake", ["truncate", "ties_away", "no_saturate"])
def test_pins_catch_planted_codec_mistakes(mistake):
    """Plants a plausible mistake in a Python copy of the codec (on the CPU)
    and checks that the independent references used above reject it."""
    def broken(v):
        a = abs(float(v))
        if mistake != "no_saturate" and a >= 448:
            return 448.0
        if a == 0:
            return 0.0
        E = max(math.floor(math.log2(a)), -6)
        q = 2.0 ** (E - 3)
        r = a / q
        if mistake == "truncate":
            n = math.floor(r)
        elif mistake == "ties_away":
            n = math.floor(r + 0.5)
        else:
            n = round(r)
        return math.copysign(n * q, v)
    v = _sweep_values()[:5000]
    v = np.concatenate([v, np.float32([464.0, 1000.0])])
    ref = np.clip(v, -448, 448).astype(ml_dtypes.float8_e4m3fn).astype(np.float64)
    out = np.array([broken(x) for x in v])
    assert not np.array_equal(out, ref)
