"""Pins of the oracle's number formats against library casts, independent
re-derivations and hand-derived cases (no GPU)."""
import math
import struct

import numpy as np
import pytest
import torch

import oracle as O
from oracle import formats as F


def _all_finite_bf16():
    u = np.arange(1 << 16, dtype=np.uint32)
    v = (u << 16).view(np.float32)
    return v[np.isfinite(v)].astype(np.float64)


def test_bf16_round_trip_all_patterns():
    v = _all_finite_bf16()
    assert np.array_equal(F.round_bf16(v), v)
    assert np.array_equal(F.decode_bf16(F.encode_bf16(v)), v)


def test_bf16_rounding_matches_torch_cast():
    v = _all_finite_bf16()
    v = v[(np.abs(v) < F.BF16_MAX) & (v != 0)]
    s = np.sort(np.unique(np.abs(v)))
    mids = (s[:-1] + s[1:]) / 2.0                       # exact in float32
    f32 = mids.astype(np.float32)
    assert np.array_equal(f32.astype(np.float64), mids)
    nxt = np.nextafter(f32, np.float32(np.inf))
    prv = np.nextafter(f32, np.float32(0))
    rng = np.random.default_rng(7)
    rnd = (rng.standard_normal(200000) * np.exp(rng.uniform(-80, 80, 200000))).astype(np.float32)
    for x in (f32, -f32, nxt, prv, rnd):
        x = x[np.isfinite(x)]
        want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
        got = F.round_bf16(x.astype(np.float64))
        ok = np.isfinite(want)
        assert np.array_equal(got[ok], want[ok])


def test_e4m3_matches_torch_cast():
    codes = np.array([c for c in range(256) if (c & 127) != 127])
    vals = F.decode_e4m3(codes)
    assert np.array_equal(F.round_e4m3(vals), vals)
    assert np.array_equal(F.encode_e4m3(vals[vals != 0]), codes[vals != 0])
    pos = np.sort(np.unique(np.abs(vals)))
    mids = (pos[:-1] + pos[1:]) / 2.0
    rng = np.random.default_rng(8)
    rnd = rng.uniform(-448, 448, 100000) * np.exp(rng.uniform(-12, 0, 100000))
    for x in (mids, -mids, np.nextafter(mids, 0), np.nextafter(mids, 1e9), rnd):
        x32 = np.clip(x, -448, 448).astype(np.float32)
        want = torch.from_numpy(x32).to(torch.float8_e4m3fn).to(torch.float64).numpy()
        assert np.array_equal(F.round_e4m3(x32.astype(np.float64)), want)
    # saturation: above 448 (including past the 464 midpoint) stays at 448
    assert np.array_equal(F.round_e4m3(np.array([449.0, 464.0, 470.0, 1e6])), [448.0] * 4)


def test_e2m1_hand_cases():
    # (input, expected) from the E2M1 grid {0,.5,1,1.5,2,3,4,6}, ties to the even code
    cases = [(0.25, 0.0), (0.2499, 0.0), (0.2501, 0.5), (0.75, 1.0), (1.25, 1.0),
             (1.75, 2.0), (2.5, 2.0), (2.51, 3.0), (3.5, 4.0), (5.0, 4.0), (5.01, 6.0),
             (6.5, 6.0), (100.0, 6.0), (-0.75, -1.0), (-5.0, -4.0), (0.0, 0.0)]
    for x, y in cases:
        assert F.round_e2m1(np.array([x]))[0] == y, (x, y)
    z = F.round_e2m1(np.array([-0.1, 0.1]))
    assert z[0] == 0 and np.signbit(z[0]) and not np.signbit(z[1])
    assert list(F.encode_e2m1(z)) == [8, 0]


def test_e2m1_equals_binary_rounding_with_one_mantissa_bit():
    # E2M1 = 2 significant bits, minimum normal exponent 0, max 6: a second,
    # independent construction of the same rounding
    rng = np.random.default_rng(9)
    q = np.concatenate([rng.uniform(-8, 8, 100000), np.arange(-32, 33) / 4.0])
    assert np.array_equal(F.round_e2m1(q), F.round_float_format(q, 2, 0, 6.0, True))


def test_int4_half_even_matches_python_round():
    rng = np.random.default_rng(10)
    q = np.concatenate([rng.uniform(-9, 9, 20000), np.arange(-20, 21) / 2.0])
    want = np.array([min(7, max(-8, round(float(x)))) for x in q], dtype=np.float64)
    assert np.array_equal(F.round_int4(q), want)


def test_e8m0_ceil_against_log2():
    rng = np.random.default_rng(11)
    x = np.exp(rng.uniform(-80, 80, 20000))
    want = np.array([2.0 ** math.ceil(math.log2(v)) for v in x])
    assert np.array_equal(F.e8m0_ceil(x), want)
    for k in (-126, -3, 0, 5, 126):
        p = 2.0 ** k
        assert F.e8m0_ceil(np.array([p]))[0] == p
        if k < 126:
            assert F.e8m0_ceil(np.array([np.nextafter(p, 1e300)]))[0] == 2 * p
    assert F.e8m0_ceil(np.array([1e-45]))[0] == 2.0 ** -126      # clamp
    assert F.e8m0_ceil(np.array([1e40]))[0] == 2.0 ** 126


def test_e8m0_nearest_brute_force():
    rng = np.random.default_rng(12)
    x = np.concatenate([np.exp(rng.uniform(-60, 60, 3000)),
                        1.5 * 2.0 ** np.arange(-20, 20)])        # exact ties
    grid = 2.0 ** np.arange(-126, 127)
    for v in x:
        d = np.abs(v - grid)
        best = grid[d == d.min()].max()                           # ties go up
        assert F.e8m0_nearest(np.array([v]))[0] == best


def test_encodings_round_trip():
    e = np.arange(1, 254)
    assert np.array_equal(F.encode_e8m0(F.decode_e8m0(e)), e)
    n = np.arange(16)
    assert np.array_equal(F.encode_int4(F.decode_int4(n)), n)
    assert np.array_equal(F.encode_e2m1(F.decode_e2m1(n)), n)
    nib = np.random.default_rng(1).integers(0, 16, (3, 10)).astype(np.uint8)
    assert np.array_equal(F.unpack_nibbles(F.pack_nibbles(nib)), nib)
    assert F.pack_nibbles(np.array([[0x3, 0xA]]))[0, 0] == 0xA3   # even column low


def test_bf16_encoding_bit_pattern():
    # 1.0 = 0x3F80, -2.0 = 0xC000, 2^-126 = 0x0080
    assert list(F.encode_bf16(np.array([1.0, -2.0, 2.0 ** -126]))) == [0x3F80, 0xC000, 0x0080]
    # struct-based check of a few random patterns
    for v in (0.015625, 3.140625, -0.0009765625):
        want = struct.unpack(">I", struct.pack(">f", v))[0] >> 16
        assert F.encode_bf16(np.array([v]))[0] == want
