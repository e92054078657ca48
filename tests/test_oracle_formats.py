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


# --------------------------------------------------------------------------- #
# The other element formats of the MX family
# --------------------------------------------------------------------------- #

def _grid_from_bits(eb, mb, bias):
    """Magnitudes of all codes of a float element format, written from the
    bit layout independently of the oracle's table (NaN/Inf codes dropped by
    the caller)."""
    out = []
    for e in range(1 << eb):
        for m in range(1 << mb):
            frac = m / (1 << mb)
            out.append(math.ldexp(frac, 1 - bias) if e == 0 else math.ldexp(1 + frac, e - bias))
    return np.array(out)


@pytest.mark.parametrize("name,eb,mb,bias,top,nfinite", [
    ("e4m3", 4, 3, 7, 448.0, 127), ("e5m2", 5, 2, 15, 57344.0, 124),
    ("e2m3", 2, 3, 1, 7.5, 32), ("e3m2", 3, 2, 3, 28.0, 32)])
def test_fp_element_rounding_brute_force(name, eb, mb, bias, top, nfinite):
    grid = _grid_from_bits(eb, mb, bias)[:nfinite]
    assert grid[-1] == top and np.all(np.diff(grid) > 0)
    vals = F.fp_element_values(name)
    assert np.array_equal(vals[:nfinite], grid) and np.all(np.isnan(vals[nfinite:]))
    rng = np.random.default_rng(11)
    mids = (grid[:-1] + grid[1:]) / 2
    x = np.concatenate([grid, mids, np.nextafter(mids, 0), np.nextafter(mids, np.inf),
                        rng.uniform(0, 1.3 * top, 4000), top * np.exp(rng.uniform(-30, 0, 4000)),
                        [top * 1.01, top * 2, 1e30]])
    x = np.concatenate([x, -x])
    got = F.round_fp_element(x, name)
    # brute force: nearest grid magnitude of min(|x|, top); ties to the even code
    ax = np.minimum(np.abs(x), top)
    d = np.abs(ax[:, None] - grid[None, :])
    best = d.min(axis=1, keepdims=True)
    cand = d == best
    idx = np.where(cand & (np.arange(nfinite) % 2 == 0), np.arange(nfinite), 1 << 20).min(axis=1)
    idx = np.where(idx == 1 << 20, np.argmax(cand, axis=1), idx)
    want = np.copysign(grid[idx], x)
    assert np.array_equal(got, want)
    assert np.array_equal(np.signbit(got), np.signbit(x))
    # codes: sign bit above the magnitude bits, round trip
    enc = F.encode_fp_element(want, name)
    assert np.array_equal(enc & ((1 << (eb + mb)) - 1), idx)
    assert np.array_equal(F.decode_fp_element(enc, name), want)


@pytest.mark.parametrize("name,dt", [("e4m3", torch.float8_e4m3fn), ("e5m2", torch.float8_e5m2)])
def test_fp8_elements_match_torch(name, dt):
    # every finite code decodes as torch decodes it
    codes = np.arange(256, dtype=np.uint8)
    tv = torch.from_numpy(codes).view(dt).to(torch.float64).numpy()
    fin = np.isfinite(tv)
    assert np.array_equal(F.decode_fp_element(codes[fin], name), tv[fin])
    # rounding of float32 inputs inside the range matches torch's cast
    top = F.FP_ELEMENTS[name][3]
    rng = np.random.default_rng(12)
    x = (rng.uniform(-top, top, 100000) * np.exp(rng.uniform(-25, 0, 100000))).astype(np.float32)
    want = torch.from_numpy(x).to(dt).to(torch.float64).numpy()
    assert np.array_equal(F.round_fp_element(x.astype(np.float64), name), want)


def test_int8_elements():
    q = np.array([2.5, -2.5, 3.5, 126.5, 127.4, 127.6, 300.0, -127.5, -128.4, -129.0, 0.49])
    assert list(F.round_int8(q)) == [2, -2, 4, 126, 127, 127, 127, -128, -128, -128, 0]
    for v in np.linspace(-200, 200, 801):
        assert F.round_int8(np.array([v]))[0] == max(-128, min(127, round(v)))
    c = np.arange(-128, 128, dtype=np.float64)
    u = F.encode_int8(c)
    assert list(u[:2]) == [0x80, 0x81] and u[128] == 0 and u[-1] == 0x7F
    assert np.array_equal(F.decode_int8(u), c)


def test_six_bit_packing():
    # four codes in one little-endian 24-bit word, the first in the low bits
    assert list(F.pack_sixbits(np.array([1, 2, 3, 4]))) == [0x81, 0x30, 0x10]
    rng = np.random.default_rng(13)
    c = rng.integers(0, 64, (3, 32)).astype(np.uint8)
    p = F.pack_sixbits(c)
    assert p.shape == (3, 24)
    assert np.array_equal(F.unpack_sixbits(p), c)
