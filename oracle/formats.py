"""Number formats of the DualQuant solver, written out from their definitions.

TEST INFRASTRUCTURE.  This package is the plain, slow fp64 reference that the
CUDA library is checked against.  Only the tests, the smoke check and the
benchmark's CPU-baseline leg may import it; the product path never does.

Every routine works on float64 numpy arrays of real values.  A value "in a
format" is the float64 number that the format's bit pattern stands for.

Sources (the DualQuant pages):
* signed INT4 codebook [-8, 7] with a BF16 scale, and the same codebook with
  E8M0 power-of-two scales of exponent in [-126, 126] (MXINT4):
  daiwk.github.io reproduction note, section "本地复现" (local reproduction).
* MXFP4 = E2M1 codes in blocks of 32 with an E8M0 shared scale; NVFP4 = E2M1
  codes in blocks of 16 with an E4M3 scale: news.yiqijian.com article, section
  "适配 MXFP4 与 NVFP4 块结构".
* The quantizer is a black box on a fixed grid and the scales are projected onto
  the format's admissible set: daiwk note, section "原始论文总结"; trove summary,
  "What it claims".

* The method claims support for the whole MX family (news.yiqijian.com
  article, same section, and the trove summary, "What it claims"); the MX
  element formats beyond MXFP4/MXINT4 are taken from the OCP Microscaling
  format definition: MXFP8 (E4M3 or E5M2 elements), MXFP6 (E2M3 or E3M2),
  MXINT8 (8-bit two's complement), all in blocks of 32 with an E8M0 scale.

Rounding rules that the pages leave open (readings, not quotations):
* BF16 and E4M3 values: round to nearest, ties to even (IEEE default).
* E4M3 saturates at 448 (the OCP "fn" variant has no infinity).
* E2M1 magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6}: nearest, ties to the code with
  an even mantissa bit, saturating at 6; the sign follows the input's sign bit.
* The other float element formats the same way (nearest, ties to even,
  saturating at the largest finite value, sign of zero from the input):
  E4M3 max 448, E5M2 max 57344, E2M3 max 7.5, E3M2 max 28 (all with
  subnormals).  INT8 elements: round half to even, clamp to [-128, 127].
"""
from __future__ import annotations

import numpy as np

BF16_MAX = (2.0 - 2.0 ** -7) * 2.0 ** 127
BF16_MIN_NORMAL = 2.0 ** -126
E4M3_MAX = 448.0
E4M3_MIN_SUB = 2.0 ** -9
E8M0_EMIN, E8M0_EMAX = -126, 126
E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _floor_log2(x: np.ndarray) -> np.ndarray:
    """Exact floor(log2 x) for positive finite float64 ``x`` (via frexp)."""
    _, e = np.frexp(x)
    return e.astype(np.int64) - 1


def round_float_format(x, p: int, emin: int, maxval: float, satfinite: bool) -> np.ndarray:
    """Round ``x`` to the nearest value of a binary float format, ties to even.

    ``p`` significant bits (implicit bit included), normal exponents down to
    ``emin`` with gradual underflow below, largest finite value ``maxval``.
    Overflow goes to ``maxval`` when ``satfinite`` else to infinity.
    """
    x = np.asarray(x, dtype=np.float64)
    ax = np.abs(x)
    out = np.zeros_like(ax)
    nz = ax > 0
    e = np.maximum(_floor_log2(np.where(nz, ax, 1.0)), emin)
    quantum = np.ldexp(1.0, (e - (p - 1)).astype(np.int64))
    k = np.rint(ax / quantum)              # division by a power of two: exact
    v = k * quantum
    big = v > maxval
    v = np.where(big, maxval if satfinite else np.inf, v)
    out = np.where(nz, v, 0.0)
    return np.copysign(out, x)


def round_bf16(x) -> np.ndarray:
    """Round to bfloat16 (8 significant bits, exponent of float32), RNE."""
    return round_float_format(x, 8, -126, BF16_MAX, satfinite=False)


def round_e4m3(x) -> np.ndarray:
    """Round to OCP FP8 E4M3 (bias 7, subnormals, max 448), RNE, saturating."""
    return round_float_format(x, 4, -6, E4M3_MAX, satfinite=True)


def e8m0_ceil(x) -> np.ndarray:
    """Smallest power of two >= x (x > 0), exponent clamped to [-126, 126]."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                     # x = m * 2^e, m in [0.5, 1)
    k = np.where(m == 0.5, e - 1, e).astype(np.int64)
    return np.ldexp(1.0, np.clip(k, E8M0_EMIN, E8M0_EMAX))


def e8m0_nearest(x) -> np.ndarray:
    """Nearest power of two to x > 0 in linear distance; an exact tie goes up.

    For x in [2^k, 2^(k+1)) the midpoint is 1.5 * 2^k.  Exponent clamped to
    [-126, 126].
    """
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                     # x = m * 2^e, x in [2^(e-1), 2^e)
    k = np.where(m < 0.75, e - 1, e).astype(np.int64)
    return np.ldexp(1.0, np.clip(k, E8M0_EMIN, E8M0_EMAX))


def round_e2m1(q) -> np.ndarray:
    """Nearest E2M1 value, ties to the even code, saturating at +-6.

    Returned as float64 values; the sign (also of a zero result) is the sign
    bit of ``q``.
    """
    q = np.asarray(q, dtype=np.float64)
    aq = np.minimum(np.abs(q), 6.0)
    d = np.abs(aq[..., None] - E2M1_GRID)          # distance to each grid value
    best = d.min(axis=-1, keepdims=True)
    cand = d == best
    # among equally near grid values take the one with an even code (index)
    idx = np.where(cand & (np.arange(8) % 2 == 0), np.arange(8), 99).min(axis=-1)
    idx = np.where(idx == 99, np.argmax(cand, axis=-1), idx)
    return np.copysign(E2M1_GRID[idx], q)


def round_int4(q) -> np.ndarray:
    """Round half to even, clamp to the signed INT4 codebook [-8, 7]."""
    return np.clip(np.rint(np.asarray(q, dtype=np.float64)), -8.0, 7.0)


def round_int8(q) -> np.ndarray:
    """Round half to even, clamp to the signed INT8 codebook [-128, 127]."""
    return np.clip(np.rint(np.asarray(q, dtype=np.float64)), -128.0, 127.0)


# Element float formats of the MX family: (exponent bits, mantissa bits, bias,
# largest finite value).  Normal exponents run from 1 - bias; the field of all
# ones is an ordinary exponent in E4M3 (save its NaN code), E2M3 and E3M2 and
# holds Inf/NaN in E5M2.
FP_ELEMENTS = {
    "e4m3": (4, 3, 7, 448.0),
    "e5m2": (5, 2, 15, 57344.0),
    "e2m3": (2, 3, 1, 7.5),
    "e3m2": (3, 2, 3, 28.0),
}


def round_fp_element(q, name: str) -> np.ndarray:
    """Nearest value of an MX float element format, ties to even, saturating."""
    eb, mb, bias, mx = FP_ELEMENTS[name]
    return round_float_format(q, mb + 1, 1 - bias, mx, satfinite=True)


def fp_element_values(name: str) -> np.ndarray:
    """Value of every code of an element format with the sign bit clear
    (index = code); codes beyond the largest finite value are NaN."""
    eb, mb, bias, mx = FP_ELEMENTS[name]
    vals = np.empty(1 << (eb + mb))
    for code in range(1 << (eb + mb)):
        e, m = code >> mb, code & ((1 << mb) - 1)
        if e == 0:
            v = (m / 2.0 ** mb) * 2.0 ** (1 - bias)
        else:
            v = (1.0 + m / 2.0 ** mb) * 2.0 ** (e - bias)
        vals[code] = v if v <= mx else np.nan
    return vals


# --------------------------------------------------------------------------- #
# Encodings of stored values (bit patterns the library writes)
# --------------------------------------------------------------------------- #

def encode_bf16(v) -> np.ndarray:
    """uint16 bit pattern of bf16-representable float64 values."""
    f = np.asarray(v, dtype=np.float64).astype(np.float32)
    return (f.view(np.uint32) >> 16).astype(np.uint16)


def decode_bf16(u) -> np.ndarray:
    return (np.asarray(u, dtype=np.uint32) << 16).view(np.float32).astype(np.float64)


def _e4m3_table() -> np.ndarray:
    vals = np.zeros(128)
    for code in range(128):
        e, m = code >> 3, code & 7
        vals[code] = (m / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7)
    vals[127] = np.nan                       # S.1111.111 is NaN in E4M3 "fn"
    return vals


E4M3_VALUES = _e4m3_table()


def encode_e4m3(v) -> np.ndarray:
    v = np.asarray(v, dtype=np.float64)
    av = np.abs(v)
    idx = np.searchsorted(E4M3_VALUES[:127], av)
    idx = np.minimum(idx, 126)
    if not np.all(E4M3_VALUES[idx] == av):
        raise ValueError("value not representable in E4M3")
    return (idx | np.where(np.signbit(v), 128, 0)).astype(np.uint8)


def decode_e4m3(u) -> np.ndarray:
    u = np.asarray(u, dtype=np.int64)
    return np.where(u & 128, -1.0, 1.0) * E4M3_VALUES[u & 127]


def encode_e8m0(v) -> np.ndarray:
    v = np.asarray(v, dtype=np.float64)
    m, e = np.frexp(v)
    if not np.all(m == 0.5):
        raise ValueError("value not a power of two")
    k = e.astype(np.int64) - 1
    if np.any((k < E8M0_EMIN) | (k > E8M0_EMAX)):
        raise ValueError("exponent out of range")
    return (k + 127).astype(np.uint8)


def decode_e8m0(u) -> np.ndarray:
    return np.ldexp(1.0, np.asarray(u, dtype=np.int64) - 127)


def encode_int4(c) -> np.ndarray:
    """Two's-complement nibble of INT4 values."""
    return (np.asarray(c).astype(np.int64) & 0xF).astype(np.uint8)


def decode_int4(n) -> np.ndarray:
    n = np.asarray(n, dtype=np.int64) & 0xF
    return np.where(n >= 8, n - 16, n).astype(np.float64)


def encode_e2m1(c) -> np.ndarray:
    """E2M1 nibble ``s|ee|m`` of E2M1 values (index into the grid + sign bit)."""
    c = np.asarray(c, dtype=np.float64)
    idx = np.searchsorted(E2M1_GRID, np.abs(c))
    if not np.all(E2M1_GRID[np.minimum(idx, 7)] == np.abs(c)):
        raise ValueError("value not on the E2M1 grid")
    return (idx | np.where(np.signbit(c), 8, 0)).astype(np.uint8)


def decode_e2m1(n) -> np.ndarray:
    n = np.asarray(n, dtype=np.int64)
    return np.where(n & 8, -1.0, 1.0) * E2M1_GRID[n & 7]


def encode_fp_element(v, name: str) -> np.ndarray:
    """Code (sign bit above the magnitude bits) of element-format values."""
    eb, mb, _, _ = FP_ELEMENTS[name]
    vals = fp_element_values(name)
    n = int(np.sum(~np.isnan(vals)))           # finite magnitudes: codes 0 .. n-1
    v = np.asarray(v, dtype=np.float64)
    av = np.abs(v)
    idx = np.minimum(np.searchsorted(vals[:n], av), n - 1)
    if not np.all(vals[idx] == av):
        raise ValueError(f"value not representable in {name}")
    return (idx | np.where(np.signbit(v), 1 << (eb + mb), 0)).astype(np.uint8)


def decode_fp_element(u, name: str) -> np.ndarray:
    eb, mb, _, _ = FP_ELEMENTS[name]
    u = np.asarray(u, dtype=np.int64)
    sign = 1 << (eb + mb)
    return np.where(u & sign, -1.0, 1.0) * fp_element_values(name)[u & (sign - 1)]


def encode_int8(c) -> np.ndarray:
    """Two's-complement byte of INT8 values."""
    return (np.asarray(c).astype(np.int64) & 0xFF).astype(np.uint8)


def decode_int8(u) -> np.ndarray:
    u = np.asarray(u, dtype=np.int64) & 0xFF
    return np.where(u >= 128, u - 256, u).astype(np.float64)


def pack_sixbits(codes: np.ndarray) -> np.ndarray:
    """Pack ``[..., 4k]`` 6-bit codes into ``[..., 3k]`` bytes: four
    consecutive codes form one little-endian 24-bit word, the first code in
    the lowest bits."""
    c = np.asarray(codes, dtype=np.uint32)
    w = c[..., 0::4] | (c[..., 1::4] << 6) | (c[..., 2::4] << 12) | (c[..., 3::4] << 18)
    out = np.empty(w.shape[:-1] + (3 * w.shape[-1],), dtype=np.uint8)
    out[..., 0::3] = w & 0xFF
    out[..., 1::3] = (w >> 8) & 0xFF
    out[..., 2::3] = (w >> 16) & 0xFF
    return out


def unpack_sixbits(b: np.ndarray) -> np.ndarray:
    b = np.asarray(b, dtype=np.uint32)
    w = b[..., 0::3] | (b[..., 1::3] << 8) | (b[..., 2::3] << 16)
    out = np.empty(w.shape[:-1] + (4 * w.shape[-1],), dtype=np.uint8)
    for k in range(4):
        out[..., k::4] = (w >> (6 * k)) & 0x3F
    return out


def pack_nibbles(nib: np.ndarray) -> np.ndarray:
    """Pack ``[..., 2k]`` nibbles into bytes: even column in the low nibble."""
    nib = np.asarray(nib, dtype=np.uint8)
    return (nib[..., 0::2] | (nib[..., 1::2] << 4)).astype(np.uint8)


def unpack_nibbles(b: np.ndarray) -> np.ndarray:
    b = np.asarray(b, dtype=np.uint8)
    out = np.empty(b.shape[:-1] + (2 * b.shape[-1],), dtype=np.uint8)
    out[..., 0::2] = b & 0xF
    out[..., 1::2] = b >> 4
    return out
