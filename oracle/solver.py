"""DualQuant dual-scale solver, written out step by step in float64.

TEST INFRASTRUCTURE.  Plain, slow and meant to be read against the pages; only
the tests, the smoke check and the benchmark's CPU-baseline leg use it.

The method (DualQuant pages):
* Model of a weight matrix, daiwk reproduction note, section "核心公式",
  eq. (1):  W ~= D_a Q(D_a^-1 W D_b^-1) D_b  with outer inverse scales
  a = alpha^-1 (one per row) and b = beta^-1 (one per column).
* Closed-form updates with the codes held fixed, same section, eq. (2):
  a_i <- Pi_Fa( sum_j W_ij R_ij / sum_j R_ij^2 ),  R = Qhat D_b,
  b_j <- Pi_Fb( sum_i W_ij S_ij / sum_i S_ij^2 ),  S = D_a Qhat.
* Order and conventions, text under eq. (2): re-quantize after the row update,
  then solve the column update and re-quantize again; a slice whose codes are
  all zero keeps scale 1; what is projected is the inverse scale.
* The solver's inputs are only the weights, the format's quantizer and scale
  set, an iteration count T and an initialization (trove summary, "How to use
  it"); it never sees activations (daiwk note, "本地复现").
* Activation side, eq. (1) second half: X W^T ~= (X D_b) Qhat^T D_a, i.e. the
  activation is multiplied by b and then quantized (trove summary, "How to use
  it": beta is applied inside the activation-quantization kernel).

Readings taken where the pages are silent (each also listed in the design notes):
* Inner copies equal the (synced) outer copies, so the grid input is W/(a b^T).
* Pi_F is the nearest admissible value in linear distance: with the codes fixed
  the objective in one scale is den * (x - x*)^2 + const, so the nearest value
  of F is the exact constrained minimiser.  BF16: round to nearest even,
  clamped to the normal range [2^-126, max].  E8M0: exponent in [-126, 126],
  midpoint 1.5 * 2^k, an exact tie goes up.
* Group quantizer Q: per row and group of G consecutive columns, m = max|Y|;
  m == 0 gives the scale 1.0; else s = P_grp(m / qmax) with
  - BF16: round to nearest even, clamped to [2^-126, max];
  - E8M0: round up to a power of two (the smallest s with m/s <= qmax), clamp;
  - E4M3: round to nearest even, saturating at 448; a positive value that
    rounds to 0 becomes the smallest subnormal 2^-9.
  Codes c = round(Y / (s * ts)) on the grid (INT4: half to even, clamp [-8,7];
  E2M1: nearest, ties to even code, saturate 6; the other MX element formats
  likewise: INT8 clamps to [-128,127], float elements saturate at their
  largest finite value).  Qhat = c * s * ts.
* NVFP4 second-level (tensor) scale for weights: ts = 2^ceil(log2(amax(W) /
  (448 * 6))), fixed from the input W at the start; ts = 1 for every other
  format and for activations.
* MSE = sum (W - D_a Qhat D_b)^2 / (rows * cols).  mse_trace[0] is the
  initial state, mse_trace[t] the state after iteration t; mse_half[t-1] the
  state right after the row half-step of iteration t.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from . import formats as F


# largest code magnitude of each element format (the grid's qmax)
QMAX = {"int4": 7.0, "e2m1": 6.0, "int8": 127.0, "e4m3": 448.0, "e5m2": 57344.0,
        "e2m3": 7.5, "e3m2": 28.0}
# stored bits per code
CODE_BITS = {"int4": 4, "e2m1": 4, "int8": 8, "e4m3": 8, "e5m2": 8, "e2m3": 6, "e3m2": 6}


@dataclass(frozen=True)
class Format:
    codes: str            # a key of QMAX
    group: int            # G, consecutive columns sharing a scale
    gscale: str           # "bf16" | "e8m0" | "e4m3"
    oscale: str           # "bf16" | "e8m0"   (set of the outer scales a, b)
    tensor_scale_auto: bool = False

    @property
    def qmax(self) -> float:
        return QMAX[self.codes]

    @property
    def code_bits(self) -> int:
        return CODE_BITS[self.codes]


PRESETS = {
    # daiwk note, 本地复现: signed INT4 [-8,7] with BF16 scales; Table 1 uses G64.
    "int4_bf16": Format("int4", 64, "bf16", "bf16"),
    # same codebook, E8M0 power-of-two scales, exponent in [-126, 126].
    "mxint4": Format("int4", 32, "e8m0", "e8m0"),
    # news article: MXFP4 = E2M1, 32-element blocks, E8M0 shared scale.
    "mxfp4": Format("e2m1", 32, "e8m0", "e8m0"),
    # news article: NVFP4 = E2M1, 16-element blocks, E4M3 scale; BF16 outer scales.
    "nvfp4": Format("e2m1", 16, "e4m3", "bf16", tensor_scale_auto=True),
    # the rest of the MX family (the pages claim it; element formats from the
    # OCP Microscaling definition): 32-element blocks, E8M0 scales
    "mxfp8_e4m3": Format("e4m3", 32, "e8m0", "e8m0"),
    "mxfp8_e5m2": Format("e5m2", 32, "e8m0", "e8m0"),
    "mxfp6_e2m3": Format("e2m3", 32, "e8m0", "e8m0"),
    "mxfp6_e3m2": Format("e3m2", 32, "e8m0", "e8m0"),
    "mxint8": Format("int8", 32, "e8m0", "e8m0"),
    # the scale-set variant: MX blocks (E8M0 group scales) with BF16 outer
    # scales (daiwk note, 本地复现: the reproduction selects the scale format
    # with a command-line flag, so group and outer sets are a choice)
    "mxint4_bf16outer": Format("int4", 32, "e8m0", "bf16"),
    "mxfp4_bf16outer": Format("e2m1", 32, "e8m0", "bf16"),
}


def preset(name: str, group: int | None = None) -> Format:
    f = PRESETS[name]
    if group is not None and group != f.group:
        f = Format(f.codes, group, f.gscale, f.oscale, f.tensor_scale_auto)
    return f


# --------------------------------------------------------------------------- #
# Projections
# --------------------------------------------------------------------------- #

def project_group_scale(g: np.ndarray, fmt: Format) -> np.ndarray:
    """P_grp: admissible group scale for g = m / qmax (g > 0)."""
    if fmt.gscale == "bf16":
        return np.clip(F.round_bf16(g), F.BF16_MIN_NORMAL, F.BF16_MAX)
    if fmt.gscale == "e8m0":
        return F.e8m0_ceil(g)
    if fmt.gscale == "e4m3":
        s = F.round_e4m3(g)
        return np.where(s == 0.0, F.E4M3_MIN_SUB, s)
    raise ValueError(fmt.gscale)


def project_outer(x: np.ndarray, fmt: Format) -> np.ndarray:
    """Pi_F for the outer inverse scales (x > 0): nearest admissible value."""
    if fmt.oscale == "bf16":
        return np.clip(F.round_bf16(x), F.BF16_MIN_NORMAL, F.BF16_MAX)
    if fmt.oscale == "e8m0":
        return F.e8m0_nearest(x)
    raise ValueError(fmt.oscale)


def round_codes(q: np.ndarray, fmt: Format) -> np.ndarray:
    if fmt.codes == "int4":
        return F.round_int4(q)
    if fmt.codes == "int8":
        return F.round_int8(q)
    if fmt.codes == "e2m1":
        return F.round_e2m1(q)
    return F.round_fp_element(q, fmt.codes)


def tensor_scale(W: np.ndarray, fmt: Format) -> float:
    """NVFP4 weight tensor scale 2^ceil(log2(amax / (448 * qmax))); else 1."""
    if not fmt.tensor_scale_auto:
        return 1.0
    amax = float(np.max(np.abs(W))) if W.size else 0.0
    if amax == 0.0:
        return 1.0
    return float(F.e8m0_ceil(amax / (F.E4M3_MAX * fmt.qmax)))


# --------------------------------------------------------------------------- #
# The black-box group quantizer Q
# --------------------------------------------------------------------------- #

def quantize(Y: np.ndarray, fmt: Format, ts: float = 1.0):
    """Q(Y) per row and group of G columns.

    Returns (codes, scales): codes [rows, cols] as grid values, scales
    [rows, cols/G] as the stored group scale values (without ts).
    """
    Y = np.asarray(Y, dtype=np.float64)
    rows, cols = Y.shape
    G = fmt.group
    assert cols % G == 0
    Yg = Y.reshape(rows, cols // G, G)
    m = np.abs(Yg).max(axis=2)
    pos = m > 0
    s = np.where(pos, project_group_scale(np.where(pos, m / (fmt.qmax * ts), 1.0), fmt), 1.0)
    c = round_codes(Yg / (s * ts)[..., None], fmt)
    return c.reshape(rows, cols), s


def dequantize(c: np.ndarray, s: np.ndarray, fmt: Format, ts: float = 1.0) -> np.ndarray:
    rows, cols = c.shape
    G = fmt.group
    return (c.reshape(rows, cols // G, G) * (s * ts)[..., None]).reshape(rows, cols)


def inner(W: np.ndarray, a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Grid input D_a^-1 W D_b^-1 (inner copies equal to the outer ones)."""
    return W / (a[:, None] * b[None, :])


def qhat(W, a, b, fmt, ts=1.0):
    c, s = quantize(inner(W, a, b), fmt, ts)
    return dequantize(c, s, fmt, ts), c, s


def mse(W, Qh, a, b) -> float:
    R = W - a[:, None] * Qh * b[None, :]
    return float(np.sum(R * R) / W.size)


# --------------------------------------------------------------------------- #
# Closed-form block updates (eq. (2))
# --------------------------------------------------------------------------- #

def row_update(W, Qh, b, fmt):
    """a_i <- Pi(sum_j W_ij R_ij / sum_j R_ij^2), R = Qhat D_b; zero slice -> 1.

    Returns (a_new, x_pre) with x_pre the unprojected ratio (nan on zero slices).
    """
    R = Qh * b[None, :]
    num = np.sum(W * R, axis=1)
    den = np.sum(R * R, axis=1)
    pos = den > 0
    x = np.where(pos, num / np.where(pos, den, 1.0), np.nan)
    a = np.where(pos, project_outer(np.where(pos, x, 1.0), fmt), 1.0)
    return a, x


def col_update(W, Qh, a, fmt):
    """b_j <- Pi(sum_i W_ij S_ij / sum_i S_ij^2), S = D_a Qhat; zero slice -> 1."""
    S = a[:, None] * Qh
    num = np.sum(W * S, axis=0)
    den = np.sum(S * S, axis=0)
    pos = den > 0
    x = np.where(pos, num / np.where(pos, den, 1.0), np.nan)
    b = np.where(pos, project_outer(np.where(pos, x, 1.0), fmt), 1.0)
    return b, x


# --------------------------------------------------------------------------- #
# Block coordinate descent
# --------------------------------------------------------------------------- #

def solve(W, fmt: Format, T: int, a0=None, b0=None):
    """DualQuant solve: T iterations of row update, re-quantize, column
    update, re-quantize (the flowchart of the daiwk note and the trove summary).
    """
    W = np.asarray(W, dtype=np.float64)
    rows, cols = W.shape
    a = np.ones(rows) if a0 is None else np.asarray(a0, dtype=np.float64).copy()
    b = np.ones(cols) if b0 is None else np.asarray(b0, dtype=np.float64).copy()
    ts = tensor_scale(W, fmt)
    Qh, c, s = qhat(W, a, b, fmt, ts)
    trace, half = [mse(W, Qh, a, b)], []
    for _ in range(T):
        a, xa = row_update(W, Qh, b, fmt)
        Qh, c, s = qhat(W, a, b, fmt, ts)
        half.append(mse(W, Qh, a, b))
        b, xb = col_update(W, Qh, a, fmt)
        Qh, c, s = qhat(W, a, b, fmt, ts)
        trace.append(mse(W, Qh, a, b))
    return dict(a=a, b=b, codes=c, scales=s, ts=ts, qhat=Qh,
                mse_trace=np.array(trace), mse_half=np.array(half))


def act_rescale_quant(X, b, fmt: Format):
    """Q_act(X D_b): multiply each input channel by b_j, then group-quantize
    with ts = 1.  Returns (codes, scales) as values."""
    X = np.asarray(X, dtype=np.float64)
    return quantize(X * np.asarray(b, dtype=np.float64)[None, :], fmt, 1.0)


# --------------------------------------------------------------------------- #
# Stored form (what the library writes)
# --------------------------------------------------------------------------- #

def encode_codes(c: np.ndarray, fmt: Format) -> np.ndarray:
    """Stored codes: 4-bit codes two per byte (even column low), 8-bit codes
    one per byte, 6-bit codes four per three bytes."""
    if fmt.codes == "int4":
        return F.pack_nibbles(F.encode_int4(c))
    if fmt.codes == "e2m1":
        return F.pack_nibbles(F.encode_e2m1(c))
    if fmt.codes == "int8":
        return F.encode_int8(c)
    u = F.encode_fp_element(c, fmt.codes)
    return F.pack_sixbits(u) if fmt.code_bits == 6 else u


def encode_scales(s: np.ndarray, fmt: Format) -> np.ndarray:
    if fmt.gscale == "bf16":
        return F.encode_bf16(s)
    if fmt.gscale == "e8m0":
        return F.encode_e8m0(s)
    return F.encode_e4m3(s)


def decode_codes(packed: np.ndarray, fmt: Format) -> np.ndarray:
    if fmt.codes == "int4":
        return F.decode_int4(F.unpack_nibbles(packed))
    if fmt.codes == "e2m1":
        return F.decode_e2m1(F.unpack_nibbles(packed))
    if fmt.codes == "int8":
        return F.decode_int8(packed)
    u = F.unpack_sixbits(packed) if fmt.code_bits == 6 else packed
    return F.decode_fp_element(u, fmt.codes)


def decode_scales(u: np.ndarray, fmt: Format) -> np.ndarray:
    if fmt.gscale == "bf16":
        return F.decode_bf16(u)
    if fmt.gscale == "e8m0":
        return F.decode_e8m0(u)
    return F.decode_e4m3(u)


# --------------------------------------------------------------------------- #
# Two-level absmax quantization (msModelSlim "DualScale" page)
# --------------------------------------------------------------------------- #

MXFP4_MAX_NORMAL = 6.0


def two_level_quant(X, dual_block: int, inner: Format):
    """Two-level absmax quant-dequant (msmodelslim.readthedocs.io, DualScale,
    "算法原理" 1(a)-(c) and 2(a)-(b)).

    Per row and block of ``dual_block`` consecutive columns (the last block
    may be shorter): outer scale S = max|X_block| / MXFP4_MAX_NORMAL, the
    block divided by S, quantized with the inner format (our Q: E8M0 group
    scale rounded up, codes nearest-even) and multiplied back by S.

    Readings (the page fixes no precision): S and X/S are float32 values
    (IEEE float32 division, i.e. the correctly rounded quotient: float64
    division followed by rounding to float32 gives the same value, since
    53 >= 2*24 + 2); an all-zero block takes S = 1; the reconstruction is the
    float32 product (c * s) * S.

    Returns (codes, inner_scales, outer_scales [rows, ceil(cols/dual_block)],
    qdq) with codes/scales as values and qdq as float64 holding float32
    values.
    """
    X = np.asarray(X, dtype=np.float64)
    rows, cols = X.shape
    nb = -(-cols // dual_block)
    S = np.ones((rows, nb))
    Y = np.empty_like(X)
    for k in range(nb):
        blk = X[:, k * dual_block:(k + 1) * dual_block]
        m = np.abs(blk).max(axis=1)
        s = np.where(m > 0, (m / MXFP4_MAX_NORMAL).astype(np.float32).astype(np.float64), 1.0)
        S[:, k] = s
        Y[:, k * dual_block:(k + 1) * dual_block] = (blk / s[:, None]).astype(np.float32)
    c, s_in = quantize(Y, inner, 1.0)
    inner_vals = dequantize(c, s_in, inner, 1.0)             # c * s: exact
    Sfull = np.repeat(S, dual_block, axis=1)[:, :cols]
    qdq = (inner_vals * Sfull).astype(np.float32).astype(np.float64)
    return c, s_in, S, qdq


# --------------------------------------------------------------------------- #
# The inference step: block-scaled W4A4 product
# --------------------------------------------------------------------------- #

def w4a4_gemm(cx, sx, cw, sw, a, fmt: Format, ts_w: float = 1.0):
    """out[m, n] = a_n * sum_k Qx[m, k] Qw[n, k] with Qx = dequantize(cx, sx),
    Qw = dequantize(cw, sw, ts_w) (eq. (1) of the daiwk note: X W^T ~= (X D_b)
    Qhat^T D_a).  Codes and scales as values; float64.  ts_w is the weights'
    tensor scale (NVFP4: E2M1 codes with an E4M3 scale per 16 elements, news
    article "适配 MXFP4 与 NVFP4 块结构", times the per-matrix power of two the
    solve takes; 1 otherwise); the activations are quantized with ts = 1."""
    Xq = dequantize(np.asarray(cx, dtype=np.float64), np.asarray(sx, dtype=np.float64), fmt)
    Wq = dequantize(np.asarray(cw, dtype=np.float64), np.asarray(sw, dtype=np.float64), fmt, ts_w)
    return (Xq @ Wq.T) * np.asarray(a, dtype=np.float64)[None, :]
