"""Seeded synthetic inputs shared by the oracle side and the CUDA side.

This module only draws numbers and lays out workload shapes.  It holds none of
the dual-scale method's arithmetic (no quantizer, no scale projection, no
update rule), so both the oracle tests and the CUDA path can read the same
buffers without sharing any of the method.

Generator: counter-based SplitMix64 (Steele, Lea, Flood, "Fast splittable
pseudorandom number generators", OOPSLA 2014; mixing constants as published by
Vigna).  Draw ``i`` of a stream with key ``k`` is ``mix(k + (i + 1) * GOLDEN)``.
Uniforms take the top 53 bits, offset by half a step so that they never hit 0.
Normals use the cosine branch of Box-Muller (two draws each).  Student-t with
4 degrees of freedom is ``Z / sqrt(V / 4)`` with ``V = -2 ln(U1 U2)`` a
chi-square(4) draw (four draws each).

Workload shapes follow the linear layers of the models the DualQuant pages run
on (SmolLM2-135M, Llama-3.1-8B, Llama-3.1-70B).  Those checkpoints and their
datasets are not available, so seeded weights of the same shapes and of the
stated distributions stand in for them.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import torch

GOLDEN = 0x9E3779B97F4A7C15
MIX1 = 0xBF58476D1CE4E5B9
MIX2 = 0x94D049BB133111EB
BASE_SEED = 42
_MASK64 = (1 << 64) - 1


def _signed(v: int) -> int:
    v &= _MASK64
    return v - (1 << 64) if v >= (1 << 63) else v


def _srl(z: torch.Tensor, s: int) -> torch.Tensor:
    """Logical right shift of int64 bit patterns."""
    return (z >> s) & ((1 << (64 - s)) - 1)


def mix64(z: torch.Tensor) -> torch.Tensor:
    """SplitMix64 finaliser on int64 tensors (two's-complement wrap-around)."""
    z = (z ^ _srl(z, 30)) * _signed(MIX1)
    z = (z ^ _srl(z, 27)) * _signed(MIX2)
    return z ^ _srl(z, 31)


def mix64_int(z: int) -> int:
    """The same finaliser on a Python int (for key derivation)."""
    z &= _MASK64
    z = ((z ^ (z >> 30)) * MIX1) & _MASK64
    z = ((z ^ (z >> 27)) * MIX2) & _MASK64
    return z ^ (z >> 31)


def stream_key(*ids: int) -> int:
    """Key of the substream named by a tuple of small integers."""
    k = BASE_SEED
    for v in ids:
        k = mix64_int((k ^ (v & _MASK64)) + GOLDEN)
    return k


_CHUNK = 1 << 24


def raw_bits(key: int, n: int, offset: int = 0, device="cpu") -> torch.Tensor:
    """Draws ``offset .. offset+n-1`` of stream ``key`` as int64 bit patterns."""
    i = torch.arange(offset + 1, offset + n + 1, dtype=torch.int64, device=device)
    return mix64(i * _signed(GOLDEN) + _signed(key))


def uniform(key: int, n: int, offset: int = 0, device="cpu") -> torch.Tensor:
    """fp64 uniforms in (0, 1)."""
    out = torch.empty(n, dtype=torch.float64, device=device)
    for c0 in range(0, n, _CHUNK):
        c1 = min(n, c0 + _CHUNK)
        z = raw_bits(key, c1 - c0, offset + c0, device)
        out[c0:c1] = (_srl(z, 11).to(torch.float64) + 0.5) * (2.0 ** -53)
    return out


def normal(key: int, n: int, device="cpu") -> torch.Tensor:
    """fp64 standard normals (Box-Muller, cosine branch, draws 2i and 2i+1)."""
    out = torch.empty(n, dtype=torch.float64, device=device)
    for c0 in range(0, n, _CHUNK):
        c1 = min(n, c0 + _CHUNK)
        u = uniform(key, 2 * (c1 - c0), 2 * c0, device).view(-1, 2)
        out[c0:c1] = torch.sqrt(-2.0 * torch.log(u[:, 0])) * torch.cos(2.0 * math.pi * u[:, 1])
    return out


def student_t4(key: int, n: int, device="cpu") -> torch.Tensor:
    """fp64 Student-t draws with 4 degrees of freedom (draws 4i .. 4i+3)."""
    out = torch.empty(n, dtype=torch.float64, device=device)
    for c0 in range(0, n, _CHUNK):
        c1 = min(n, c0 + _CHUNK)
        u = uniform(key, 4 * (c1 - c0), 4 * c0, device).view(-1, 4)
        z = torch.sqrt(-2.0 * torch.log(u[:, 0])) * torch.cos(2.0 * math.pi * u[:, 1])
        v = -2.0 * torch.log(u[:, 2] * u[:, 3])
        out[c0:c1] = z / torch.sqrt(v / 4.0)
    return out


def distinct_indices(key: int, n_total: int, k: int) -> torch.Tensor:
    """``k`` distinct sorted indices in ``[0, n_total)`` (ranks of seeded uniforms)."""
    if k <= 0:
        return torch.empty(0, dtype=torch.int64)
    u = uniform(key, n_total)
    return torch.sort(torch.argsort(u)[:k]).values


# --------------------------------------------------------------------------- #
# Workloads
# --------------------------------------------------------------------------- #

@dataclass(frozen=True)
class Linear:
    name: str
    rows: int      # out-features
    cols: int      # in-features (the group / reduction dimension)


@dataclass(frozen=True)
class Workload:
    name: str
    index: int                 # 1-based position in the list below
    linears: tuple             # Linear shapes of one decoder
    decoders: int
    dtype: str                 # "bf16" | "f32"
    dist: str                  # "normal" | "t4"
    scale: float
    outlier_frac: float        # fraction of input columns scaled (rounded to nearest)
    outlier_count: int         # fixed count instead of a fraction (0: use the fraction)
    outlier_factor: float
    zero_rows: int
    fmt: str                   # format preset name
    group: int
    T: int
    act: dict = field(default_factory=dict)   # tokens, K, frac, factor, fmt, group

    @property
    def matrices(self):
        return [(d, i, l) for d in range(self.decoders) for i, l in enumerate(self.linears)]

    @property
    def elements(self) -> int:
        return self.decoders * sum(l.rows * l.cols for l in self.linears)


def _llama(h, kv, ff):
    return (Linear("q_proj", h, h), Linear("k_proj", kv, h), Linear("v_proj", kv, h),
            Linear("o_proj", h, h), Linear("gate_proj", ff, h), Linear("up_proj", ff, h),
            Linear("down_proj", h, ff))


WORKLOADS = {
    "toy256x512_int4_g32": Workload(
        "toy256x512_int4_g32", 1, (Linear("w", 256, 512),), 1, "f32", "normal", 0.02,
        0.0, 4, 20.0, 1, "int4_bf16", 32, 15),
    "smollm2_135m_mxint4_g32": Workload(
        "smollm2_135m_mxint4_g32", 2, _llama(576, 192, 1536), 30, "bf16", "t4", 0.02,
        0.01, 0, 10.0, 0, "mxint4", 32, 5),
    "llama31_8b_int4_g64": Workload(
        "llama31_8b_int4_g64", 3, _llama(4096, 1024, 14336), 32, "bf16", "t4", 0.02,
        0.01, 0, 10.0, 0, "int4_bf16", 64, 15,
        dict(tokens=16 * 2048, K=4096, frac=0.005, factor=30.0, fmt="int4_bf16", group=64)),
    "llama31_8b_nvfp4_g16": Workload(
        "llama31_8b_nvfp4_g16", 4, _llama(4096, 1024, 14336), 32, "bf16", "t4", 0.02,
        0.01, 0, 10.0, 0, "nvfp4", 16, 15,
        dict(tokens=16 * 2048, K=4096, frac=0.005, factor=30.0, fmt="nvfp4", group=16)),
    "llama31_70b_decoder_mxfp4_g32": Workload(
        "llama31_70b_decoder_mxfp4_g32", 5, _llama(8192, 1024, 28672), 1, "bf16", "t4", 0.015,
        0.01, 0, 10.0, 0, "mxfp4", 32, 15,
        dict(tokens=8 * 4096, K=8192, frac=0.005, factor=30.0, fmt="mxfp4", group=32)),
}


# The same 70B decoder weights and activations in the other formats of the
# MX family (the pages claim the whole family; element formats from the OCP
# Microscaling definition).
for _f in ("mxint8", "mxfp8_e4m3", "mxfp8_e5m2", "mxfp6_e2m3", "mxfp6_e3m2"):
    _base = WORKLOADS["llama31_70b_decoder_mxfp4_g32"]
    WORKLOADS[f"llama31_70b_decoder_{_f}_g32"] = replace(
        _base, name=f"llama31_70b_decoder_{_f}_g32", fmt=_f, act=dict(_base.act, fmt=_f))


# The same weights with BF16 outer scales (the scale-set variant: E8M0
# group scales, BF16 a and b); the activations stay MXFP4.
WORKLOADS["llama31_70b_decoder_mxfp4_bf16outer_g32"] = replace(
    WORKLOADS["llama31_70b_decoder_mxfp4_g32"], name="llama31_70b_decoder_mxfp4_bf16outer_g32",
    fmt="mxfp4_bf16outer")


def outlier_count(n: int, frac: float) -> int:
    return int(math.floor(n * frac + 0.5))


def weight(wl: Workload, decoder: int, index: int, device="cpu",
           rows: int | None = None, cols: int | None = None) -> torch.Tensor:
    """Seeded weight matrix ``[rows, cols]`` of the workload's distribution.

    ``rows``/``cols`` override the shape (for reduced-size cases of the same
    distribution); the outlier-column count follows the overriding width.
    """
    lin = wl.linears[index]
    r = lin.rows if rows is None else rows
    c = lin.cols if cols is None else cols
    base = (wl.index, decoder, index)
    n = r * c
    draw = student_t4 if wl.dist == "t4" else normal
    w = draw(stream_key(*base, 1), n, device=device).view(r, c) * wl.scale
    k = wl.outlier_count if wl.outlier_count else outlier_count(c, wl.outlier_frac)
    cols_idx = distinct_indices(stream_key(*base, 2), c, k).to(device)
    if k:
        w[:, cols_idx] *= wl.outlier_factor
    if wl.zero_rows:
        zr = distinct_indices(stream_key(*base, 3), r, wl.zero_rows).to(device)
        w[zr, :] = 0.0
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    return w.to(dt)


def activation(wl: Workload, device="cpu", tokens: int | None = None) -> torch.Tensor:
    """Seeded activation ``[tokens, K]`` bf16: N(0,1) with outlier channels."""
    a = wl.act
    t = a["tokens"] if tokens is None else tokens
    K = a["K"]
    x = torch.empty(t, K, dtype=torch.float64, device=device)
    rows_per = max(1, _CHUNK // K)
    key = stream_key(wl.index, 1000, 0, 1)
    for r0 in range(0, t, rows_per):
        r1 = min(t, r0 + rows_per)
        # row r of the activation always uses draws [r*K, (r+1)*K): a reduced
        # token count is a prefix of the full one.
        u = uniform(key, 2 * (r1 - r0) * K, 2 * r0 * K, device).view(-1, 2)
        x[r0:r1] = (torch.sqrt(-2.0 * torch.log(u[:, 0])) * torch.cos(2.0 * math.pi * u[:, 1])).view(r1 - r0, K)
    k = outlier_count(K, a["frac"])
    ch = distinct_indices(stream_key(wl.index, 1000, 0, 2), K, k).to(device)
    x[:, ch] *= a["factor"]
    return x.to(torch.bfloat16)


def scaled_columns(wl: Workload, decoder: int, index: int, cols: int | None = None) -> torch.Tensor:
    """Indices of the seeded outlier columns of one linear (for tests)."""
    c = wl.linears[index].cols if cols is None else cols
    k = wl.outlier_count if wl.outlier_count else outlier_count(c, wl.outlier_frac)
    return distinct_indices(stream_key(wl.index, decoder, index, 2), c, k)
