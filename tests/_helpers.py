"""Shared helpers of the GPU parity tests (oracle side and conversions)."""
import numpy as np
import torch

import oracle as O

PRESET_COMBOS = {
    # name -> (oracle Format factory); the library's presets carry the same sets
    "int4_bf16": lambda G: O.preset("int4_bf16", G),
    "mxint4": lambda G: O.preset("mxint4", G),
    "mxfp4": lambda G: O.preset("mxfp4", G),
    "nvfp4": lambda G: O.preset("nvfp4", G),
    # BF16 outer scales with E8M0 group scales (descriptor variant)
    "mxint4_bf16outer": lambda G: O.Format("int4", G, "e8m0", "bf16"),
    "mxfp4_bf16outer": lambda G: O.Format("e2m1", G, "e8m0", "bf16"),
    # NVFP4 without the second-level tensor scale (the literal reading: E4M3
    # group scales of small weights fall into E4M3's subnormal range)
    "nvfp4_ts1": lambda G: O.Format("e2m1", G, "e4m3", "bf16", tensor_scale_auto=False),
    # the rest of the MX family
    "mxint8": lambda G: O.preset("mxint8", G),
    "mxfp8_e4m3": lambda G: O.preset("mxfp8_e4m3", G),
    "mxfp8_e5m2": lambda G: O.preset("mxfp8_e5m2", G),
    "mxfp6_e2m3": lambda G: O.preset("mxfp6_e2m3", G),
    "mxfp6_e3m2": lambda G: O.preset("mxfp6_e3m2", G),
}
MX_MORE = ["mxint8", "mxfp8_e4m3", "mxfp8_e5m2", "mxfp6_e2m3", "mxfp6_e3m2"]


def code_boundaries(fo):
    """Decision boundaries of the code grid (code magnitudes' midpoints)."""
    if fo.codes == "int4":
        return np.arange(0, 7) + 0.5
    if fo.codes == "int8":
        return np.arange(0, 127) + 0.5
    if fo.codes == "e2m1":
        grid = O.E2M1_GRID
    else:
        v = O.fp_element_values(fo.codes)
        grid = v[~np.isnan(v)]
    return (grid[:-1] + grid[1:]) / 2


def lib_format(name, G):
    import dual_scale_solver_b200 as dq
    if name.endswith("_bf16outer"):
        f = dq.format_preset(name.split("_")[0], G)
        f.outer_scale = 0
        return f
    if name == "nvfp4_ts1":
        f = dq.format_preset("nvfp4", G)
        f.tensor_scale_auto = 0
        return f
    return dq.format_preset(name, G)


def np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def gpu_scales_np(gs: torch.Tensor) -> np.ndarray:
    g = gs.detach().cpu().numpy()
    return g.view(np.uint16) if g.dtype == np.int16 else g


def oracle_encoded(W64, a, b, fmt, ts=1.0):
    """Packed codes and encoded group scales of Q(W / (a b^T)) by the oracle."""
    c, s = O.quantize(O.inner(W64, a, b), fmt, ts)
    return O.encode_codes(c, fmt), O.encode_scales(s, fmt)


def random_outer(fmt, n, key, spread=0.7):
    """Seeded outer scales in the format's set (inputs of a parity case)."""
    import synth
    u = synth.uniform(key, n).numpy()
    return O.project_outer(np.exp((2 * u - 1) * spread), fmt)


def near_outer_boundary(x, fmt, rel=1e-5):
    """True where x is within `rel` of a decision boundary of the outer projection."""
    x = np.asarray(x, dtype=np.float64)
    if fmt.oscale == "e8m0":
        m, e = np.frexp(x)                       # x = m 2^e, boundary at m = 0.75
        return np.abs(m - 0.75) <= 0.75 * rel
    lo = O.project_outer(x * (1 - rel), fmt)
    hi = O.project_outer(x * (1 + rel), fmt)
    return lo != hi


def check_projected(gpu, orc, pre, fmt, what, max_frac=1e-3):
    """Projected outer scales of the GPU against the oracle's.

    E8M0 outer scales must agree exactly.  BF16 outer scales must agree
    except where the oracle's unprojected ratio lies within 1e-5 relative of
    a bf16 rounding boundary: there the GPU's float32 statistics (within
    1e-5 of the fp64 ones) may round to the other neighbour.  At most
    `max_frac` of the scales (at least one) may flip; the count is printed
    and returned."""
    gpu, orc = np.asarray(gpu), np.asarray(orc)
    diff = gpu != orc
    if fmt.oscale == "e8m0":
        bad = np.argwhere(diff).ravel()
        assert bad.size == 0, f"{what}: {bad.size} E8M0 scales differ, first {bad[:5].tolist()}"
        return 0
    near = near_outer_boundary(pre, fmt)
    unexplained = np.argwhere(diff & ~near).ravel()
    assert unexplained.size == 0, f"{what}: {unexplained.size} differ away from a boundary"
    n = int(diff.sum())
    assert n <= max(1, max_frac * diff.size), f"{what}: {n} near-boundary flips"
    if n:
        print(f"{what}: {n} of {diff.size} BF16 scales flipped at a rounding boundary")
    return n
