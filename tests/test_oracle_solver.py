"""Pins of the oracle's quantizer, closed-form updates and loop (no GPU).

Each check rests on something other than the oracle itself: an exact
rational re-derivation in pure Python, a brute-force scan over every
admissible scale, a mathematical property of the method (least squares with
fixed codes, power-of-two invariance) or a hand-derived case.
"""
from fractions import Fraction as Fr

import numpy as np
import pytest
import torch

import oracle as O
import synth

FORMATS = ["int4_bf16", "mxint4", "mxfp4", "nvfp4"]
# the rest of the MX family
MX_MORE = ["mxfp8_e4m3", "mxfp8_e5m2", "mxfp6_e2m3", "mxfp6_e3m2", "mxint8"]
ALL_FORMATS = FORMATS + MX_MORE
# element float formats: (significant bits, lowest normal exponent, largest value)
FP_ELEM = {"e4m3": (4, -6, Fr(448)), "e5m2": (3, -14, Fr(57344)),
           "e2m3": (4, 0, Fr(15, 2)), "e3m2": (3, -2, Fr(28))}
E2M1 = [Fr(0), Fr(1, 2), Fr(1), Fr(3, 2), Fr(2), Fr(3), Fr(4), Fr(6)]


# --------------------------------------------------------------------------- #
# An exact rational restatement of Q, pure Python, for small matrices
# --------------------------------------------------------------------------- #

def _floor_log2(x: Fr) -> int:
    e = 0
    while Fr(2) ** e > x:
        e -= 1
    while Fr(2) ** (e + 1) <= x:
        e += 1
    return e


def _rne(x: Fr, p: int, emin: int, maxval: Fr) -> Fr:
    e = max(_floor_log2(x), emin)
    quantum = Fr(2) ** (e - (p - 1))
    v = round(x / quantum) * quantum           # round() on Fraction: half to even
    return min(v, maxval)


def py_group_scale(g: Fr, gscale: str) -> Fr:
    if gscale == "bf16":
        v = _rne(g, 8, -126, Fr(2) ** 127 * (2 - Fr(1, 128)))
        return max(v, Fr(2) ** -126)
    if gscale == "e8m0":
        e = -126
        while Fr(2) ** e < g and e < 126:
            e += 1
        return Fr(2) ** e
    v = _rne(g, 4, -6, Fr(448))
    return v if v > 0 else Fr(2) ** -9


def py_code(q: Fr, codes: str) -> Fr:
    if codes == "int4":
        return Fr(min(7, max(-8, round(q))))
    if codes == "int8":
        return Fr(min(127, max(-128, round(q))))
    if codes in FP_ELEM:
        p, emin, mx = FP_ELEM[codes]
        v = Fr(0) if q == 0 else _rne(abs(q), p, emin, mx)
        return v if q >= 0 else -v
    aq = min(abs(q), Fr(6))
    d = [abs(aq - g) for g in E2M1]
    best = min(d)
    idx = [i for i in range(8) if d[i] == best]
    i = idx[0] if len(idx) == 1 else [i for i in idx if i % 2 == 0][0]
    return E2M1[i] if q >= 0 else -E2M1[i]


def py_quantize(Y, fmt, ts=Fr(1)):
    rows, cols = len(Y), len(Y[0])
    G = fmt.group
    C = [[None] * cols for _ in range(rows)]
    S = [[None] * (cols // G) for _ in range(rows)]
    for i in range(rows):
        for g in range(cols // G):
            grp = Y[i][g * G:(g + 1) * G]
            m = max(abs(v) for v in grp)
            s = Fr(1) if m == 0 else py_group_scale(m / (Fr(fmt.qmax) * ts), fmt.gscale)
            S[i][g] = s
            for k, v in enumerate(grp):
                C[i][g * G + k] = py_code(v / (s * ts), fmt.codes)
    return C, S


def _small_matrix(rows, cols, seed, outliers=True):
    rng = np.random.default_rng(seed)
    W = rng.standard_t(4, (rows, cols)) * 0.02
    if outliers:
        W[:, rng.choice(cols, 3, replace=False)] *= 10
    return torch.from_numpy(W).to(torch.bfloat16).double().numpy()


@pytest.mark.parametrize("name", ALL_FORMATS)
@pytest.mark.parametrize("G", [16, 32, 64])
def test_quantize_matches_exact_rational_restatement(name, G):
    fmt = O.preset(name, G)
    W = _small_matrix(3, 2 * G, seed=G)
    rng = np.random.default_rng(3)
    a = O.project_outer(np.exp(rng.uniform(-1, 1, 3)), fmt)
    b = O.project_outer(np.exp(rng.uniform(-1, 1, 2 * G)), fmt)
    ts = 2.0 ** -9 if fmt.tensor_scale_auto else 1.0
    c, s = O.quantize(O.inner(W, a, b), fmt, ts)
    Y = [[Fr(float(W[i, j])) / (Fr(float(a[i])) * Fr(float(b[j]))) for j in range(2 * G)]
         for i in range(3)]
    C, S = py_quantize(Y, fmt, Fr(ts))
    assert np.array_equal(c, np.array([[float(v) for v in r] for r in C]))
    assert np.array_equal(s, np.array([[float(v) for v in r] for r in S]))


def test_quantize_hand_cases():
    # INT4 with BF16 scale, G16: max 7/8 -> s = (7/8)/7 = 1/8 exactly; codes are
    # Y*8 rounded half to even: 3.5->4, -3.5->-4, 2.5->2, 0.5->0, 1.5->2.
    fmt = O.preset("int4_bf16", 16)
    y = np.array([7, 3.5, -3.5, 2.5, 0.5, -0.5, 1.5, 0, 1, 2, 3, 4, 5, 6, -7, 6.5]) / 8.0
    c, s = O.quantize(y[None, :], fmt)
    assert s[0, 0] == 0.125
    assert list(c[0]) == [7, 4, -4, 2, 0, 0, 2, 0, 1, 2, 3, 4, 5, 6, -7, 6]
    # MXFP4, G32: max 1.5 -> 1.5/6 = 0.25 is a power of two -> s = 0.25; codes
    # on the E2M1 grid: 0.25->0, 0.75->1, 1.25->1, 1.75->2, 2.5->2, 3.5->4, 5->4.
    fmt = O.preset("mxfp4", 32)
    q = np.array([6, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5] + [0] * 24, dtype=float)
    c, s = O.quantize((q * 0.25)[None, :], fmt)
    assert s[0, 0] == 0.25
    assert list(c[0, :8]) == [6, 0, 1, 1, 2, 2, 4, 4]
    # MXINT4: max 7.5/16 -> 7.5/16/7 is just above 1/16 -> rounds up to 1/8;
    # then 7.5/16 / (1/8) = 3.75 -> 4.
    fmt = O.preset("mxint4", 32)
    c, s = O.quantize(np.array([[7.5 / 16] + [0.0] * 31]), fmt)
    assert s[0, 0] == 0.125 and c[0, 0] == 4
    # NVFP4 (ts=1): max 1.8 -> 1.8/6 = 0.3 -> E4M3 nearest 0.3125 (1.010b x 2^-2).
    fmt = O.preset("nvfp4", 16)
    c, s = O.quantize(np.array([[1.8] + [0.0] * 15]), fmt)
    assert s[0, 0] == 0.3125 and c[0, 0] == 6     # 5.76 -> 6
    # all-zero group: scale 1, codes 0
    c, s = O.quantize(np.zeros((1, 16)), fmt)
    assert s[0, 0] == 1.0 and np.all(c == 0)
    # E4M3 saturation: max/6 above 448 -> s = 448, codes saturate at 6
    c, s = O.quantize(np.array([[6000.0, -3000.0] + [0.0] * 14]), fmt)
    assert s[0, 0] == 448.0 and c[0, 0] == 6 and c[0, 1] == -6


@pytest.mark.parametrize("name", ALL_FORMATS)
def test_quantizer_idempotent(name):
    fmt = O.preset(name)
    W = _small_matrix(16, 4 * fmt.group, seed=5)
    # adversarial groups: maxima exactly on scale boundaries
    W[0, :fmt.group] = np.linspace(-1, 1, fmt.group) * fmt.qmax * 2.0 ** -4
    W[1, :fmt.group] *= 0.0
    W[1, 0] = 1.5 * 2.0 ** -5
    ts = O.tensor_scale(W, fmt)
    c, s = O.quantize(W, fmt, ts)
    Qh = O.dequantize(c, s, fmt, ts)
    c2, s2 = O.quantize(Qh, fmt, ts)
    assert np.array_equal(O.dequantize(c2, s2, fmt, ts), Qh)


def test_tensor_scale():
    fmt = O.preset("nvfp4")
    W = np.zeros((1, 16))
    W[0, 3] = 448 * 6 * 2.0 ** -3
    assert O.tensor_scale(W, fmt) == 2.0 ** -3
    W[0, 3] = np.nextafter(W[0, 3], np.inf)
    assert O.tensor_scale(W, fmt) == 2.0 ** -2
    assert O.tensor_scale(np.zeros((2, 16)), fmt) == 1.0
    assert O.tensor_scale(W, O.preset("mxfp4")) == 1.0


# --------------------------------------------------------------------------- #
# Closed-form updates: brute force over every admissible scale
# --------------------------------------------------------------------------- #

def _admissible(fmt, x):
    if fmt.oscale == "e8m0":
        return 2.0 ** np.arange(-126, 127)
    # every bf16 value within a factor 4 of x
    u = np.arange(1 << 15, dtype=np.uint32)
    v = (u << 16).view(np.float32)
    v = v[np.isfinite(v)].astype(np.float64)
    v = v[v >= 2.0 ** -126]
    return v[(v > x / 4) & (v < x * 4)]


@pytest.mark.parametrize("name", ALL_FORMATS)
def test_row_and_column_updates_minimise_over_the_scale_set(name):
    fmt = O.preset(name)
    W = _small_matrix(6, 2 * fmt.group, seed=17)
    rng = np.random.default_rng(2)
    a0 = O.project_outer(np.exp(rng.uniform(-0.5, 0.5, 6)), fmt)
    b0 = O.project_outer(np.exp(rng.uniform(-0.5, 0.5, 2 * fmt.group)), fmt)
    ts = O.tensor_scale(W, fmt)
    Qh, _, _ = O.qhat(W, a0, b0, fmt, ts)
    a, xa = O.row_update(W, Qh, b0, fmt)
    R = Qh * b0[None, :]
    for i in range(6):
        cand = _admissible(fmt, xa[i])
        obj = ((W[i][None, :] - cand[:, None] * R[i][None, :]) ** 2).sum(1)
        mine = ((W[i] - a[i] * R[i]) ** 2).sum()
        assert mine <= obj.min() * (1 + 1e-12), (i, a[i], cand[obj.argmin()])
    b, xb = O.col_update(W, Qh, a0, fmt)
    S = a0[:, None] * Qh
    for j in range(2 * fmt.group):
        cand = _admissible(fmt, xb[j])
        obj = ((W[:, j][None, :] - cand[:, None] * S[:, j][None, :]) ** 2).sum(1)
        mine = ((W[:, j] - b[j] * S[:, j]) ** 2).sum()
        assert mine <= obj.min() * (1 + 1e-12), (j, b[j], cand[obj.argmin()])


def test_closed_form_ratio_direction():
    # With Qhat fixed and one row, the unprojected a* is <W,R>/<R,R>
    # (least squares of W ~ a R); a 2-element case worked by hand:
    # W = [2, 1], R = [1, 1] -> a* = 3/2.
    fmt = O.preset("int4_bf16", 16)
    W = np.zeros((1, 16))
    W[0, :2] = [2.0, 1.0]
    Qh = np.zeros((1, 16))
    Qh[0, :2] = [1.0, 1.0]
    a, x = O.row_update(W, Qh, np.ones(16), fmt)
    assert x[0] == 1.5 and a[0] == 1.5
    b, xb = O.col_update(W, Qh, np.array([2.0]), fmt)
    assert xb[0] == 1.0 and xb[1] == 0.5       # (2*2)/(2*2), (1*2)/(2*2)


def test_zero_slices_keep_scale_one():
    fmt = O.preset("int4_bf16", 32)
    W = _small_matrix(4, 64, seed=3)
    W[:, 5] = 1e-6                                 # tiny column: codes all zero
    W[2, :] = 0.0                                  # all-zero row
    Qh, c, _ = O.qhat(W, np.full(4, 0.5), np.full(64, 2.0), fmt)
    assert np.all(c[:, 5] == 0) and np.all(c[2] == 0)
    a, xa = O.row_update(W, Qh, np.full(64, 2.0), fmt)
    b, xb = O.col_update(W, Qh, np.full(4, 0.5), fmt)
    assert a[2] == 1.0 and np.isnan(xa[2])
    assert b[5] == 1.0 and np.isnan(xb[5])


@pytest.mark.parametrize("name", ALL_FORMATS)
def test_outputs_are_representable(name):
    fmt = O.preset(name)
    W = _small_matrix(32, 4 * fmt.group, seed=23)
    r = O.solve(W, fmt, 3)
    O.encode_scales(r["scales"], fmt)                              # raises if not
    O.encode_codes(r["codes"], fmt)
    if fmt.oscale == "e8m0":
        from oracle import formats as F
        F.encode_e8m0(r["a"]), F.encode_e8m0(r["b"])
    else:
        assert np.array_equal(O.project_outer(r["a"], fmt), r["a"])
        assert np.array_equal(O.project_outer(r["b"], fmt), r["b"])


# --------------------------------------------------------------------------- #
# The loop
# --------------------------------------------------------------------------- #

def test_initial_state_is_single_scale_rtn():
    fmt = O.preset("int4_bf16", 16)
    W = _small_matrix(4, 48, seed=31)
    r = O.solve(W, fmt, 0)
    C, S = py_quantize([[Fr(float(v)) for v in row] for row in W], fmt)
    err = sum((Fr(float(W[i, j])) - C[i][j] * S[i][j // 16]) ** 2
              for i in range(4) for j in range(48)) / (4 * 48)
    assert r["mse_trace"][0] == pytest.approx(float(err), rel=1e-13)


@pytest.mark.parametrize("name", ALL_FORMATS)
def test_fixed_code_half_steps_never_increase_the_error(name):
    # with the codes held fixed, each closed-form + nearest-projection step is
    # the exact minimiser over the scale set, so it cannot raise the MSE
    fmt = O.preset(name)
    W = _small_matrix(24, 4 * fmt.group, seed=41)
    ts = O.tensor_scale(W, fmt)
    a, b = np.ones(24), np.ones(4 * fmt.group)
    for _ in range(4):
        Qh, _, _ = O.qhat(W, a, b, fmt, ts)
        before = O.mse(W, Qh, a, b)
        a2, _ = O.row_update(W, Qh, b, fmt)
        assert O.mse(W, Qh, a2, b) <= before * (1 + 1e-13)
        a = a2
        Qh, _, _ = O.qhat(W, a, b, fmt, ts)
        before = O.mse(W, Qh, a, b)
        b2, _ = O.col_update(W, Qh, a, fmt)
        assert O.mse(W, Qh, a, b2) <= before * (1 + 1e-13)
        b = b2


@pytest.mark.parametrize("name", ["mxint4", "mxfp4"] + MX_MORE)
def test_power_of_two_row_step_leaves_mx_reconstruction_unchanged(name):
    # E8M0 row scale with E8M0 group scales: a power of two only shifts every
    # group exponent, so D_a Qhat is unchanged and the row half-step MSE equals
    # the previous full-step MSE exactly.
    fmt = O.preset(name)
    W = _small_matrix(16, 4 * fmt.group, seed=43)
    r = O.solve(W, fmt, 4)
    assert np.array_equal(r["mse_half"], r["mse_trace"][:-1])


@pytest.mark.parametrize("name", ALL_FORMATS)
def test_solve_is_equivariant_under_row_and_group_permutations(name):
    # Each row's update reads only that row (given b), each group's scale only
    # that group (given a and b), each column's update only that column (given
    # a): permuting the rows, the column groups and the columns inside each
    # group of W permutes a, b, the codes and the group scales the same way
    # and leaves the error unchanged.  An index slip or a transposed operand
    # (a read by column, b by row) breaks this.
    fmt = O.preset(name)
    G, rows, ng = fmt.group, 20, 5
    W = _small_matrix(rows, ng * G, seed=53)
    rng = np.random.default_rng(7)
    pr, pg = rng.permutation(rows), rng.permutation(ng)
    pc = np.concatenate([g * G + rng.permutation(G) for g in pg])
    r = O.solve(W, fmt, 4)
    p = O.solve(W[pr][:, pc], fmt, 4)
    assert np.array_equal(p["a"], r["a"][pr])
    assert np.array_equal(p["b"], r["b"][pc])
    assert np.array_equal(p["codes"], r["codes"][pr][:, pc])
    assert np.array_equal(p["scales"], r["scales"][pr][:, pg])
    assert p["ts"] == r["ts"]
    assert np.allclose(p["mse_trace"], r["mse_trace"], rtol=1e-12, atol=0)


@pytest.mark.parametrize("name", ALL_FORMATS)
@pytest.mark.parametrize("k", [3, -5])
def test_solve_scales_with_powers_of_two(name, k):
    # W -> 2^k W moves every group maximum (and the NVFP4 tensor scale) by
    # 2^k; every scale set is closed under that shift in this range and the
    # projections commute with it, so the codes, a and b stay the same, the
    # group scales (or, with a tensor scale, that scale) move by 2^k, and the
    # error moves by exactly 4^k.
    fmt = O.preset(name)
    W = _small_matrix(16, 4 * fmt.group, seed=59)
    r = O.solve(W, fmt, 4)
    p = O.solve(W * 2.0 ** k, fmt, 4)
    assert np.array_equal(p["a"], r["a"])
    assert np.array_equal(p["b"], r["b"])
    assert np.array_equal(p["codes"], r["codes"])
    if fmt.tensor_scale_auto:
        assert p["ts"] == r["ts"] * 2.0 ** k
        assert np.array_equal(p["scales"], r["scales"])
    else:
        assert np.array_equal(p["scales"], r["scales"] * 2.0 ** k)
    assert np.array_equal(p["mse_trace"], r["mse_trace"] * 4.0 ** k)


# --------------------------------------------------------------------------- #
# The order of the steps, against an exact restatement of whole iterations
# --------------------------------------------------------------------------- #

def _py_project_outer(x: Fr, oscale: str) -> Fr:
    """Nearest admissible outer scale, exactly (BF16: nearest even in the
    normal range; E8M0: midpoint 1.5 * 2^k, a tie goes up, |k| <= 126)."""
    if oscale == "bf16":
        return max(_rne(x, 8, -126, Fr(2) ** 127 * (2 - Fr(1, 128))), Fr(2) ** -126)
    k = max(min(_floor_log2(x), 126), -127)
    if x >= Fr(3, 2) * Fr(2) ** k:
        k += 1
    return Fr(2) ** max(min(k, 126), -126)


def py_solve(W, fmt, T):
    """T iterations of the dual-scale solve in exact rational arithmetic,
    written from the text under eq. (2) of the daiwk note: update the row
    scales from R = Qhat D_b with the codes fixed, re-quantize, update the
    column scales from S = D_a Qhat with the codes fixed, re-quantize; a
    slice with no non-zero code keeps scale 1.  Q is py_quantize; the NVFP4
    tensor scale is 2^ceil(log2(amax / (448 qmax)))."""
    rows, cols = len(W), len(W[0])
    ts = Fr(1)
    if fmt.tensor_scale_auto:
        amax = max(abs(v) for r in W for v in r)
        if amax > 0:
            ts = py_group_scale(amax / (448 * Fr(fmt.qmax)), "e8m0")
    a, b = [Fr(1)] * rows, [Fr(1)] * cols
    G = fmt.group

    def qhat():
        C, S = py_quantize([[W[i][j] / (a[i] * b[j]) for j in range(cols)] for i in range(rows)],
                           fmt, ts)
        return [[C[i][j] * S[i][j // G] * ts for j in range(cols)] for i in range(rows)]

    def err(Qh):
        return sum((W[i][j] - a[i] * Qh[i][j] * b[j]) ** 2
                   for i in range(rows) for j in range(cols)) / (rows * cols)

    Qh = qhat()
    trace, half = [err(Qh)], []
    for _ in range(T):
        for i in range(rows):
            R = [Qh[i][j] * b[j] for j in range(cols)]
            den = sum(v * v for v in R)
            a[i] = _py_project_outer(sum(W[i][j] * R[j] for j in range(cols)) / den,
                                     fmt.oscale) if den > 0 else Fr(1)
        Qh = qhat()
        half.append(err(Qh))
        for j in range(cols):
            S = [a[i] * Qh[i][j] for i in range(rows)]
            den = sum(v * v for v in S)
            b[j] = _py_project_outer(sum(W[i][j] * S[i] for i in range(rows)) / den,
                                     fmt.oscale) if den > 0 else Fr(1)
        Qh = qhat()
        trace.append(err(Qh))
    return a, b, trace, half


def _order_matrix(seed):
    # 3 x 32: one outlier column, one all-zero row (second row)
    rng = np.random.default_rng(seed)
    W = rng.standard_t(4, (3, 32)) * 0.02
    W[:, rng.choice(32, 1, replace=False)] *= 10
    W[1, :] = 0.0
    return torch.from_numpy(W).to(torch.bfloat16).double().numpy()


# (format, G, seed): inputs on which the first two iterations move scales --
# with BF16 outer scales both a and b; with E8M0 outer scales b (a power-of-two
# row scale only shifts the group exponents, so a stays)
ORDER_CASES = [("int4_bf16", 16, 4), ("nvfp4", 16, 0), ("mxint4", 16, 1)]


@pytest.mark.parametrize("name,G,seed", ORDER_CASES)
def test_solve_follows_the_step_order_exactly(name, G, seed):
    # The oracle's loop (row update, re-quantize, column update, re-quantize;
    # mse_half right after the row half-step) against the exact restatement
    # over two iterations.  Running the column step first, skipping the
    # re-quantization between the steps, or recording mse_half after the
    # column step each changes a, b or the traces here.
    fmt = O.preset(name, G)
    W = _order_matrix(seed)
    r = O.solve(W, fmt, 2)
    a, b, trace, half = py_solve([[Fr(float(v)) for v in row] for row in W], fmt, 2)
    assert list(r["a"]) == [float(v) for v in a]
    assert list(r["b"]) == [float(v) for v in b]
    assert np.allclose(r["mse_trace"], [float(v) for v in trace], rtol=1e-12, atol=0)
    assert np.allclose(r["mse_half"], [float(v) for v in half], rtol=1e-12, atol=0)
    # the case is not at a fixed point: scales move in the first iteration
    r1 = O.solve(W, fmt, 1)
    assert np.any(r1["b"] != 1.0)
    if fmt.oscale == "bf16":
        assert np.any(r1["a"] != 1.0) and np.any(r["a"] != r1["a"])
        assert half[0] != trace[0] and half[0] != trace[1]


@pytest.mark.parametrize("name", FORMATS)
def test_dual_scale_beats_single_scale_on_outlier_matrices(name):
    fmt = O.preset(name)
    W = _small_matrix(64, 8 * fmt.group, seed=47)
    r = O.solve(W, fmt, 5)
    assert r["mse_trace"][-1] < r["mse_trace"][0]


def test_toy_workload_trace():
    wl = synth.WORKLOADS["toy256x512_int4_g32"]
    W = synth.weight(wl, 0, 0).double().numpy()
    assert (W == 0).all(axis=1).sum() == 1
    r = O.solve(W, O.preset(wl.fmt, wl.group), wl.T)
    zr = np.where((W == 0).all(axis=1))[0][0]
    assert r["a"][zr] == 1.0
    assert r["mse_trace"][-1] < 0.5 * r["mse_trace"][0]


# --------------------------------------------------------------------------- #
# Activation rescale + quantize
# --------------------------------------------------------------------------- #

@pytest.mark.parametrize("name", ALL_FORMATS)
def test_activation_path(name):
    fmt = O.preset(name)
    rng = np.random.default_rng(5)
    X = torch.from_numpy(rng.standard_normal((8, 4 * fmt.group))).to(torch.bfloat16).double().numpy()
    c1, s1 = O.act_rescale_quant(X, np.ones(X.shape[1]), fmt)
    c0, s0 = O.quantize(X, fmt, 1.0)
    assert np.array_equal(c1, c0) and np.array_equal(s1, s0)
    # b multiplies the channel: b = 2 on all channels is Q(2X)
    c2, s2 = O.act_rescale_quant(X, np.full(X.shape[1], 2.0), fmt)
    c3, s3 = O.quantize(2 * X, fmt, 1.0)
    assert np.array_equal(c2, c3) and np.array_equal(s2, s3)


def test_activation_identity():
    # eq. (1): X W^T ~ (X D_b) Qhat^T D_a with What = D_a Qhat D_b
    fmt = O.preset("int4_bf16", 16)
    W = _small_matrix(5, 32, seed=8)
    r = O.solve(W, fmt, 2)
    What = r["a"][:, None] * r["qhat"] * r["b"][None, :]
    X = np.random.default_rng(1).standard_normal((3, 32))
    lhs = (X * r["b"][None, :]) @ r["qhat"].T * r["a"][None, :]
    assert np.allclose(lhs, X @ What.T, rtol=1e-12, atol=1e-14)


# --------------------------------------------------------------------------- #
# The seeded generator
# --------------------------------------------------------------------------- #

def test_generator_matches_integer_splitmix64():
    M = (1 << 64) - 1

    def sm(z):
        z = (z + synth.GOLDEN) & M
        z = ((z ^ (z >> 30)) * synth.MIX1) & M
        z = ((z ^ (z >> 27)) * synth.MIX2) & M
        return z ^ (z >> 31)

    key = synth.stream_key(3, 1, 4)
    bits = synth.raw_bits(key, 50, offset=1000)
    for i in range(50):
        want = sm((key + (1000 + i) * synth.GOLDEN) & M)
        assert (int(bits[i]) & M) == want
    u = synth.uniform(key, 50, offset=1000)
    assert float(u[0]) == ((sm((key + 1000 * synth.GOLDEN) & M) >> 11) + 0.5) * 2.0 ** -53


@pytest.mark.parametrize("name,s,c_max,c_03", [
    # group max 1.0 and an element 0.3, G32, E8M0 scale = smallest 2^e >= 1/qmax
    ("mxfp8_e4m3", 2.0 ** -8, 256.0, 80.0),      # 0.3*256 = 76.8 -> grid step 8 -> 80
    ("mxfp8_e5m2", 2.0 ** -15, 32768.0, 10240.0),  # 9830.4 -> step 2048 -> 10240
    ("mxfp6_e2m3", 2.0 ** -2, 4.0, 1.25),        # 1.2 -> step 0.125 -> 1.25
    ("mxfp6_e3m2", 2.0 ** -4, 16.0, 5.0),        # 4.8 -> step 1 -> 5
    ("mxint8", 2.0 ** -6, 64.0, 19.0),           # 19.2 -> 19
])
def test_quantize_hand_cases_mx_family(name, s, c_max, c_03):
    fmt = O.preset(name)
    y = np.zeros((1, 32))
    y[0, 0], y[0, 1], y[0, 2] = 1.0, 0.3, -0.3
    c, sc = O.quantize(y, fmt)
    assert sc[0, 0] == s
    assert c[0, 0] == c_max and c[0, 1] == c_03 and c[0, 2] == -c_03


# --------------------------------------------------------------------------- #
# Two-level absmax quantization (msModelSlim DualScale page)
# --------------------------------------------------------------------------- #

def _rn32(x: Fr) -> Fr:
    """Exact rational rounding to the nearest float32, ties to even."""
    if x == 0:
        return Fr(0)
    v = _rne(abs(x), 24, -126, Fr(2) ** 127 * (2 - Fr(2) ** -23))
    return v if x > 0 else -v


def test_two_level_quant_matches_rational_restatement():
    fmt = O.preset("mxfp4")
    rng = np.random.default_rng(21)
    X = (rng.standard_normal((3, 1056)) * np.exp(rng.uniform(-3, 3, (3, 1)))).astype(np.float32)
    X[1, 512:1024] = 0.0                                   # an all-zero block
    X = X.astype(np.float64)
    c, s_in, S, qdq = O.two_level_quant(X, 512, fmt)
    assert S.shape == (3, 3)                               # ragged last block of 32 columns
    for i in range(3):
        Y = []
        Sr = []
        for k in range(3):
            blk = [Fr(float(v)) for v in X[i, k * 512:(k + 1) * 512]]
            m = max(abs(v) for v in blk)
            s = Fr(1) if m == 0 else _rn32(m / 6)
            Sr.append(s)
            Y += [_rn32(v / s) for v in blk]
        C, Sg = py_quantize([Y], fmt)
        assert [float(v) for v in Sr] == list(S[i])
        assert [float(v) for v in C[0]] == list(c[i])
        assert [float(v) for v in Sg[0]] == list(s_in[i])
        want = [float(_rn32(C[0][j] * Sg[0][j // 32] * Sr[j // 512])) for j in range(1056)]
        assert want == list(qdq[i])


def test_two_level_quant_special_cases():
    fmt = O.preset("mxfp4")
    rng = np.random.default_rng(22)
    X = rng.standard_normal((4, 1024)).astype(np.float32).astype(np.float64)
    # block maxima 6 * 2^k: the outer scales are powers of two, so the result
    # is plain MXFP4 of X
    for i in range(4):
        for k in range(2):
            blk = X[i, k * 512:(k + 1) * 512]
            blk *= 1.0 / np.abs(blk).max()
            blk[np.argmax(np.abs(blk))] = np.sign(blk[np.argmax(np.abs(blk))])
            blk *= 6.0 * 2.0 ** (i - k)
    c, s_in, S, qdq = O.two_level_quant(X, 512, fmt)
    assert np.array_equal(S, np.ldexp(1.0, np.array([[i - k for k in range(2)] for i in range(4)])))
    c0, s0 = O.quantize(X, fmt)
    assert np.array_equal(qdq, O.dequantize(c0, s0, fmt))
    # scaling X by a power of two scales S and keeps codes and inner scales
    c2, s2, S2, q2 = O.two_level_quant(X * 8.0, 512, fmt)
    assert np.array_equal(c2, c) and np.array_equal(s2, s_in) and np.array_equal(S2, 8 * S)
    assert np.array_equal(q2, 8 * qdq)
    # zero input: S = 1, codes 0, scales 1, reconstruction 0
    c3, s3, S3, q3 = O.two_level_quant(np.zeros((2, 512)), 512, fmt)
    assert np.all(S3 == 1) and np.all(c3 == 0) and np.all(s3 == 1) and np.all(q3 == 0)


def test_w4a4_gemm_against_explicit_sums():
    # out[m, n] = a_n sum_k (c_x s_x)(c_w s_w), written out with fractions
    fmt = O.preset("mxfp4")
    rng = np.random.default_rng(31)
    M, N, K = 3, 2, 64
    grid = np.concatenate([O.E2M1_GRID, -O.E2M1_GRID])
    cx, cw = rng.choice(grid, (M, K)), rng.choice(grid, (N, K))
    sx = np.ldexp(1.0, rng.integers(-8, 8, (M, K // 32)))
    sw = np.ldexp(1.0, rng.integers(-8, 8, (N, K // 32)))
    a = np.array([0.5, 4.0])
    out = O.w4a4_gemm(cx, sx, cw, sw, a, fmt)
    for m in range(M):
        for n in range(N):
            acc = sum(Fr(float(cx[m, k])) * Fr(float(sx[m, k // 32])) * Fr(float(cw[n, k])) *
                      Fr(float(sw[n, k // 32])) for k in range(K))
            assert out[m, n] == float(acc * Fr(float(a[n])))
    # the eq. (1) identity: with the solver's state, the product approximates X W^T
    W = _small_matrix(64, 128, seed=32)
    r = O.solve(W, fmt, 3)
    X = rng.standard_normal((16, 128))
    cxa, sxa = O.act_rescale_quant(X, r["b"], fmt)
    approx = O.w4a4_gemm(cxa, sxa, r["codes"], r["scales"], r["a"], fmt)
    exact = X @ W.T
    assert np.linalg.norm(approx - exact) < 0.25 * np.linalg.norm(exact)


def test_w4a4_gemm_nvfp4_against_explicit_sums():
    # NVFP4: E4M3 group scales per 16 elements and the weights' tensor scale,
    # out[m, n] = a_n ts_w sum_k (c_x s_x)(c_w s_w), written out with fractions
    fmt = O.preset("nvfp4")
    rng = np.random.default_rng(33)
    M, N, K = 3, 2, 48
    grid = np.concatenate([O.E2M1_GRID, -O.E2M1_GRID])
    e4m3 = O.decode_e4m3(np.arange(1, 127, dtype=np.uint8))       # positive finite values
    cx, cw = rng.choice(grid, (M, K)), rng.choice(grid, (N, K))
    sx, sw = rng.choice(e4m3, (M, K // 16)), rng.choice(e4m3, (N, K // 16))
    a = np.array([0.75, 3.0])
    ts = 2.0 ** -7
    out = O.w4a4_gemm(cx, sx, cw, sw, a, fmt, ts)
    for m in range(M):
        for n in range(N):
            acc = sum(Fr(float(cx[m, k])) * Fr(float(sx[m, k // 16])) * Fr(float(cw[n, k])) *
                      Fr(float(sw[n, k // 16])) for k in range(K))
            want = acc * Fr(ts) * Fr(float(a[n]))
            assert abs(Fr(float(out[m, n])) - want) <= abs(want) * Fr(2) ** -50
    # the eq. (1) identity with the NVFP4 solve (tensor scale from W) and
    # activations quantized with ts = 1
    W = _small_matrix(64, 128, seed=34)
    r = O.solve(W, fmt, 3)
    assert r["ts"] != 1.0
    X = rng.standard_normal((16, 128))
    cxa, sxa = O.act_rescale_quant(X, r["b"], fmt)
    approx = O.w4a4_gemm(cxa, sxa, r["codes"], r["scales"], r["a"], fmt, r["ts"])
    exact = X @ W.T
    assert np.linalg.norm(approx - exact) < 0.2 * np.linalg.norm(exact)
    # without the tensor scale the product is off by 1/ts
    wrong = O.w4a4_gemm(cxa, sxa, r["codes"], r["scales"], r["a"], fmt)
    assert np.linalg.norm(wrong - exact) > 0.9 * np.linalg.norm(exact)
