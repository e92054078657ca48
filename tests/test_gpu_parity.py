"""GPU path versus the fp64 oracle, element by element, on seeded inputs.

Bars (derived from the method's arithmetic):
* codes and group scales of Q given identical (a, b, ts): bit-exact;
* activation codes and scales given identical b: bit-exact;
* one half-step from an identical state: unprojected ratios within 1e-5
  relative (float32 sums over <= 28672 terms against fp64); projected E8M0
  scales equal; projected BF16 scales equal except where the ratio lies
  within 1e-5 of a bf16 rounding boundary (counted, at most 1e-3 of the
  scales);
* after T iterations: every mse_trace entry within 1e-4 relative; E8M0
  scales of the whole trajectory equal to the oracle's.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from _helpers import (MX_MORE, PRESET_COMBOS, check_projected, code_boundaries, gpu_scales_np,
                      lib_format, np64, oracle_encoded, random_outer)

pytestmark = pytest.mark.gpu

dq = pytest.importorskip("dual_scale_solver_b200")

ALL = list(PRESET_COMBOS)
DEFAULT_G = {"int4_bf16": 64, "mxint4": 32, "mxfp4": 32, "nvfp4": 16,
             "mxint4_bf16outer": 32, "mxfp4_bf16outer": 32, "nvfp4_ts1": 16,
             **{n: 32 for n in MX_MORE}}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from dual_scale_solver_b200 import build
    build.build()


def _weights(rows, cols, dtype, key=7, scale=0.02, outliers=0.01):
    n = rows * cols
    w = synth.student_t4(synth.stream_key(90, key, rows, cols), n).view(rows, cols) * scale
    k = max(1, int(round(outliers * cols)))
    idx = synth.distinct_indices(synth.stream_key(91, key, cols), cols, k)
    w[:, idx] *= 10
    return w.to(dtype)


# --------------------------------------------------------------------------- #
# Q itself
# --------------------------------------------------------------------------- #

@pytest.mark.parametrize("name", ALL)
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("shape", [(300, 2240), (37, 576), (5, 64)])
def test_quantize_bit_exact(name, dtype, shape):
    G = DEFAULT_G[name]
    rows, cols = shape
    if cols % G:
        pytest.skip("shape not a multiple of G")
    fo = PRESET_COMBOS[name](G)
    fl = lib_format(name, G)
    W = _weights(rows, cols, dtype, key=ALL.index(name))
    a = random_outer(fo, rows, synth.stream_key(92, rows))
    b = random_outer(fo, cols, synth.stream_key(93, cols))
    ts = 2.0 ** -10 if fo.tensor_scale_auto else 1.0
    Wd = W.cuda()
    codes, gs = dq.quantize(Wd, fl, torch.tensor(a, dtype=torch.float32, device="cuda"),
                            torch.tensor(b, dtype=torch.float32, device="cuda"), ts)
    torch.cuda.synchronize()
    ec, es = oracle_encoded(np64(W), a, b, fo, ts)
    gc, gsn = codes.cpu().numpy(), gpu_scales_np(gs)
    bad_s = np.argwhere(gsn != es)
    assert bad_s.size == 0, f"{len(bad_s)} group scales differ, first {bad_s[:5].tolist()}"
    bad_c = np.argwhere(gc != ec)
    assert bad_c.size == 0, f"{len(bad_c)} code bytes differ, first {bad_c[:5].tolist()}"


def _tie_matrix(fo, kind):
    """fp32 rows whose values sit exactly on decision boundaries of Q (and one
    float32 ulp either side) for a = b = non-trivial BF16/E8M0 values."""
    G = fo.group
    rows = []
    rng = np.random.default_rng(3)
    # decision boundaries of the code grid (midpoints of code magnitudes)
    grid = code_boundaries(fo)
    for r in range(24):
        s = 2.0 ** int(rng.integers(-9, -3))
        if fo.gscale == "bf16":
            s *= 1 + int(rng.integers(0, 8)) / 8.0
        vals = [fo.qmax * s]                    # fixes the group max: g = s exactly
        while len(vals) < G:
            q = grid[int(rng.integers(0, len(grid)))]
            v = q * s * (1 if rng.random() < 0.5 else -1)
            if kind == 1:
                v = float(np.nextafter(np.float32(v), np.float32(np.inf)))
            elif kind == 2:
                v = float(np.nextafter(np.float32(v), np.float32(-np.inf)))
            vals.append(v)
        rows.append(vals * 2)
    return np.array(rows, dtype=np.float32).astype(np.float64)


@pytest.mark.parametrize("name", ALL)
@pytest.mark.parametrize("kind", [0, 1, 2])
def test_quantize_ties_and_neighbours(name, kind):
    G = DEFAULT_G[name]
    fo = PRESET_COMBOS[name](G)
    fl = lib_format(name, G)
    Y = _tie_matrix(fo, kind)                        # quantizer input for a = b = 1
    rows, cols = Y.shape
    a_val = 1.0 if fo.oscale == "e8m0" else 1.125    # BF16 outer: exercise inexact paths
    a = np.full(rows, a_val)
    b = np.ones(cols)
    W = (Y * a_val).astype(np.float32)
    ts = 1.0
    Wd = torch.from_numpy(W).cuda()
    codes, gs = dq.quantize(Wd, fl, torch.tensor(a, dtype=torch.float32, device="cuda"),
                            torch.tensor(b, dtype=torch.float32, device="cuda"), ts)
    ec, es = oracle_encoded(W.astype(np.float64), a, b, fo, ts)
    assert np.array_equal(gpu_scales_np(gs), es)
    assert np.array_equal(codes.cpu().numpy(), ec)


def test_group_scale_ties_bf16():
    # group max exactly 7 * (bf16 midpoint) * a: the scale rounds to the even neighbour
    fo = O.preset("int4_bf16", 16)
    fl = dq.format_preset("int4_bf16", 16)
    mids = []
    for k in range(40):
        lo = (1 + k / 128.0) * 2.0 ** -5
        mids.append(lo + 2.0 ** -13)                  # half a bf16 ulp above lo
    a = 1.0 + 3 / 128.0
    W = np.zeros((len(mids), 16), dtype=np.float32)
    for i, m in enumerate(mids):
        W[i, 0] = 7 * m * a
        W[i, 1] = np.nextafter(np.float32(7 * m * a), np.float32(0))
    assert np.all(W[:, 0].astype(np.float64) == 7 * np.array(mids) * a)
    av = np.full(len(mids), a)
    codes, gs = dq.quantize(torch.from_numpy(W).cuda(), fl,
                            torch.tensor(av, dtype=torch.float32, device="cuda"), None, 1.0)
    ec, es = oracle_encoded(W.astype(np.float64), av, np.ones(16), fo)
    assert np.array_equal(gpu_scales_np(gs), es)
    assert np.array_equal(codes.cpu().numpy(), ec)


# --------------------------------------------------------------------------- #
# Activation rescale + quantize
# --------------------------------------------------------------------------- #

@pytest.mark.parametrize("name", ["int4_bf16", "nvfp4", "mxfp4", "mxint4"] + MX_MORE)
@pytest.mark.parametrize("tokens", [1, 333])
def test_act_rescale_quant_bit_exact(name, tokens):
    G = DEFAULT_G[name]
    fo = PRESET_COMBOS[name](G)
    fl = dq.format_preset(name, G)
    K = 4096
    wl = synth.WORKLOADS["llama31_8b_int4_g64"]
    X = synth.activation(wl, tokens=tokens)
    b = random_outer(fo, K, synth.stream_key(94, K))
    codes, gs = dq.act_rescale_quant(X.cuda(), torch.tensor(b, dtype=torch.float32, device="cuda"), fl)
    c, s = O.act_rescale_quant(np64(X), b, fo)
    assert np.array_equal(gpu_scales_np(gs), O.encode_scales(s, fo))
    assert np.array_equal(codes.cpu().numpy(), O.encode_codes(c, fo))


# --------------------------------------------------------------------------- #
# One half-step from an identical state
# --------------------------------------------------------------------------- #

@pytest.mark.parametrize("name", ALL)
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_half_steps_from_identical_state(name, dtype):
    G = DEFAULT_G[name]
    fo = PRESET_COMBOS[name](G)
    fl = lib_format(name, G)
    rows, cols = 333, 4160
    W = _weights(rows, cols, dtype, key=11)
    W64 = np64(W)
    a = random_outer(fo, rows, synth.stream_key(95, 1), 0.3)
    b = random_outer(fo, cols, synth.stream_key(95, 2), 0.3)
    ts = O.tensor_scale(W64, fo)
    Wd = W.cuda()
    ad = torch.tensor(a, dtype=torch.float32, device="cuda")
    bd = torch.tensor(b, dtype=torch.float32, device="cuda")
    # row step
    a_gpu, a_pre, mse0 = dq.row_update(Wd, fl, ad, bd, ts)
    Qh, _, _ = O.qhat(W64, a, b, fo, ts)
    a_or, x_or = O.row_update(W64, Qh, b, fo)
    pre = np64(a_pre)
    ok = ~np.isnan(x_or)
    assert np.array_equal(np.isnan(pre), np.isnan(x_or))
    assert np.max(np.abs(pre[ok] - x_or[ok]) / x_or[ok]) < 1e-5
    check_projected(np64(a_gpu), a_or, x_or, fo, "a")
    # (4-bit codes: the state's error is formed per row as sum W^2 - 2 a sum
    # W R + a^2 sum R^2 from float32 row sums, each about 100 times the
    # error; wider codes sum (W - a R)^2 directly)
    tol0 = 1e-6 if name in MX_MORE else 2e-5
    assert abs(mse0.item() - O.mse(W64, Qh, a, b)) <= tol0 * O.mse(W64, Qh, a, b)
    # column step from (a_gpu, b)
    a1 = np64(a_gpu)
    b_gpu, b_pre, mse1 = dq.col_update(Wd, fl, a_gpu, bd, ts)
    Qh1, _, _ = O.qhat(W64, a1, b, fo, ts)
    b_or, xb_or = O.col_update(W64, Qh1, a1, fo)
    pre = np64(b_pre)
    ok = ~np.isnan(xb_or)
    assert np.array_equal(np.isnan(pre), np.isnan(xb_or))
    assert np.max(np.abs(pre[ok] - xb_or[ok]) / xb_or[ok]) < 1e-5
    check_projected(np64(b_gpu), b_or, xb_or, fo, "b")
    ref = O.mse(W64, Qh1, a1, b)
    assert abs(mse1.item() - ref) <= 1e-6 * ref


# --------------------------------------------------------------------------- #
# Whole solves
# --------------------------------------------------------------------------- #

def _solve_and_compare(Ws, fo, fl, T, tol=1e-4):
    outs = dq.solve_dual_scale_batched([W.cuda() for W in Ws], fl, T, half=True)
    torch.cuda.synchronize()
    worst = 0.0
    for W, o in zip(Ws, outs):
        W64 = np64(W)
        r = O.solve(W64, fo, T)
        tr = np64(o["mse_trace"])
        rel = np.abs(tr - r["mse_trace"]) / r["mse_trace"]
        worst = max(worst, rel.max())
        assert rel.max() < tol, (rel, tr, r["mse_trace"])
        hf = np64(o["mse_half"])[:T]
        assert np.max(np.abs(hf - r["mse_half"]) / r["mse_half"]) < tol
        assert float(o["tensor_scale"].item()) == r["ts"]
        # the stored codes are Q at the GPU's own final state, bit for bit
        a, b = np64(o["a"]), np64(o["b"])
        ec, es = oracle_encoded(W64, a, b, fo, r["ts"])
        assert np.array_equal(o["codes"].cpu().numpy(), ec)
        assert np.array_equal(gpu_scales_np(o["gscales"]), es)
        # E8M0 scales follow the oracle's trajectory exactly; BF16 scales
        # may part from it after a flip at a rounding boundary (counted)
        if fo.oscale == "e8m0":
            assert np.array_equal(a, r["a"]) and np.array_equal(b, r["b"])
        else:
            same = (np.mean(a == r["a"]) + np.mean(b == r["b"])) / 2
            print(f"trajectory: {np.sum(a != r['a'])} of {a.size} a and "
                  f"{np.sum(b != r['b'])} of {b.size} b differ from the oracle's")
            assert same > 0.97, same
    return worst


def test_solve_toy_workload():
    wl = synth.WORKLOADS["toy256x512_int4_g32"]
    W = synth.weight(wl, 0, 0)
    fo = O.preset(wl.fmt, wl.group)
    fl = dq.format_preset(wl.fmt, wl.group)
    _solve_and_compare([W], fo, fl, wl.T)


@pytest.mark.parametrize("name", ["int4_bf16", "nvfp4", "nvfp4_ts1", "mxfp4"] + MX_MORE)
def test_solve_single_matrix_entry_point(name):
    G = DEFAULT_G[name]
    fo, fl = PRESET_COMBOS[name](G), lib_format(name, G)
    W = _weights(200, 1536, torch.bfloat16, key=5)
    o = dq.solve_dual_scale(W.cuda(), fl, 4)
    torch.cuda.synchronize()
    r = O.solve(np64(W), fo, 4)
    tr = np64(o["mse_trace"])
    assert np.max(np.abs(tr - r["mse_trace"]) / r["mse_trace"]) < 1e-4


@pytest.mark.parametrize("name", MX_MORE)
def test_solve_mx_family_batched(name):
    # three matrices of one batch against the oracle's whole trajectory,
    # codes and scales at the GPU's final state bit for bit
    fo, fl = PRESET_COMBOS[name](32), dq.format_preset(name)
    Ws = [_weights(r, c, torch.bfloat16, key=30 + k)
          for k, (r, c) in enumerate([(300, 2240), (64, 576), (17, 1024)])]
    _solve_and_compare(Ws, fo, fl, 4)


def test_solve_smollm2_decoder0_batched_with_all_30():
    wl = synth.WORKLOADS["smollm2_135m_mxint4_g32"]
    fo = O.preset(wl.fmt, wl.group)
    fl = dq.format_preset(wl.fmt, wl.group)
    mats = wl.matrices
    Ws = [synth.weight(wl, d, i, device="cuda") for d, i, _ in mats]
    outs = dq.solve_dual_scale_batched(Ws, fl, wl.T, half=True)
    torch.cuda.synchronize()
    assert len(outs) == 210
    for k in range(7):                       # decoder 0 against the oracle
        W64 = np64(Ws[k])
        r = O.solve(W64, fo, wl.T)
        tr = np64(outs[k]["mse_trace"])
        assert np.max(np.abs(tr - r["mse_trace"]) / r["mse_trace"]) < 1e-4
        ec, es = oracle_encoded(W64, np64(outs[k]["a"]), np64(outs[k]["b"]), fo)
        assert np.array_equal(outs[k]["codes"].cpu().numpy(), ec)
        assert np.array_equal(gpu_scales_np(outs[k]["gscales"]), es)
    # dual-scale never ends above single-scale (with E8M0 outer scales most of
    # these solves stay at RTN: no b_j leaves 1, in the oracle as well)
    final = np.array([np64(o["mse_trace"])[-1] for o in outs])
    start = np.array([np64(o["mse_trace"])[0] for o in outs])
    # (start and end residuals are summed over different tile shapes: allow
    # float32 summation noise)
    assert np.all(final <= start * (1 + 1e-6))
    assert np.any(final < start * (1 - 1e-4))


def test_solve_is_deterministic():
    wl = synth.WORKLOADS["llama31_8b_nvfp4_g16"]
    fl = dq.format_preset(wl.fmt, wl.group)
    Ws = [synth.weight(wl, 0, i, device="cuda", rows=512, cols=1024) for i in range(3)]
    o1 = dq.solve_dual_scale_batched(Ws, fl, 3)
    o2 = dq.solve_dual_scale_batched(Ws, fl, 3)
    torch.cuda.synchronize()
    for x, y in zip(o1, o2):
        for k in ("codes", "gscales", "a", "b", "mse_trace"):
            assert torch.equal(x[k], y[k]), k


# --------------------------------------------------------------------------- #
# Edge cases and device status
# --------------------------------------------------------------------------- #

def test_empty_and_degenerate_shapes():
    fl = dq.format_preset("mxfp4")
    W = torch.zeros(0, 64, dtype=torch.bfloat16, device="cuda")
    o = dq.solve_dual_scale(W, fl, 2)
    torch.cuda.synchronize()
    assert o["a"].numel() == 0
    # all-zero matrix: scales stay 1, codes 0, mse 0
    Z = torch.zeros(40, 96, dtype=torch.bfloat16, device="cuda")
    o = dq.solve_dual_scale(Z, fl, 3)
    torch.cuda.synchronize()
    assert torch.all(o["a"] == 1) and torch.all(o["b"] == 1)
    assert torch.all(o["codes"] == 0) and torch.all(o["mse_trace"] == 0)
    assert torch.all(o["gscales"] == 127)
    # one group wide, one row tall
    W = _weights(1, 32, torch.bfloat16).cuda()
    o = dq.solve_dual_scale(W, fl, 2)
    torch.cuda.synchronize()
    r = O.solve(np64(W), O.preset("mxfp4"), 2)
    assert np.allclose(np64(o["mse_trace"]), r["mse_trace"], rtol=1e-4, atol=0)
    assert dq.last_device_status() == 0


@pytest.mark.parametrize("bad", [float("nan"), float("inf")])
def test_nonfinite_input_sets_device_flag(bad):
    fl = dq.format_preset("int4_bf16")
    W = _weights(64, 128, torch.bfloat16).cuda()
    W[3, 17] = bad
    assert dq.last_device_status() == 0
    dq.solve_dual_scale(W, fl, 1)
    assert dq.last_device_status() == -4
    assert dq.last_device_status() == 0      # read clears
    dq.quantize(W, fl)
    assert dq.last_device_status() == -4


# --------------------------------------------------------------------------- #
# MX formats: one-pass iterations against the literal steps
# --------------------------------------------------------------------------- #

def _literal_sequence(W, fl, T, a0, b0):
    """T iterations through the step entry points (literal row pass, then
    literal column pass with the new a)."""
    a, b = a0.clone(), b0.clone()
    for _ in range(T):
        a, _, _ = dq.row_update(W, fl, a, b)
        b, _, _ = dq.col_update(W, fl, a, b)
    return a, b


@pytest.mark.parametrize("name", ["mxfp4", "mxint4"] + MX_MORE)
@pytest.mark.parametrize("extreme", [None, -124, 126])
def test_mx_solve_equals_the_literal_steps(name, extreme):
    # With power-of-two scales the solve takes both statistics of an
    # iteration from one pass; the result must equal the literal row and
    # column steps bit for bit.  extreme = -124: rows whose a0 = 2^-124 still
    # keep every group exponent in range (no fallback); extreme = 126: group
    # exponents of those rows clamp, so the iteration falls back to the
    # literal passes.
    fl = dq.format_preset(name)
    fo = PRESET_COMBOS[name](32)
    rows, cols = 300, 2240
    W = _weights(rows, cols, torch.bfloat16, key=23).cuda()
    a0 = torch.ones(rows, device="cuda")
    if extreme is not None:
        a0[::7] = 2.0 ** extreme
    b0 = torch.ones(cols, device="cuda")
    T = 4
    o = dq.solve_dual_scale(W, fl, T, a0=a0, b0=b0)
    a, b = _literal_sequence(W, fl, T, a0, b0)
    torch.cuda.synchronize()
    assert torch.equal(o["a"], a)
    assert torch.equal(o["b"], b)
    tr, hf = np64(o["mse_trace"]), np64(o["mse_half"])
    if extreme is None:
        r = O.solve(np64(W), fo, T)
        assert np.max(np.abs(tr - r["mse_trace"]) / r["mse_trace"]) < 1e-4
        # a power-of-two row step leaves D_a Qhat unchanged: half == trace
        assert np.array_equal(hf, tr[:T])
        assert dq.last_device_status() == 0
    else:
        # extreme scales can push float32 statistics out of range; the device
        # reports it (and the literal steps agree with the solve all the same)
        assert dq.last_device_status() in (0, -4, -5)


# spread of log(b0) per format, wide enough that some columns' values fall
# where the element grid is coarse (fixed-point or subnormal codes), so that
# column ratios leave [0.75, 1.5) and b moves; MXFP8 E5M2 would need a range
# of 2^32, so only its zero columns move
_MOVING_SPREAD = {"mxfp4": 1.5, "mxint4": 1.5, "mxint8": 6.0, "mxfp6_e2m3": 6.0,
                  "mxfp6_e3m2": 6.0, "mxfp8_e4m3": 12.0, "mxfp8_e5m2": 1.5}


def _moving_state(name, fo, rows=300, cols=2240):
    """Weights and a seeded E8M0 starting state (a0, b0) from which the solve
    moves.  Rows 0-3 repeat, per group of 32, one element at (113/32) 2^-6-r
    and 31 at +-(33/64) 2^-6-r (times a0_r b0_j): MXINT4 codes 4 and +-1, a
    row ratio of about 0.64, so a_r halves.  Row 4 and columns 7 and 1000
    are zero and start away from 1: their scales return to 1."""
    a0 = random_outer(fo, rows, synth.stream_key(98, 1), 1.5)
    b0 = random_outer(fo, cols, synth.stream_key(98, 2), _MOVING_SPREAD[name])
    a0[4], b0[7], b0[1000] = 4.0, 2.0, 0.25
    W = _weights(rows, cols, torch.float32, key=23)
    pat = torch.tensor([33 / 64 if k % 2 else -33 / 64 for k in range(32)])
    pat[5] = 113 / 32
    b0t = torch.tensor(b0, dtype=torch.float32)
    for r in range(4):
        W[r] = pat.repeat(cols // 32) * b0t * float(a0[r]) * 2.0 ** (-6 - r)
    W[4] = 0.0
    W[:, [7, 1000]] = 0.0
    return W.to(torch.bfloat16), a0, b0


@pytest.mark.parametrize("name", ["mxfp4", "mxint4"])
def test_exactly_representable_matrix_has_zero_error(name):
    # Every group is codes times a power of two with the top code in it, so Q
    # reproduces W and a = b = 1 stay.  The one-pass iterations of the 4-bit
    # formats take each row's error from its row sums, sum W^2 - 2 sum W R +
    # sum R^2, with sum W^2 summed in the order of the other two: for such a
    # row the three are the same bits and the error is exactly 0.
    fl = dq.format_preset(name)
    g = torch.Generator().manual_seed(41)
    rows, cols = 200, 2240                      # ragged: 2240 = 8.75 x 256
    if name == "mxfp4":
        grid = torch.tensor([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
        top = 6.0
    else:
        grid = torch.arange(0.0, 8.0)
        top = 7.0
    vals = grid[torch.randint(0, len(grid), (rows, cols), generator=g)]
    vals = vals * (torch.randint(0, 2, (rows, cols), generator=g) * 2.0 - 1.0)
    v3 = vals.view(rows, cols // 32, 32)
    v3[:, :, 5] = top * (torch.randint(0, 2, (rows, cols // 32), generator=g) * 2.0 - 1.0)
    e = torch.randint(-12, 6, (rows, cols // 32), generator=g).double()
    W = (v3.double() * torch.pow(2.0, e)[:, :, None]).reshape(rows, cols)
    W[17] = 0.0
    T = 3
    o = dq.solve_dual_scale(W.to(torch.bfloat16).cuda(), fl, T)
    torch.cuda.synchronize()
    assert torch.all(o["mse_trace"] == 0) and torch.all(o["mse_half"] == 0)
    assert torch.all(o["a"] == 1) and torch.all(o["b"] == 1)


@pytest.mark.parametrize("name", ["mxfp4", "mxint4"] + MX_MORE)
def test_mx_solve_from_a_moving_state(name):
    # The one-pass iteration from a seeded state with a != 1 and b != 1 whose
    # scales are updated: equal to the literal row and column steps bit for
    # bit, and to the oracle's whole trajectory (E8M0 scales exactly, MSE
    # within 1e-4).  A slip in the fused path's row values (Qhat s) b_j or in
    # the 1/a scaling of its row sums would show here.
    fl = dq.format_preset(name)
    fo = PRESET_COMBOS[name](32)
    W, a0, b0 = _moving_state(name, fo)
    Wd = W.cuda()
    a0d = torch.tensor(a0, dtype=torch.float32, device="cuda")
    b0d = torch.tensor(b0, dtype=torch.float32, device="cuda")
    T = 4
    o = dq.solve_dual_scale(Wd, fl, T, a0=a0d, b0=b0d)
    # the literal steps, iteration by iteration, recording which scales move
    a, b = a0d.clone(), b0d.clone()
    moved_a, moved_b, lit_mse = [], [], []
    for _ in range(T):
        a1, _, m = dq.row_update(Wd, fl, a, b)
        b1, _, _ = dq.col_update(Wd, fl, a1, b)
        moved_a.append(np.flatnonzero((a1 != a).cpu().numpy()))
        moved_b.append(np.flatnonzero((b1 != b).cpu().numpy()))
        lit_mse.append(m.item())
        a, b = a1, b1
    torch.cuda.synchronize()
    assert torch.equal(o["a"], a) and torch.equal(o["b"], b)
    # the one-pass squared error (for 4-bit codes from the row sums, sum W^2
    # - 2 sum W R + sum R^2) against the literal row pass's sum of (W - R)^2
    # at the same states
    lit = np.array(lit_mse)
    assert np.max(np.abs(np64(o["mse_trace"])[:T] - lit) / lit) < 2e-5
    # the state moves: the zero row and columns in the first iteration, and
    # (but for MXFP8 E5M2) other columns; MXINT4's constructed rows halve a
    assert 4 in moved_a[0] and {7, 1000} <= set(moved_b[0].tolist())
    if name != "mxfp8_e5m2":
        assert len(set(np.concatenate(moved_b).tolist()) - {7, 1000}) > 0
    if name == "mxint4":
        assert {0, 1, 2, 3} <= set(moved_a[0].tolist())
    # the oracle's trajectory from the same state
    r = O.solve(np64(W), fo, T, a0=a0, b0=b0)
    assert np.array_equal(np64(o["a"]), r["a"]) and np.array_equal(np64(o["b"]), r["b"])
    tr, hf = np64(o["mse_trace"]), np64(o["mse_half"])
    assert np.max(np.abs(tr - r["mse_trace"]) / r["mse_trace"]) < 1e-4
    assert np.array_equal(hf, tr[:T])
    ec, es = oracle_encoded(np64(W), r["a"], r["b"], fo)
    assert np.array_equal(o["codes"].cpu().numpy(), ec)
    assert np.array_equal(gpu_scales_np(o["gscales"]), es)
    assert dq.last_device_status() == 0


@pytest.mark.parametrize("name", ["mxint4", "mxint8", "mxfp8_e4m3", "mxfp6_e2m3", "mxfp4"])
def test_literal_steps_small_row_scales_with_zero_groups(name):
    # The literal row and column steps (also the fallback of the one-pass
    # iteration) with row scales a = 2^-8 on a matrix whose last column block
    # is partly past the last column (2240 columns) and with all-zero groups:
    # an all-zero group (and a lane past the last column) takes scale 1, so
    # 1 / (a s) stays finite; E8M0 scales exactly as the oracle's.
    fl, fo = dq.format_preset(name), PRESET_COMBOS[name](32)
    rows, cols = 64, 2240
    W = _weights(rows, cols, torch.bfloat16, key=31)
    W[3, 64:96] = 0.0                                  # one all-zero group
    W[7] = 0.0                                         # an all-zero row
    W64 = np64(W)
    a = np.full(rows, 2.0 ** -8)
    b = random_outer(fo, cols, synth.stream_key(95, 7), 0.7)
    ad = torch.tensor(a, dtype=torch.float32, device="cuda")
    bd = torch.tensor(b, dtype=torch.float32, device="cuda")
    dq.last_device_status()
    a1, a1pre, _ = dq.row_update(W.cuda(), fl, ad, bd)
    b1, b1pre, _ = dq.col_update(W.cuda(), fl, a1, bd)
    torch.cuda.synchronize()
    assert dq.last_device_status() == 0
    Qh, _, _ = O.qhat(W64, a, b, fo)
    a_or, x_or = O.row_update(W64, Qh, b, fo)
    check_projected(np64(a1), a_or, x_or, fo, "a")
    Qh1, _, _ = O.qhat(W64, np64(a1), b, fo)
    b_or, xb_or = O.col_update(W64, Qh1, np64(a1), fo)
    check_projected(np64(b1), b_or, xb_or, fo, "b")


@pytest.mark.parametrize("name", ["mxfp4", "mxint8"])
def test_mx_group_exponent_out_of_range_falls_back(name):
    # Rows scaled by 2^-112 and 2^108 give group scales 2^e with |e| > 100 on
    # the one-pass iteration, which then redoes its steps literally; the
    # solve equals the literal steps bit for bit (float32 statistics of such
    # rows leave the normal range, so the comparison is on the bits and the
    # device status may report it).
    fl = dq.format_preset(name)
    rows, cols = 300, 2240
    W = _weights(rows, cols, torch.float32, key=29)
    W[::5] *= 2.0 ** -112
    W[1::5] *= 2.0 ** 108
    W = W.to(torch.bfloat16).cuda()
    a0 = torch.ones(rows, device="cuda")
    b0 = torch.ones(cols, device="cuda")
    T = 3
    o = dq.solve_dual_scale(W, fl, T, a0=a0, b0=b0)
    a, b = _literal_sequence(W, fl, T, a0, b0)
    torch.cuda.synchronize()
    assert torch.equal(o["a"].view(torch.int32), a.view(torch.int32))
    assert torch.equal(o["b"].view(torch.int32), b.view(torch.int32))
    assert dq.last_device_status() in (0, -4, -5)


def test_batched_mx_solve_equals_single_solves():
    wl = synth.WORKLOADS["llama31_70b_decoder_mxfp4_g32"]
    fl = dq.format_preset(wl.fmt, wl.group)
    Ws = [synth.weight(wl, 0, i, device="cuda", rows=r, cols=c)
          for i, (r, c) in enumerate([(512, 1024), (96, 2048), (300, 512)])]
    outs = dq.solve_dual_scale_batched(Ws, fl, 3)
    for W, o in zip(Ws, outs):
        s = dq.solve_dual_scale(W, fl, 3)
        torch.cuda.synchronize()
        for k in ("codes", "gscales", "a", "b"):
            assert torch.equal(o[k], s[k]), k
        assert torch.equal(o["mse_trace"], s["mse_trace"])


@pytest.mark.parametrize("name", ALL)
def test_dequantize_reconstruction(name):
    # D_a Qhat D_b from stored codes and scales: c * (s * ts) is exact in
    # float32 for every code set; the products with a_i and b_j round twice
    G = DEFAULT_G[name]
    fo, fl = PRESET_COMBOS[name](G), lib_format(name, G)
    rows, cols = 37, 8 * G
    W = _weights(rows, cols, torch.float32, key=40)
    a = random_outer(fo, rows, synth.stream_key(96, rows))
    b = random_outer(fo, cols, synth.stream_key(96, cols))
    ts = 2.0 ** -10 if fo.tensor_scale_auto else 1.0
    ad = torch.tensor(a, dtype=torch.float32, device="cuda")
    bd = torch.tensor(b, dtype=torch.float32, device="cuda")
    codes, gs = dq.quantize(W.cuda(), fl, ad, bd, ts)
    out = dq.dequantize(codes, gs, rows, cols, fl, ts, ad, bd)
    torch.cuda.synchronize()
    c = O.decode_codes(codes.cpu().numpy(), fo)
    s = O.decode_scales(gpu_scales_np(gs), fo)
    ref = a[:, None] * O.dequantize(c, s, fo, ts) * b[None, :]
    got = np64(out)
    assert np.all(np.abs(got - ref) <= 2.0 ** -22 * np.abs(ref))


def test_measurement_support():
    # event timing of selected tile-kernel kinds and the launch counter
    fl = dq.format_preset("mxfp4")
    W = _weights(256, 1024, torch.bfloat16, key=41).cuda()
    dq.solve_dual_scale(W, fl, 2)                # warm
    torch.cuda.synchronize()
    for k in range(5):
        dq.kernel_time(k)
    n0 = dq.launch_count()
    dq.kernel_timing(True, kinds=[dq.KIND_FUSED])
    dq.solve_dual_scale(W, fl, 3)
    torch.cuda.synchronize()
    ms, n = dq.kernel_time(dq.KIND_FUSED)
    ms_pack, n_pack = dq.kernel_time(dq.KIND_PACK)
    dq.kernel_timing(False)
    assert n == 3 and ms > 0.0                   # one fused pass per iteration
    assert n_pack == 0                            # kinds not selected are not timed
    assert dq.launch_count() - n0 >= 3 * 5 + 1    # per iteration: fused, 2 gated, 2 finalize, mse
