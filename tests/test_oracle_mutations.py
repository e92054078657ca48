"""The oracle's pins catch plausible mistakes: each mistake below is planted
in the oracle (on the CPU, by monkeypatching one of its functions) and at
least one of the pins in test_oracle_solver.py / test_oracle_formats.py must
then fail.  Nothing here touches the GPU path."""
import numpy as np
import pytest

import oracle as O
from oracle import formats as F
from oracle import solver as S

import test_oracle_formats as TF
import test_oracle_solver as TS

_row, _col, _quantize, _inner = S.row_update, S.col_update, S.quantize, S.inner
_e8m0_nearest, _round_e2m1, _round_int4 = F.e8m0_nearest, F.round_e2m1, F.round_int4


def _row_no_db(W, Qh, b, fmt):                      # R = Qhat instead of Qhat D_b
    return _row(W, Qh, np.ones_like(b), fmt)


def _row_inverted(W, Qh, b, fmt):                   # <R,R> / <W,R> instead of <W,R> / <R,R>
    R = Qh * b[None, :]
    num, den = np.sum(W * R, axis=1), np.sum(R * R, axis=1)
    pos = num > 0
    x = np.where(pos, den / np.where(pos, num, 1.0), np.nan)
    return np.where(pos, S.project_outer(np.where(pos, x, 1.0), fmt), 1.0), x


def _col_no_da(W, Qh, a, fmt):                      # S = Qhat instead of D_a Qhat
    return _col(W, Qh, np.ones_like(a), fmt)


def _quantize_no_ts(Y, fmt, ts=1.0):                # the tensor scale dropped
    return _quantize(Y, fmt, 1.0)


def _inner_no_a(W, a, b):                           # grid input W / b instead of W / (a b)
    return W / b[None, :]


def _e8m0_tie_down(x):                              # an exact tie goes down
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    k = np.where(m <= 0.75, e - 1, e).astype(np.int64)
    return np.ldexp(1.0, np.clip(k, F.E8M0_EMIN, F.E8M0_EMAX))


def _e2m1_ties_away(q):                             # ties away from zero
    q = np.asarray(q, dtype=np.float64)
    grid = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    a = np.minimum(np.abs(q), 6.0)
    d = np.abs(a[..., None] - grid)
    best = np.where(d == d.min(-1, keepdims=True), grid, -1.0).max(-1)
    return np.copysign(best, q)


def _int4_clamp_7(q):                               # clamps to [-7, 7]
    return np.clip(_round_int4(q), -7, 7)


def _solve_with(order):
    """The oracle's loop with one slip in the order of its steps."""
    def solve(W, fmt, T, a0=None, b0=None):
        W = np.asarray(W, dtype=np.float64)
        rows, cols = W.shape
        a = np.ones(rows) if a0 is None else np.asarray(a0, dtype=np.float64).copy()
        b = np.ones(cols) if b0 is None else np.asarray(b0, dtype=np.float64).copy()
        ts = S.tensor_scale(W, fmt)
        Qh, c, s = S.qhat(W, a, b, fmt, ts)
        trace, half = [S.mse(W, Qh, a, b)], []
        for _ in range(T):
            if order == "column first":
                b, _ = S.col_update(W, Qh, a, fmt)
                Qh, c, s = S.qhat(W, a, b, fmt, ts)
                half.append(S.mse(W, Qh, a, b))
                a, _ = S.row_update(W, Qh, b, fmt)
            else:
                a, _ = S.row_update(W, Qh, b, fmt)
                if order != "no re-quantize":
                    Qh, c, s = S.qhat(W, a, b, fmt, ts)
                if order != "half after column":
                    half.append(S.mse(W, Qh, a, b))
                b, _ = S.col_update(W, Qh, a, fmt)
            Qh, c, s = S.qhat(W, a, b, fmt, ts)
            if order == "half after column":
                half.append(S.mse(W, Qh, a, b))
            trace.append(S.mse(W, Qh, a, b))
        return dict(a=a, b=b, codes=c, scales=s, ts=ts, qhat=Qh,
                    mse_trace=np.array(trace), mse_half=np.array(half))
    return solve


_ORDER_PINS = [(TS.test_solve_follows_the_step_order_exactly, c) for c in TS.ORDER_CASES]


MUTATIONS = {
    "row update without D_b": ([(S, "row_update", _row_no_db), (O, "row_update", _row_no_db)],
                               [(TS.test_row_and_column_updates_minimise_over_the_scale_set, ("int4_bf16",))]),
    "inverted closed form": ([(S, "row_update", _row_inverted), (O, "row_update", _row_inverted)],
                             [(TS.test_closed_form_ratio_direction, ())]),
    "column update without D_a": ([(S, "col_update", _col_no_da), (O, "col_update", _col_no_da)],
                                  [(TS.test_row_and_column_updates_minimise_over_the_scale_set, ("int4_bf16",))]),
    "tensor scale dropped": ([(S, "quantize", _quantize_no_ts), (O, "quantize", _quantize_no_ts)],
                             [(TS.test_quantize_matches_exact_rational_restatement, ("nvfp4", 16))]),
    "a dropped from the grid input": ([(S, "inner", _inner_no_a), (O, "inner", _inner_no_a)],
                                      [(TS.test_quantize_matches_exact_rational_restatement, ("int4_bf16", 32))]),
    "E8M0 tie rounded down": ([(F, "e8m0_nearest", _e8m0_tie_down), (O, "e8m0_nearest", _e8m0_tie_down)],
                              [(TF.test_e8m0_nearest_brute_force, ())]),
    "E2M1 ties away from zero": ([(F, "round_e2m1", _e2m1_ties_away), (O, "round_e2m1", _e2m1_ties_away)],
                                 [(TF.test_e2m1_hand_cases, ())]),
    "INT4 clamped to [-7, 7]": ([(F, "round_int4", _int4_clamp_7), (O, "round_int4", _int4_clamp_7)],
                                [(TF.test_int4_half_even_matches_python_round, ()),
                                 (TS.test_quantize_matches_exact_rational_restatement, ("int4_bf16", 16))]),
    # the order of the steps (text under eq. (2) of the daiwk note)
    "column step first": ([(S, "solve", _solve_with("column first")),
                           (O, "solve", _solve_with("column first"))], _ORDER_PINS),
    "no re-quantize between the steps": ([(S, "solve", _solve_with("no re-quantize")),
                                          (O, "solve", _solve_with("no re-quantize"))], _ORDER_PINS),
    "mse_half after the column step": ([(S, "solve", _solve_with("half after column")),
                                        (O, "solve", _solve_with("half after column"))], _ORDER_PINS),
}


@pytest.mark.parametrize("name", list(MUTATIONS))
def test_planted_mistake_fails_a_pin(name, monkeypatch):
    patches, pins = MUTATIONS[name]
    for mod, attr, fn in patches:
        assert hasattr(mod, attr), (mod, attr)
        monkeypatch.setattr(mod, attr, fn)
    failed = []
    for pin, args in pins:
        try:
            pin(*args)
        except Exception as e:          # an assertion, or a shape/encoding error
            failed.append((pin.__name__, type(e).__name__))
    assert failed, f"no pin caught: {name}"


def test_unmutated_pins_pass():
    # the same pins pass on the oracle as it stands
    for _, pins in MUTATIONS.values():
        for pin, args in pins:
            pin(*args)
