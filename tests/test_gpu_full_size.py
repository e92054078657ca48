"""GPU parity at the workloads' full sizes, in the batched launch configuration
the benchmark times, on outputs the oracle can compute one by one.

For every workload all of its matrices are solved in one batched call with
the workload's T.  Then, on seeded samples:
* rows of the final codes and group scales are bit-exact against the oracle's
  Q at the GPU's own final (a, b);
* one row step and one column step from the final state: unprojected ratios
  within 1e-5 relative of the oracle's; projected E8M0 scales equal, BF16
  scales equal away from a bf16 rounding boundary;
* the final MSE equals the MSE of the dequantized codes (checked in fp64);
* one small full-size matrix of each set runs the oracle's whole T-iteration
  solve (MSE trace within 1e-4 relative);
* the activation path at its full size, sampled token rows bit-exact.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from _helpers import check_projected, gpu_scales_np, np64

pytestmark = pytest.mark.gpu

dq = pytest.importorskip("dual_scale_solver_b200")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from dual_scale_solver_b200 import build
    build.build()


def _sample(n, k, key):
    return np.sort(synth.distinct_indices(synth.stream_key(99, key, n), n, min(k, n)).numpy())


def _check_matrix(W, o, fo, fl, key, n_rows=12, n_groups=4):
    """Sampled checks of one solved matrix."""
    rows, cols = W.shape
    G = fo.group
    a, b = np64(o["a"]), np64(o["b"])
    ts = float(o["tensor_scale"].item())
    amax = float(W.abs().max().item())                 # torch's exact max of |W|
    assert ts == O.tensor_scale(np.array([[amax]]), fo)
    ri = _sample(rows, n_rows, key)
    Wr = np64(W[ri])
    # final codes and group scales of the sampled rows
    c, s = O.quantize(O.inner(Wr, a[ri], b), fo, ts)
    assert np.array_equal(o["codes"][ri].cpu().numpy(), O.encode_codes(c, fo))
    assert np.array_equal(gpu_scales_np(o["gscales"][ri]), O.encode_scales(s, fo))
    # one row step from the final state
    ad, bd = o["a"], o["b"]
    a1, a1pre, _ = dq.row_update(W, fl, ad, bd, ts)
    Qh = O.dequantize(c, s, fo, ts)
    a_or, x_or = O.row_update(Wr, Qh, b, fo)
    pre = np64(a1pre)[ri]
    ok = ~np.isnan(x_or)
    assert np.array_equal(np.isnan(pre), np.isnan(x_or))
    assert np.all(np.abs(pre[ok] - x_or[ok]) <= 1e-5 * x_or[ok])
    check_projected(np64(a1)[ri], a_or, x_or, fo, "a (row step from the final state)")
    # one column step from the final state, on the columns of sampled groups
    b1, b1pre, _ = dq.col_update(W, fl, ad, bd, ts)
    gi = _sample(cols // G, n_groups, key + 1)
    cj = np.concatenate([np.arange(g * G, (g + 1) * G) for g in gi])
    Wc = np64(W[:, cj])
    cc, sc = O.quantize(O.inner(Wc, a, b[cj]), fo, ts)
    b_or, xb_or = O.col_update(Wc, O.dequantize(cc, sc, fo, ts), a, fo)
    preb = np64(b1pre)[cj]
    okb = ~np.isnan(xb_or)
    assert np.array_equal(np.isnan(preb), np.isnan(xb_or))
    assert np.all(np.abs(preb[okb] - xb_or[okb]) <= 1e-5 * xb_or[okb])
    check_projected(np64(b1)[cj], b_or, xb_or, fo, "b (column step from the final state)")
    # the final MSE is the MSE of the stored codes and scales, decoded in fp64
    R = _decode_fp64(o["codes"], o["gscales"], fo, ts, ad, bd)
    mse = ((W.double() - R) ** 2).mean().item()
    del R
    T = o["mse_trace"].numel() - 1
    assert abs(np64(o["mse_trace"])[T] - mse) <= 1e-6 * mse


_INT4 = torch.tensor([0, 1, 2, 3, 4, 5, 6, 7, -8, -7, -6, -5, -4, -3, -2, -1], dtype=torch.float64)
_E2M1 = torch.tensor([0, .5, 1, 1.5, 2, 3, 4, 6, -0., -.5, -1, -1.5, -2, -3, -4, -6],
                     dtype=torch.float64)


def _code_values(codes, fo):
    """Code values [rows, cols] (float64) of stored codes, by table lookup
    (tables from the oracle's decoders)."""
    rows = codes.shape[0]
    if fo.code_bits == 4:
        tab = (_INT4 if fo.codes == "int4" else _E2M1).to(codes.device)
        idx = torch.stack([codes & 0xF, codes >> 4], dim=-1).view(rows, -1).long()
    elif fo.code_bits == 8:
        tab = torch.tensor(O.decode_codes(np.arange(256, dtype=np.uint8)[None, :], fo)[0],
                           dtype=torch.float64, device=codes.device)
        idx = codes.long()
    else:                                            # four 6-bit codes per 3 bytes
        tab = torch.tensor(O.decode_fp_element(np.arange(64), fo.codes), dtype=torch.float64,
                           device=codes.device)
        b3 = codes.view(rows, -1, 3).long()
        w = b3[..., 0] | (b3[..., 1] << 8) | (b3[..., 2] << 16)
        idx = torch.stack([(w >> (6 * k)) & 0x3F for k in range(4)], dim=-1).view(rows, -1)
    return tab[idx]


def _decode_fp64(codes, gscales, fo, ts, a, b):
    """a_i c_ij s_g ts b_j in float64 with torch (table lookups, exact casts)."""
    rows = codes.shape[0]
    c = _code_values(codes, fo)
    if fo.gscale == "bf16":
        sc = (gscales.view(torch.int16).to(torch.int32) << 16).view(torch.float32).double()
    elif fo.gscale == "e8m0":
        sc = torch.exp2(gscales.double() - 127)
    else:
        sc = gscales.view(torch.float8_e4m3fn).double()
    G = fo.group
    v = (c.view(rows, -1, G) * (sc * ts).unsqueeze(-1)).view(rows, -1)
    return v * a.double().unsqueeze(1) * b.double().unsqueeze(0)


def _solve_workload(wl, decoders=None):
    fl = dq.format_preset(wl.fmt, wl.group)
    fo = O.preset(wl.fmt, wl.group)
    mats = [(d, i) for d, i, _ in wl.matrices if decoders is None or d in decoders]
    Ws = [synth.weight(wl, d, i, device="cuda") for d, i in mats]
    outs = dq.solve_dual_scale_batched(Ws, fl, wl.T, half=True)
    torch.cuda.synchronize()
    return fl, fo, mats, Ws, outs


def _trajectory_against_oracle(W, o, fo, T):
    # the oracle's whole solve on one full-size matrix (its first T iterations
    # when the E2M1 oracle would take minutes for all of them)
    r = O.solve(np64(W), fo, T)
    tr = np64(o["mse_trace"])[:T + 1]
    assert np.max(np.abs(tr - r["mse_trace"]) / r["mse_trace"]) < 1e-4
    assert float(o["tensor_scale"].item()) == r["ts"]


@pytest.mark.parametrize("fmt", ["mxfp4", "mxint8", "mxfp8_e4m3", "mxfp8_e5m2", "mxfp6_e2m3",
                                 "mxfp6_e3m2"])
def test_full_size_70b_decoder_mx(fmt):
    wl = synth.WORKLOADS[f"llama31_70b_decoder_{fmt}_g32"]
    fl, fo, mats, Ws, outs = _solve_workload(wl)
    assert sum(W.numel() for W in Ws) == 855638016
    for k, (W, o) in enumerate(zip(Ws, outs)):
        _check_matrix(W, o, fo, fl, key=500 + k)
        # power-of-two row steps leave D_a Qhat unchanged: half == trace
        assert np.array_equal(np64(o["mse_half"]), np64(o["mse_trace"])[:wl.T])
    _trajectory_against_oracle(Ws[1], outs[1], fo, 5)              # k_proj 1024 x 8192
    assert dq.last_device_status() == 0


@pytest.mark.parametrize("fmt", ["mxfp4", "mxint8", "mxfp8_e4m3", "mxfp8_e5m2", "mxfp6_e2m3",
                                 "mxfp6_e3m2"])
def test_full_size_70b_activation_mx(fmt):
    wl = synth.WORKLOADS[f"llama31_70b_decoder_{fmt}_g32"]
    act = wl.act
    fa, foa = dq.format_preset(act["fmt"], act["group"]), O.preset(act["fmt"], act["group"])
    X = synth.activation(wl, device="cuda")
    assert X.shape == (32768, 8192)
    b = torch.tensor(O.project_outer(np.exp(np.linspace(-1, 1, act["K"])), O.preset(wl.fmt)),
                     dtype=torch.float32, device="cuda")
    codes, gs = dq.act_rescale_quant(X, b, fa)
    torch.cuda.synchronize()
    ti = _sample(X.shape[0], 64, 7)
    c, s = O.act_rescale_quant(np64(X[ti]), np64(b), foa)
    assert np.array_equal(codes[ti].cpu().numpy(), O.encode_codes(c, foa))
    assert np.array_equal(gs[ti].cpu().numpy(), O.encode_scales(s, foa))


@pytest.mark.parametrize("name", ["llama31_8b_int4_g64", "llama31_8b_nvfp4_g16"])
def test_full_size_8b_all_decoders(name):
    wl = synth.WORKLOADS[name]
    fl, fo, mats, Ws, outs = _solve_workload(wl)
    assert len(outs) == 224 and sum(W.numel() for W in Ws) == 6979321856
    picks = [0, 1, 4, 6, 7 * 17 + 2, 7 * 31 + 5]                  # decoders 0, 17, 31
    for k in picks:
        _check_matrix(Ws[k], outs[k], fo, fl, key=600 + k, n_rows=8, n_groups=3)
    _trajectory_against_oracle(Ws[1], outs[1], fo, wl.T if fo.codes == "int4" else 5)  # k_proj
    # activation path at full size with the solved b of decoder-0 q_proj
    act = wl.act
    fa, foa = dq.format_preset(act["fmt"], act["group"]), O.preset(act["fmt"], act["group"])
    X = synth.activation(wl, device="cuda")
    assert X.shape == (32768, 4096)
    b = outs[0]["b"]
    codes, gs = dq.act_rescale_quant(X, b, fa)
    torch.cuda.synchronize()
    ti = _sample(X.shape[0], 48, 8)
    c, s = O.act_rescale_quant(np64(X[ti]), np64(b), foa)
    assert np.array_equal(codes[ti].cpu().numpy(), O.encode_codes(c, foa))
    assert np.array_equal(gpu_scales_np(gs[ti]), O.encode_scales(s, foa))
    del Ws, outs
    torch.cuda.empty_cache()


@pytest.mark.parametrize("fmt,T", [("mxfp4", 2), ("int4_bf16", 1)])
def test_matrix_beyond_int32_elements(fmt, T):
    # 65536 x 32832 = 2,151,677,952 elements (> 2^31): every flat offset of
    # the last rows needs 64 bits; sampled rows include the last ones
    wl = synth.WORKLOADS["llama31_70b_decoder_mxfp4_g32"]
    rows, cols = 65536, 32832
    W = synth.weight(wl, 0, 4, device="cuda", rows=rows, cols=cols)
    assert W.numel() > 2 ** 31
    fl = dq.format_preset(fmt, 32)
    fo = O.preset(fmt, 32)
    o = dq.solve_dual_scale(W, fl, T)
    torch.cuda.synchronize()
    assert dq.last_device_status() == 0
    a, b = np64(o["a"]), np64(o["b"])
    ri = np.concatenate([_sample(rows, 6, 77), np.arange(rows - 4, rows)])
    c, s = O.quantize(O.inner(np64(W[ri]), a[ri], b), fo)
    assert np.array_equal(o["codes"][ri].cpu().numpy(), O.encode_codes(c, fo))
    assert np.array_equal(gpu_scales_np(o["gscales"][ri]), O.encode_scales(s, fo))
    # the activation path on a batch of the same size
    if fmt == "mxfp4":
        X = W.view(rows, cols)                     # any bf16 [tokens, K] input
        codes, gs = dq.act_rescale_quant(X, o["b"], fl)
        torch.cuda.synchronize()
        ca, sa = O.act_rescale_quant(np64(X[ri]), b, fo)
        assert np.array_equal(codes[ri].cpu().numpy(), O.encode_codes(ca, fo))
        assert np.array_equal(gs[ri].cpu().numpy(), O.encode_scales(sa, fo))
    del W, o
    torch.cuda.empty_cache()
