"""Two-level absmax quantization on the GPU against the oracle, bit for bit:
codes, inner E8M0 scales, outer float32 scales and the float32
reconstruction (msModelSlim DualScale page, "算法原理")."""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from _helpers import np64

pytestmark = pytest.mark.gpu

dq = pytest.importorskip("dual_scale_solver_b200")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from dual_scale_solver_b200 import build
    build.build()


def _check(X, D):
    fo = O.preset("mxfp4")
    codes, isc, osc, qdq = dq.two_level_quant(X.cuda(), D)
    torch.cuda.synchronize()
    c, s, S, q = O.two_level_quant(np64(X), D, fo)
    assert np.array_equal(osc.cpu().numpy().astype(np.float64), S)
    assert np.array_equal(isc.cpu().numpy(), O.encode_scales(s, fo))
    assert np.array_equal(codes.cpu().numpy(), O.encode_codes(c, fo))
    assert np.array_equal(qdq.cpu().numpy().astype(np.float64), q)


@pytest.mark.parametrize("D", [256, 512, 1024])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("shape", [(300, 2240), (5, 512), (33, 96)])
def test_two_level_bit_exact(D, dtype, shape):
    rows, cols = shape
    x = synth.normal(synth.stream_key(80, rows, cols, D), rows * cols).view(rows, cols)
    x = x * torch.exp(synth.normal(synth.stream_key(81, rows), rows)).view(rows, 1)
    x[:, ::37] *= 30.0                              # outlier channels
    x[1, :min(cols, D)] = 0.0                       # an all-zero block
    _check(x.to(dtype), D)


def test_two_level_on_activations_with_outlier_channels():
    wl = synth.WORKLOADS["llama31_70b_decoder_mxfp4_g32"]
    X = synth.activation(wl, tokens=64)
    _check(X, 512)


def test_two_level_without_reconstruction_and_nonfinite_flag():
    x = synth.normal(synth.stream_key(82, 1), 4 * 1024).view(4, 1024).to(torch.bfloat16).cuda()
    c1, s1, S1, q1 = dq.two_level_quant(x, 512, qdq=False)
    c2, s2, S2, q2 = dq.two_level_quant(x, 512)
    torch.cuda.synchronize()
    assert q1 is None and torch.equal(c1, c2) and torch.equal(s1, s2) and torch.equal(S1, S2)
    assert dq.last_device_status() == 0
    x[2, 7] = float("nan")
    dq.two_level_quant(x, 512)
    assert dq.last_device_status() == -4
