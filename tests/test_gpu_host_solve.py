"""The host-streamed batched solve (inputs and outputs in page-locked host
memory, transfers overlapped with the solves) gives the same bits as the
device batched solve, on the host and in its device outputs, call after
call with reused buffers."""
import pytest
import torch

import synth
from _helpers import lib_format

pytestmark = pytest.mark.gpu

dq = pytest.importorskip("dual_scale_solver_b200")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from dual_scale_solver_b200 import build
    build.build()


KEYS = ("codes", "gscales", "a", "b", "tensor_scale", "mse_trace", "mse_half")


def _same(o, r):
    for k in KEYS:
        if r.get(k) is None:
            continue
        x, y = o[k].cpu(), r[k].cpu()
        assert x.dtype == y.dtype and torch.equal(x.view(torch.uint8), y.view(torch.uint8)), k


@pytest.mark.parametrize("name", ["mxfp4", "int4_bf16", "nvfp4"])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("grouping", ["all", "one"])
def test_host_solve_equals_device_batched(name, dtype, grouping):
    # "all": workspace for every shape (the matrices go as one group);
    # "one": workspace for the largest single matrix (one matrix per group)
    G = {"mxfp4": 32, "int4_bf16": 64, "nvfp4": 16}[name]
    fmt = lib_format(name, G)
    shapes = [(300, 40 * G), (64, 8 * G), (1, G), (517, 24 * G)]
    g = torch.Generator().manual_seed(3)
    Ws = [(torch.randn(r, c, generator=g) * 0.02).to(dtype) for r, c in shapes]
    hW = [W.pin_memory() for W in Ws]
    T = 4
    ref = dq.solve_dual_scale_batched([W.cuda() for W in Ws], fmt, T, half=True)
    ws = None
    if grouping == "one":
        ws = torch.empty(max(dq.workspace_size([s], fmt) for s in shapes), dtype=torch.uint8,
                         device="cuda")
    outs, dev_outs = dq.solve_dual_scale_batched_host(hW, fmt, T, half=True, ws=ws)
    torch.cuda.synchronize()
    assert dq.last_device_status() == 0
    for o, d, r in zip(outs, dev_outs, ref):
        assert not o["codes"].is_cuda and o["codes"].is_pinned()
        _same(o, r)
        _same(d, r)


def test_host_solve_repeated_calls_reuse_buffers():
    wl = synth.WORKLOADS["llama31_70b_decoder_mxfp4_g32"]
    fmt = dq.format_preset("mxfp4")
    Ws = [synth.weight(wl, 0, i, rows=256 * (i + 1), cols=1024) for i in range(3)]
    hW = [W.pin_memory() for W in Ws]
    ref = dq.solve_dual_scale_batched([W.cuda() for W in Ws], fmt, 6)
    outs = dev_outs = None
    for _ in range(3):                       # back to back, the same buffers
        outs, dev_outs = dq.solve_dual_scale_batched_host(hW, fmt, 6, outs=outs, dev_outs=dev_outs)
    torch.cuda.synchronize()
    for o, r in zip(outs, ref):
        _same(o, r)
    # inputs changed between calls: the second call sees its own inputs
    hW2 = [(W.float() * 2).to(W.dtype).pin_memory() for W in Ws]
    ref2 = dq.solve_dual_scale_batched([W.cuda() for W in hW2], fmt, 6)
    outs, dev_outs = dq.solve_dual_scale_batched_host(hW, fmt, 6, outs=outs, dev_outs=dev_outs)
    outs2, _ = dq.solve_dual_scale_batched_host(hW2, fmt, 6)
    torch.cuda.synchronize()
    for o, r in zip(outs, ref):
        _same(o, r)
    for o, r in zip(outs2, ref2):
        _same(o, r)


def test_host_solve_many_small_matrices_in_groups():
    # 40 small matrices (about 3 MB of inputs): fewer groups than matrices
    fmt = dq.format_preset("mxint4")
    g = torch.Generator().manual_seed(5)
    Ws = [(torch.randn(96 + 32 * (i % 5), 576, generator=g) * 0.02).to(torch.bfloat16)
          for i in range(40)]
    ref = dq.solve_dual_scale_batched([W.cuda() for W in Ws], fmt, 5)
    outs, _ = dq.solve_dual_scale_batched_host([W.pin_memory() for W in Ws], fmt, 5)
    torch.cuda.synchronize()
    for o, r in zip(outs, ref):
        _same(o, r)


def test_host_solve_workspace_too_small():
    fmt = dq.format_preset("mxfp4")
    W = torch.zeros(256, 1024, dtype=torch.bfloat16).pin_memory()
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(dq.DqError) as e:
        dq.solve_dual_scale_batched_host([W], fmt, 3, ws=ws)
    assert e.value.status == -7


def test_host_solve_empty_and_zero_matrices():
    # a matrix with no rows and an all-zero matrix among ordinary ones
    fmt = dq.format_preset("mxfp4")
    g = torch.Generator().manual_seed(9)
    Ws = [torch.zeros(0, 64, dtype=torch.bfloat16), torch.zeros(40, 96, dtype=torch.bfloat16),
          (torch.randn(64, 128, generator=g) * 0.02).to(torch.bfloat16)]
    ref = dq.solve_dual_scale_batched([W.cuda() for W in Ws], fmt, 3)
    outs, _ = dq.solve_dual_scale_batched_host([W.pin_memory() for W in Ws], fmt, 3)
    torch.cuda.synchronize()
    assert dq.last_device_status() == 0
    for o, r in zip(outs, ref):
        _same(o, r)
    assert torch.all(outs[1]["codes"] == 0) and torch.all(outs[1]["mse_trace"] == 0)


def test_host_solve_of_a_tall_batch_equals_device_batched():
    # A batch of many short matrices (170 x 15 column-pass tiles at the
    # default geometry) takes taller tiles; the host-streamed solve solves it
    # in groups of about 50 matrices, each of which alone would not, and
    # still gives the device batched solve's bits.
    fmt = lib_format("mxfp4", 32)
    g = torch.Generator().manual_seed(8)
    Ws = [(torch.randn(576, 576, generator=g) * 0.02).to(torch.bfloat16) for _ in range(170)]
    T = 2
    ref = dq.solve_dual_scale_batched([W.cuda() for W in Ws], fmt, T, half=True)
    outs, dev_outs = dq.solve_dual_scale_batched_host([W.pin_memory() for W in Ws], fmt, T,
                                                      half=True)
    torch.cuda.synchronize()
    assert dq.last_device_status() == 0
    for o, r in zip(outs, ref):
        _same(o, r)
