"""The solve entry point that allocates nothing.

Some callers cannot allocate device memory: code running inside another
framework's memory pool or under a fixed memory budget, plug-ins that may not
call cudaMalloc.  dq_solve_dual_scale_noalloc serves them by keeping the
solver's per-tile partial sums and flag words in a 32 MiB buffer built into
the library.  These tests call it through the C ABI and check it against
dq_solve_dual_scale (caller-provided workspace), which runs the same launch
sequence: results must agree exactly.  Two calls in a row check that what the
buffer must start with (the tensor-scale amax word, the flag words of the
one-pass MX iteration) is cleared between calls.  This file is collected
last so that a failure here stops a run only after every other test ran.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

dq = pytest.importorskip("dual_scale_solver_b200")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from dual_scale_solver_b200 import build
    build.build()


def _matrix(rows, cols, key, scale, dtype=torch.bfloat16):
    w = synth.student_t4(synth.stream_key(97, key), rows * cols).view(rows, cols) * scale
    return w.to(dtype).cuda()


def _noalloc(W, fmt, T):
    rows, cols = W.shape
    dev = W.device
    out = dict(codes=torch.empty(rows, cols // 2, dtype=torch.uint8, device=dev),
               gscales=torch.empty(rows, cols // fmt.group, dtype=dq.gscale_dtype(fmt), device=dev),
               a=torch.empty(rows, dtype=torch.float32, device=dev),
               b=torch.empty(cols, dtype=torch.float32, device=dev),
               tensor_scale=torch.empty(1, dtype=torch.float32, device=dev),
               mse_trace=torch.empty(T + 1, dtype=torch.float64, device=dev),
               mse_half=torch.empty(T, dtype=torch.float64, device=dev))
    p = lambda t: t.data_ptr()
    dt = dq.DQ_DT_F32 if W.dtype == torch.float32 else dq.DQ_DT_BF16
    s = dq.lib().dq_solve_dual_scale_noalloc(
        p(W), dt, rows, cols, ctypes.byref(fmt), T, None, None, p(out["codes"]),
        p(out["gscales"]), p(out["a"]), p(out["b"]), p(out["tensor_scale"]),
        p(out["mse_trace"]), p(out["mse_half"]), torch.cuda.current_stream().cuda_stream)
    assert s == 0, dq.lib().dq_strerror(s)
    return out


def _same(got, ref):
    for k in ("codes", "gscales", "a", "b", "tensor_scale"):
        assert torch.equal(got[k], ref[k]), k
    for k in ("mse_trace", "mse_half"):
        g, r = got[k].cpu().numpy(), ref[k].cpu().numpy()
        assert np.allclose(g, r, rtol=1e-12, atol=0), (k, g, r)


@pytest.mark.parametrize("name,dtype", [("nvfp4", torch.bfloat16), ("mxfp4", torch.bfloat16),
                                        ("mxint4", torch.bfloat16), ("int4_bf16", torch.bfloat16),
                                        ("int4_bf16", torch.float32)])
def test_noalloc_solve_matches_workspace_solve_twice_in_a_row(name, dtype):
    dq.last_device_status()                   # clear flags left by earlier tests
    fmt = dq.format_preset(name)
    # The second matrix has a much smaller amax: a stale amax word would give
    # it the first matrix's tensor scale (NVFP4).  The first matrix's rows
    # scaled by 2^-112 take the MX one-pass iteration out of its exponent
    # range, so that call raises its flag words and redoes its steps
    # literally (the fallback inside this entry point, checked against the
    # workspace solve like the rest).
    W1 = _matrix(512, 1024, 1, 0.5, dtype)
    W1[::9] *= 2.0 ** -112
    cases = [(W1, 3), (_matrix(300, 2048, 2, 0.002, dtype), 4)]
    mx = fmt.group_scale == dq.DQ_SCALE_E8M0 and fmt.outer_scale == dq.DQ_SCALE_E8M0
    for k, (W, T) in enumerate(cases):
        torch.cuda.synchronize()
        dq.kernel_time(dq.KIND_FUSED)
        dq.kernel_time(dq.KIND_ROW)
        dq.kernel_timing(True, kinds=[dq.KIND_FUSED, dq.KIND_ROW])
        got = _noalloc(W, fmt, T)
        torch.cuda.synchronize()
        dq.kernel_timing(False)
        n_fused = dq.kernel_time(dq.KIND_FUSED)[1]
        n_row = dq.kernel_time(dq.KIND_ROW)[1]
        ref = dq.solve_dual_scale(W, fmt, T)
        torch.cuda.synchronize()
        _same(got, ref)
        # the MX formats take the one-pass kernel every iteration (the
        # literal row pass is launched too, behind its flag, and returns at
        # once unless the flag is up); the others take the literal row pass
        assert (n_fused, n_row) == ((T, T) if mx else (0, T)), (n_fused, n_row)
    status = dq.last_device_status()
    assert status in (0, dq.DQ_ERR_NONFINITE, dq.DQ_ERR_RANGE)   # 2^-112 rows


def test_noalloc_refuses_a_matrix_beyond_its_scratch():
    fmt = dq.format_preset("mxfp4")
    fake = ctypes.c_void_p(1 << 20)           # never dereferenced: refused before any launch
    s = dq.lib().dq_solve_dual_scale_noalloc(fake, dq.DQ_DT_BF16, 65536, 28672,
                                             ctypes.byref(fmt), 1, None, None, fake, fake, fake,
                                             fake, fake, None, None, None)
    assert s == -10
    assert "32 MiB" in dq.lib().dq_strerror(s).decode()
