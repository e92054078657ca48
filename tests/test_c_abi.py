"""The library driven from C (tests/c/*.c compiled with gcc against
include/dq.h and libdq.so): the header is plain C99, the host-side calls run
without a GPU, and a solve run from C matches the oracle."""
import os
import shutil
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "dual_scale_solver_b200")
CUDA = "/usr/local/cuda"

pytestmark = pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not available")


@pytest.fixture(scope="module", autouse=True)
def built():
    from dual_scale_solver_b200 import build
    build.build()


def _compile(src, exe, cuda=False):
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c", src), "-o", str(exe), "-L", PKG, "-ldq",
           f"-Wl,-rpath,{PKG}"]
    if cuda:
        cmd[1:1] = ["-I", f"{CUDA}/include"]
        cmd += ["-L", f"{CUDA}/lib64", "-lcudart", f"-Wl,-rpath,{CUDA}/lib64"]
    else:
        cmd.insert(2, "-pedantic")
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_host_calls_from_c(tmp_path):
    exe = tmp_path / "host_calls"
    _compile("host_calls.c", exe)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.startswith("ok ")


@pytest.mark.gpu
@pytest.mark.parametrize("name,G", [("mxfp4", 32), ("int4_bf16", 64)])
def test_solve_from_c_matches_oracle(tmp_path, name, G):
    import torch

    import oracle as O
    import synth
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    exe = tmp_path / "solve_file"
    _compile("solve_file.c", exe, cuda=True)
    wl = synth.WORKLOADS["llama31_70b_decoder_mxfp4_g32"]
    W = synth.weight(wl, 0, 1, rows=192, cols=768)             # bf16, a k_proj-like slice
    rows, cols, T = W.shape[0], W.shape[1], 4
    W.view(torch.int16).numpy().tofile(tmp_path / "w.bin")
    r = subprocess.run([str(exe), str(tmp_path / "w.bin"), str(rows), str(cols), str(T), name,
                        str(G), str(tmp_path / "out.bin")], capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    raw = (tmp_path / "out.bin").read_bytes()
    off = 0

    def take(dtype, n):
        nonlocal off
        a = np.frombuffer(raw, dtype=dtype, count=n, offset=off)
        off += a.nbytes
        return a

    assert take(np.int32, 1)[0] == 0
    ts = float(take(np.float32, 1)[0])
    a = take(np.float32, rows).astype(np.float64)
    b = take(np.float32, cols).astype(np.float64)
    mse = take(np.float64, T + 1)
    fo = O.preset(name, G)
    codes = take(np.uint8, rows * cols // 2).reshape(rows, cols // 2)
    gs = take(np.uint16 if fo.gscale == "bf16" else np.uint8, rows * cols // G)
    assert off == len(raw)
    W64 = W.double().numpy()
    ref = O.solve(W64, fo, T)
    assert np.max(np.abs(mse - ref["mse_trace"]) / ref["mse_trace"]) < 1e-4
    # the codes and group scales are Q at the state the C call returned
    c, s = O.quantize(O.inner(W64, a, b), fo, ts)
    assert np.array_equal(codes, O.encode_codes(c, fo))
    assert np.array_equal(gs.reshape(rows, cols // G), O.encode_scales(s, fo))
