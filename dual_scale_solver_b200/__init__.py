"""dual_scale_solver_b200 — Python binding of the ``dq`` C ABI (``include/dq.h``).

Argument marshalling only: every step of the solver runs in the CUDA kernels
of ``libdq.so``.  Torch tensors supply device memory and the current CUDA
stream; outputs that the caller does not pass are allocated with torch.
There is no CPU fallback: without the built library every call raises.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import c_char_p, c_double, c_float, c_int32, c_int64, c_size_t, c_void_p, POINTER

import torch

__all__ = [
    "DqError", "dq_format", "dq_matrix", "lib", "library_path", "version", "format_preset",
    "workspace_size", "quantize", "dequantize", "solve_dual_scale", "solve_dual_scale_batched",
    "row_update", "col_update", "act_rescale_quant", "last_device_status", "EXPORTS",
    "kernel_timing", "kernel_time", "launch_count", "solve_dual_scale_noalloc", "code_bytes",
    "two_level_quant", "w4a4_gemm", "scale_tiles", "solve_dual_scale_batched_host", "copy_streams",
    "SolveGraph", "solve_dual_scale_batched_graph", "col_row_block", "col_partials", "col_finalize",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libdq.so")

DQ_CODES_INT4, DQ_CODES_E2M1, DQ_CODES_INT8, DQ_CODES_E4M3 = 0, 1, 2, 3
DQ_CODES_E5M2, DQ_CODES_E2M3, DQ_CODES_E3M2 = 4, 5, 6
DQ_SCALE_BF16, DQ_SCALE_E8M0, DQ_SCALE_E4M3 = 0, 1, 2
DQ_DT_F32, DQ_DT_BF16 = 0, 1
DQ_OK, DQ_ERR_ARG, DQ_ERR_NONFINITE, DQ_ERR_RANGE = 0, -1, -4, -5

EXPORTS = ("dq_version", "dq_strerror", "dq_format_preset", "dq_workspace_size", "dq_quantize",
           "dq_dequantize", "dq_solve_dual_scale", "dq_solve_dual_scale_batched",
           "dq_row_update", "dq_col_update", "dq_act_rescale_quant", "dq_last_device_status",
           "dq_kernel_timing", "dq_kernel_time", "dq_launch_count",
           "dq_solve_dual_scale_noalloc", "dq_code_bytes", "dq_two_level_quant", "dq_w4a4_gemm",
           "dq_scale_tiles", "dq_solve_dual_scale_batched_host", "dq_test_stall_next_gemm",
           "dq_graph_solve_batched", "dq_graph_launch", "dq_graph_launches", "dq_graph_destroy",
           "dq_col_row_block", "dq_col_partials", "dq_col_finalize")


class DqError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {_strerror(status)} (status {status})")


class dq_format(ctypes.Structure):
    _fields_ = [("codes", c_int32), ("group", c_int32), ("group_scale", c_int32),
                ("outer_scale", c_int32), ("tensor_scale_auto", c_int32)]

    def __repr__(self):
        return (f"dq_format(codes={self.codes}, group={self.group}, group_scale={self.group_scale}, "
                f"outer_scale={self.outer_scale}, tensor_scale_auto={self.tensor_scale_auto})")


class dq_matrix(ctypes.Structure):
    _fields_ = [("W", c_void_p), ("rows", c_int64), ("cols", c_int64), ("a0", c_void_p),
                ("b0", c_void_p), ("codes", c_void_p), ("gscales", c_void_p), ("a", c_void_p),
                ("b", c_void_p), ("tensor_scale", c_void_p), ("mse_trace", c_void_p),
                ("mse_half", c_void_p)]


_lib = None


def library_path() -> str:
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    """The loaded ``libdq.so``; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"libdq.so not built at {_LIB_PATH}; run "
                          "`python -m dual_scale_solver_b200.build` (no CPU fallback exists)")
    L = ctypes.CDLL(_LIB_PATH)
    P = POINTER
    sig = {
        "dq_version": (c_char_p, []),
        "dq_strerror": (c_char_p, [c_int32]),
        "dq_format_preset": (c_int32, [c_char_p, c_int32, P(dq_format)]),
        "dq_workspace_size": (c_int32, [c_int32, P(c_int64), P(c_int64), P(dq_format), P(c_size_t)]),
        "dq_quantize": (c_int32, [c_void_p, c_int32, c_int64, c_int64, P(dq_format), c_void_p,
                                  c_void_p, c_float, c_void_p, c_void_p, c_void_p]),
        "dq_dequantize": (c_int32, [c_void_p, c_void_p, c_int64, c_int64, P(dq_format), c_float,
                                    c_void_p, c_void_p, c_void_p, c_void_p]),
        "dq_solve_dual_scale": (c_int32, [c_void_p, c_int32, c_int64, c_int64, P(dq_format),
                                          c_int32, c_void_p, c_void_p, c_void_p, c_void_p,
                                          c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                          c_void_p, c_size_t, c_void_p]),
        "dq_solve_dual_scale_batched": (c_int32, [c_int32, P(dq_matrix), c_int32, P(dq_format),
                                                  c_int32, c_void_p, c_size_t, c_void_p]),
        "dq_row_update": (c_int32, [c_void_p, c_int32, c_int64, c_int64, P(dq_format), c_float,
                                    c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                    c_size_t, c_void_p]),
        "dq_col_update": (c_int32, [c_void_p, c_int32, c_int64, c_int64, P(dq_format), c_float,
                                    c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                    c_size_t, c_void_p]),
        "dq_col_row_block": (c_int64, [c_int64, c_int64, c_int32]),
        "dq_col_partials": (c_int32, [c_void_p, c_int32, c_int64, c_int64, P(dq_format), c_float,
                                      c_void_p, c_void_p, c_int64, c_void_p, c_void_p, c_void_p,
                                      c_size_t, c_void_p]),
        "dq_col_finalize": (c_int32, [c_void_p, c_int64, c_int64, P(dq_format), c_void_p,
                                      c_void_p, c_void_p]),
        "dq_act_rescale_quant": (c_int32, [c_void_p, c_int64, c_int64, c_void_p, P(dq_format),
                                           c_void_p, c_void_p, c_void_p]),
        "dq_last_device_status": (c_int32, [c_void_p]),
        "dq_kernel_timing": (c_int32, [c_int32]),
        "dq_kernel_time": (c_int32, [c_int32, P(c_double), P(c_int64)]),
        "dq_launch_count": (c_int64, []),
        "dq_code_bytes": (c_int64, [P(dq_format), c_int64, c_int64]),
        "dq_w4a4_gemm": (c_int32, [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                   c_int64, c_int64, c_int64, P(dq_format), c_void_p, c_void_p]),
        "dq_scale_tiles": (c_int32, [c_void_p, c_int64, c_int64, c_int32, c_void_p, c_void_p]),
        "dq_test_stall_next_gemm": (c_int32, []),
        "dq_graph_solve_batched": (c_int32, [c_int32, P(dq_matrix), c_int32, P(dq_format), c_int32,
                                             c_void_p, c_size_t, P(c_void_p)]),
        "dq_graph_launch": (c_int32, [c_void_p, c_void_p]),
        "dq_graph_launches": (c_int64, [c_void_p]),
        "dq_graph_destroy": (c_int32, [c_void_p]),
        "dq_solve_dual_scale_batched_host": (c_int32, [c_int32, P(dq_matrix), P(dq_matrix), c_int32,
                                                       P(dq_format), c_int32, c_void_p, c_size_t,
                                                       c_void_p, c_void_p, c_void_p]),
        "dq_two_level_quant": (c_int32, [c_void_p, c_int32, c_int64, c_int64, c_int32,
                                         P(dq_format), c_void_p, c_void_p, c_void_p, c_void_p,
                                         c_void_p]),
        "dq_solve_dual_scale_noalloc": (c_int32, [c_void_p, c_int32, c_int64, c_int64,
                                                  P(dq_format), c_int32, c_void_p, c_void_p,
                                                  c_void_p, c_void_p, c_void_p, c_void_p,
                                                  c_void_p, c_void_p, c_void_p, c_void_p]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    _lib = L
    return L


def _strerror(s: int) -> str:
    return lib().dq_strerror(s).decode()


def _check(s: int, where: str):
    if s != DQ_OK:
        raise DqError(s, where)


def version() -> str:
    return lib().dq_version().decode()


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return DQ_DT_BF16
    if t.dtype == torch.float32:
        return DQ_DT_F32
    raise TypeError(f"unsupported input dtype {t.dtype} (bfloat16 or float32)")


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("tensors must be CUDA tensors")


def format_preset(name: str, group: int = 0) -> dq_format:
    f = dq_format()
    _check(lib().dq_format_preset(name.encode(), group, ctypes.byref(f)), "dq_format_preset")
    return f


def gscale_dtype(fmt: dq_format) -> torch.dtype:
    return torch.int16 if fmt.group_scale == DQ_SCALE_BF16 else torch.uint8


def workspace_size(shapes, fmt: dq_format) -> int:
    n = len(shapes)
    rows = (c_int64 * max(n, 1))(*[int(r) for r, _ in shapes])
    cols = (c_int64 * max(n, 1))(*[int(c) for _, c in shapes])
    out = c_size_t(0)
    _check(lib().dq_workspace_size(n, rows, cols, ctypes.byref(fmt), ctypes.byref(out)),
           "dq_workspace_size")
    return out.value


def workspace(shapes, fmt: dq_format, device=None) -> torch.Tensor:
    return torch.empty(workspace_size(shapes, fmt), dtype=torch.uint8,
                       device=device or torch.device("cuda"))


def code_bytes(fmt, rows, cols) -> int:
    """Bytes of the codes of a rows x cols matrix (rows of cols*bits/8 bytes)."""
    n = lib().dq_code_bytes(ctypes.byref(fmt), rows, cols)
    if n < 0:
        raise DqError(-3 if cols % max(fmt.group, 1) == 0 else -2, "dq_code_bytes")
    return n


def _outputs(rows, cols, fmt, device, codes=None, gscales=None):
    if codes is None:
        per_row = code_bytes(fmt, 1, cols) if rows > 0 else 0
        codes = torch.empty(rows, per_row, dtype=torch.uint8, device=device)
    if gscales is None:
        gscales = torch.empty(rows, cols // fmt.group, dtype=gscale_dtype(fmt), device=device)
    return codes, gscales


def quantize(X, fmt, a=None, b=None, tensor_scale: float = 1.0, codes=None, gscales=None,
             stream=None):
    """Q(X / (a b^T)) -> (codes [rows, cols*bits/8] uint8, group scales [rows, cols/G])."""
    _need_cuda(X, a, b)
    rows, cols = X.shape
    codes, gscales = _outputs(rows, cols, fmt, X.device, codes, gscales)
    _check(lib().dq_quantize(_ptr(X), _dtype_code(X), rows, cols, ctypes.byref(fmt), _ptr(a),
                             _ptr(b), float(tensor_scale), _ptr(codes), _ptr(gscales),
                             _stream(stream)), "dq_quantize")
    return codes, gscales


def dequantize(codes, gscales, rows, cols, fmt, tensor_scale=1.0, a=None, b=None, out=None,
               stream=None):
    """a_i * c_ij * s_g * ts * b_j as float32 [rows, cols]."""
    if out is None:
        out = torch.empty(rows, cols, dtype=torch.float32, device=codes.device)
    _check(lib().dq_dequantize(_ptr(codes), _ptr(gscales), rows, cols, ctypes.byref(fmt),
                               float(tensor_scale), _ptr(a), _ptr(b), _ptr(out),
                               _stream(stream)), "dq_dequantize")
    return out


def solve_dual_scale(W, fmt, T, a0=None, b0=None, ws=None, half=True, stream=None):
    """Full DualQuant solve of one matrix.  Returns a dict of device tensors:
    codes, gscales, a, b, tensor_scale, mse_trace (T+1), mse_half (T)."""
    _need_cuda(W, a0, b0)
    rows, cols = W.shape
    dev = W.device
    codes, gscales = _outputs(rows, cols, fmt, dev)
    a = torch.empty(rows, dtype=torch.float32, device=dev)
    b = torch.empty(cols, dtype=torch.float32, device=dev)
    ts = torch.empty(1, dtype=torch.float32, device=dev)
    trace = torch.empty(T + 1, dtype=torch.float64, device=dev)
    mhalf = torch.empty(max(T, 1), dtype=torch.float64, device=dev) if half else None
    if ws is None:
        ws = workspace([(rows, cols)], fmt, dev)
    _check(lib().dq_solve_dual_scale(_ptr(W), _dtype_code(W), rows, cols, ctypes.byref(fmt), T,
                                     _ptr(a0), _ptr(b0), _ptr(codes), _ptr(gscales), _ptr(a),
                                     _ptr(b), _ptr(ts), _ptr(trace), _ptr(mhalf), _ptr(ws),
                                     ws.numel(), _stream(stream)), "dq_solve_dual_scale")
    return dict(codes=codes, gscales=gscales, a=a, b=b, tensor_scale=ts, mse_trace=trace,
                mse_half=mhalf[:T] if half else None)


NOALLOC_SCRATCH_BYTES = 32 << 20


def solve_dual_scale_noalloc(W, fmt, T, a0=None, b0=None, half=True, stream=None):
    """The solve of ``solve_dual_scale`` without a workspace: for callers that
    cannot allocate device scratch (the library keeps a 32 MiB buffer per
    device for it; concurrent calls on one device race).  Outputs are
    allocated here with torch; pass them to the C call yourself to avoid that."""
    _need_cuda(W, a0, b0)
    rows, cols = W.shape
    dev = W.device
    codes, gscales = _outputs(rows, cols, fmt, dev)
    a = torch.empty(rows, dtype=torch.float32, device=dev)
    b = torch.empty(cols, dtype=torch.float32, device=dev)
    ts = torch.empty(1, dtype=torch.float32, device=dev)
    trace = torch.empty(T + 1, dtype=torch.float64, device=dev)
    mhalf = torch.empty(max(T, 1), dtype=torch.float64, device=dev) if half else None
    _check(lib().dq_solve_dual_scale_noalloc(_ptr(W), _dtype_code(W), rows, cols,
                                             ctypes.byref(fmt), T, _ptr(a0), _ptr(b0),
                                             _ptr(codes), _ptr(gscales), _ptr(a), _ptr(b),
                                             _ptr(ts), _ptr(trace), _ptr(mhalf), _stream(stream)),
           "dq_solve_dual_scale_noalloc")
    return dict(codes=codes, gscales=gscales, a=a, b=b, tensor_scale=ts, mse_trace=trace,
                mse_half=mhalf[:T] if half else None)


def _batch(Ws, fmt, T, ws, outs, half):
    """The dq_matrix array of a batch (outputs and workspace allocated when
    not given): (mats, dtype code, outs, ws)."""
    n = len(Ws)
    dt = _dtype_code(Ws[0])
    dev = Ws[0].device
    if outs is None:
        outs = []
        for W in Ws:
            rows, cols = W.shape
            codes, gscales = _outputs(rows, cols, fmt, dev)
            outs.append(dict(
                codes=codes, gscales=gscales,
                a=torch.empty(rows, dtype=torch.float32, device=dev),
                b=torch.empty(cols, dtype=torch.float32, device=dev),
                tensor_scale=torch.empty(1, dtype=torch.float32, device=dev),
                mse_trace=torch.empty(T + 1, dtype=torch.float64, device=dev),
                mse_half=torch.empty(max(T, 1), dtype=torch.float64, device=dev) if half else None))
    if ws is None:
        ws = workspace([tuple(W.shape) for W in Ws], fmt, dev)
    mats = (dq_matrix * n)()
    for i, (W, o) in enumerate(zip(Ws, outs)):
        if _dtype_code(W) != dt:
            raise TypeError("all matrices of a batch share one dtype")
        m = mats[i]
        m.W, m.rows, m.cols = _ptr(W), W.shape[0], W.shape[1]
        m.a0 = m.b0 = None
        m.codes, m.gscales = _ptr(o["codes"]), _ptr(o["gscales"])
        m.a, m.b, m.tensor_scale = _ptr(o["a"]), _ptr(o["b"]), _ptr(o["tensor_scale"])
        m.mse_trace, m.mse_half = _ptr(o["mse_trace"]), _ptr(o.get("mse_half"))
    return mats, dt, outs, ws


def solve_dual_scale_batched(Ws, fmt, T, ws=None, outs=None, half=False, stream=None):
    """Solve a list of independent matrices (same dtype) in one launch sequence.
    ``outs`` (optional) is a list of dicts as returned by this function, reused."""
    if len(Ws) == 0:
        return []
    mats, dt, outs, ws = _batch(Ws, fmt, T, ws, outs, half)
    _check(lib().dq_solve_dual_scale_batched(len(Ws), mats, dt, ctypes.byref(fmt), T, _ptr(ws),
                                             ws.numel(), _stream(stream)),
           "dq_solve_dual_scale_batched")
    return outs


class SolveGraph:
    """A batched solve captured as a CUDA graph (dq_graph_solve_batched).
    Holds the weights, outputs and workspace it was made with: ``launch``
    solves the weights as they are at that time into ``outs``."""

    def __init__(self, handle, Ws, outs, ws):
        self._h, self.Ws, self.outs, self.ws = handle, Ws, outs, ws

    @property
    def launches(self):
        return int(lib().dq_graph_launches(self._h)) if self._h else 0

    def launch(self, stream=None):
        if not self._h:
            raise DqError(-1, "dq_graph_launch (graph closed)")
        _check(lib().dq_graph_launch(self._h, _stream(stream)), "dq_graph_launch")
        return self.outs

    def close(self):
        """Free the graph (a replay in flight completes first)."""
        if self._h:
            lib().dq_graph_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def solve_dual_scale_batched_graph(Ws, fmt, T, ws=None, outs=None, half=False):
    """Capture the batched solve of ``Ws`` as a graph (nothing runs yet);
    ``SolveGraph.launch`` replays it."""
    if len(Ws) == 0:
        raise ValueError("a graph needs at least one matrix")
    mats, dt, outs, ws = _batch(Ws, fmt, T, ws, outs, half)
    h = c_void_p()
    _check(lib().dq_graph_solve_batched(len(Ws), mats, dt, ctypes.byref(fmt), T, _ptr(ws),
                                        ws.numel(), ctypes.byref(h)),
           "dq_graph_solve_batched")
    return SolveGraph(h, list(Ws), outs, ws)


_COPY_STREAMS = {}


def copy_streams(device):
    """One host-to-device and one device-to-host stream per device (kept)."""
    idx = torch.device(device).index
    idx = torch.cuda.current_device() if idx is None else idx
    if idx not in _COPY_STREAMS:
        _COPY_STREAMS[idx] = (torch.cuda.Stream(idx), torch.cuda.Stream(idx))
    return _COPY_STREAMS[idx]


def _solve_outputs(rows, cols, fmt, T, half, device, pin=False):
    codes, gscales = _outputs(rows, cols, fmt, device)
    kw = dict(device=device, pin_memory=pin)
    if pin:
        codes, gscales = codes.pin_memory(), gscales.pin_memory()
    return dict(codes=codes, gscales=gscales,
                a=torch.empty(rows, dtype=torch.float32, **kw),
                b=torch.empty(cols, dtype=torch.float32, **kw),
                tensor_scale=torch.empty(1, dtype=torch.float32, **kw),
                mse_trace=torch.empty(T + 1, dtype=torch.float64, **kw),
                mse_half=torch.empty(max(T, 1), dtype=torch.float64, **kw) if half else None)


def _fill_matrix(m, W, o):
    m.W, m.rows, m.cols = _ptr(W), W.shape[0], W.shape[1]
    m.a0 = m.b0 = None
    m.codes, m.gscales = _ptr(o["codes"]), _ptr(o["gscales"])
    m.a, m.b, m.tensor_scale = _ptr(o["a"]), _ptr(o["b"]), _ptr(o["tensor_scale"])
    m.mse_trace, m.mse_half = _ptr(o["mse_trace"]), _ptr(o.get("mse_half"))


def solve_dual_scale_batched_host(Ws, fmt, T, outs=None, dev_outs=None, staging=None, ws=None,
                                  half=False, device=None, stream=None, wait_out=True):
    """Solve matrices held in host memory (CPU tensors of one dtype; pin them
    for the copies to overlap): matrix i+1 is copied in while matrix i is
    solved and matrix i-1's results are copied back (dq_solve_dual_scale_batched_host).
    Consecutive matrices are solved in groups (one batched solve each), as
    far as `ws` allows (default: room for all of them).
    Returns (outs, dev_outs): per matrix a dict of page-locked CPU tensors and
    one of the device tensors holding the same results.  `stream` (default:
    the current stream) runs the solves and, on return, also waits for the
    copies back, so work ordered after it sees the host results (with
    wait_out=False it does not: the caller orders its reads after
    `copy_streams(device)[1]`, the copy-back stream).  `outs`,
    `dev_outs`, `staging` (device copies of W) and `ws` may be passed back in
    to reuse them."""
    n = len(Ws)
    if n == 0:
        return [], []
    dev = torch.device(device or "cuda")
    dt = _dtype_code(Ws[0])
    shapes = [tuple(W.shape) for W in Ws]
    if outs is None:
        outs = [_solve_outputs(r, c, fmt, T, half, "cpu", pin=True) for r, c in shapes]
    if dev_outs is None:
        dev_outs = [_solve_outputs(r, c, fmt, T, half, dev) for r, c in shapes]
    if staging is None:
        staging = [torch.empty(W.shape, dtype=W.dtype, device=dev) for W in Ws]
    if ws is None:                # room for every grouping the library may choose
        ws = workspace(shapes, fmt, dev)
    host, devm = (dq_matrix * n)(), (dq_matrix * n)()
    for i in range(n):
        if _dtype_code(Ws[i]) != dt or Ws[i].is_cuda:
            raise TypeError("host matrices: CPU tensors of one dtype")
        _fill_matrix(host[i], Ws[i], outs[i])
        _fill_matrix(devm[i], staging[i], dev_outs[i])
    compute = stream if stream is not None else torch.cuda.current_stream(dev)
    h2d, d2h = copy_streams(dev)
    _check(lib().dq_solve_dual_scale_batched_host(n, host, devm, dt, ctypes.byref(fmt), T, _ptr(ws),
                                                  ws.numel(), compute.cuda_stream, h2d.cuda_stream,
                                                  d2h.cuda_stream),
           "dq_solve_dual_scale_batched_host")
    if wait_out:
        compute.wait_stream(d2h)
    return outs, dev_outs


def _step(fn, name, W, fmt, tensor_scale, a_in, b_in, out_len, ws, stream):
    _need_cuda(W, a_in, b_in)
    rows, cols = W.shape
    dev = W.device
    out = torch.empty(out_len, dtype=torch.float32, device=dev)
    pre = torch.empty(out_len, dtype=torch.float32, device=dev)
    mse = torch.empty(1, dtype=torch.float64, device=dev)
    if ws is None:
        ws = workspace([(rows, cols)], fmt, dev)
    _check(fn(_ptr(W), _dtype_code(W), rows, cols, ctypes.byref(fmt), float(tensor_scale),
              _ptr(a_in), _ptr(b_in), _ptr(out), _ptr(pre), _ptr(mse), _ptr(ws), ws.numel(),
              _stream(stream)), name)
    return out, pre, mse


def row_update(W, fmt, a_in, b_in, tensor_scale=1.0, ws=None, stream=None):
    """One row half-step: returns (a_out, a_pre, mse_of_input_state)."""
    return _step(lib().dq_row_update, "dq_row_update", W, fmt, tensor_scale, a_in, b_in,
                 W.shape[0], ws, stream)


def col_update(W, fmt, a_in, b_in, tensor_scale=1.0, ws=None, stream=None):
    """One column half-step: returns (b_out, b_pre, mse_of_input_state)."""
    return _step(lib().dq_col_update, "dq_col_update", W, fmt, tensor_scale, a_in, b_in,
                 W.shape[1], ws, stream)


def col_row_block(rows, cols, dtype=torch.bfloat16) -> int:
    """Rows per row block of the column statistics of a rows x cols matrix."""
    v = lib().dq_col_row_block(rows, cols, DQ_DT_F32 if dtype == torch.float32 else DQ_DT_BF16)
    if v < 0:
        raise DqError(DQ_ERR_ARG, "dq_col_row_block")
    return int(v)


def col_partials(W, fmt, a, b, row_block, tensor_scale=1.0, out=None, ws=None, stream=None):
    """Column partial sums of a row shard W (its rows' a, the matrix's b) per
    block of `row_block` rows: returns (partials [ceil(rows/row_block), cols,
    2] float32, mse of the input state over the shard)."""
    _need_cuda(W, a, b)
    rows, cols = W.shape
    nrb = -(-rows // row_block)
    if out is None:
        out = torch.empty(nrb, cols, 2, dtype=torch.float32, device=W.device)
    mse = torch.empty(1, dtype=torch.float64, device=W.device)
    if ws is None:
        ws = workspace([(rows, cols)], fmt, W.device)
    _check(lib().dq_col_partials(_ptr(W), _dtype_code(W), rows, cols, ctypes.byref(fmt),
                                 float(tensor_scale), _ptr(a), _ptr(b), row_block, _ptr(out),
                                 _ptr(mse), _ptr(ws), ws.numel(), _stream(stream)),
           "dq_col_partials")
    return out, mse


def col_finalize(partials, fmt, b_out=None, stream=None):
    """b from column partial slabs [row_blocks, cols, 2] (fixed-order sums):
    returns (b, b_pre)."""
    _need_cuda(partials)
    nrb, cols = partials.shape[0], partials.shape[1]
    if b_out is None:
        b_out = torch.empty(cols, dtype=torch.float32, device=partials.device)
    pre = torch.empty(cols, dtype=torch.float32, device=partials.device)
    _check(lib().dq_col_finalize(_ptr(partials), nrb, cols, ctypes.byref(fmt), _ptr(b_out),
                                 _ptr(pre), _stream(stream)), "dq_col_finalize")
    return b_out, pre


def act_rescale_quant(X, b, fmt, codes=None, gscales=None, stream=None):
    """Q(X D_b): returns (codes [tokens, K*bits/8], group scales [tokens, K/G])."""
    _need_cuda(X, b)
    if X.dtype != torch.bfloat16:
        raise TypeError("activations are bfloat16")
    tokens, K = X.shape
    codes, gscales = _outputs(tokens, K, fmt, X.device, codes, gscales)
    _check(lib().dq_act_rescale_quant(_ptr(X), tokens, K, _ptr(b), ctypes.byref(fmt), _ptr(codes),
                                      _ptr(gscales), _stream(stream)), "dq_act_rescale_quant")
    return codes, gscales


def two_level_quant(X, dual_block=512, inner=None, qdq=True, stream=None):
    """Two-level absmax quantization: returns (codes [rows, cols/2], inner
    E8M0 scales [rows, cols/32], outer float32 scales [rows, ceil(cols/D)],
    reconstruction float32 [rows, cols] or None)."""
    _need_cuda(X)
    inner = format_preset("mxfp4") if inner is None else inner
    rows, cols = X.shape
    dev = X.device
    nb = -(-cols // dual_block) if cols else 0
    codes = torch.empty(rows, cols // 2, dtype=torch.uint8, device=dev)
    isc = torch.empty(rows, cols // 32, dtype=torch.uint8, device=dev)
    osc = torch.empty(rows, nb, dtype=torch.float32, device=dev)
    out = torch.empty(rows, cols, dtype=torch.float32, device=dev) if qdq else None
    _check(lib().dq_two_level_quant(_ptr(X), _dtype_code(X), rows, cols, int(dual_block),
                                    ctypes.byref(inner), _ptr(codes), _ptr(isc), _ptr(osc),
                                    _ptr(out), _stream(stream)), "dq_two_level_quant")
    return codes, isc, osc, out


def scale_tiles(scales, K=None, out=None, stream=None, group=32):
    """Row-major group scales [rows, K/group] (E8M0 for MXFP4, group 32; E4M3
    for NVFP4, group 16) -> the scale tiles dq_w4a4_gemm reads (rows * K /
    group bytes, uint8)."""
    _need_cuda(scales)
    rows = scales.shape[0]
    K = group * scales.shape[1] if K is None else K
    if out is None:
        out = torch.empty(rows * K // group, dtype=torch.uint8, device=scales.device)
    _check(lib().dq_scale_tiles(_ptr(scales), rows, K, group, _ptr(out), _stream(stream)),
           "dq_scale_tiles")
    return out


def w4a4_gemm(codes_x, scales_x, codes_w, scales_w, a, fmt=None, out=None, stream=None,
              tiled=False, tensor_scale=None):
    """out[M, N] = a_n * ts * sum_k Qx[m, k] Qw[n, k] (float32) from E2M1 codes
    and group scales of the activations (M rows) and the weights (N rows):
    MXFP4 (E8M0 scales per 32, the default) or NVFP4 (E4M3 scales per 16; ts
    = the weights' tensor scale, a one-element device tensor as the solve
    returns it, None for 1).  The scales are row-major [rows, K/G]
    (tiled=False: rewritten into scale tiles first, one extra launch each) or
    already scale tiles (tiled=True)."""
    _need_cuda(codes_x, scales_x, codes_w, scales_w, a)
    fmt = format_preset("mxfp4") if fmt is None else fmt
    M, N, K = codes_x.shape[0], codes_w.shape[0], 2 * codes_x.shape[1]
    if not tiled:
        scales_x = scale_tiles(scales_x, K, stream=stream, group=fmt.group)
        scales_w = scale_tiles(scales_w, K, stream=stream, group=fmt.group)
    if out is None:
        out = torch.empty(M, N, dtype=torch.float32, device=codes_x.device)
    ts = None if tensor_scale is None else _ptr(tensor_scale)
    _check(lib().dq_w4a4_gemm(_ptr(codes_x), _ptr(scales_x), _ptr(codes_w), _ptr(scales_w),
                              _ptr(a), ts, M, N, K, ctypes.byref(fmt), _ptr(out), _stream(stream)),
           "dq_w4a4_gemm")
    return out


KIND_ROW, KIND_COL, KIND_PACK, KIND_ACT, KIND_FUSED = 0, 1, 2, 3, 4


def kernel_timing(enable: bool, kinds=None):
    """Bracket the tile-kernel launches of the given kinds (all when None)
    with CUDA events on their stream; enable=False turns timing off."""
    mask = 0
    if enable:
        mask = 0x1F if kinds is None else sum(1 << int(k) for k in kinds)
    _check(lib().dq_kernel_timing(mask), "dq_kernel_timing")


def kernel_time(kind: int):
    """(summed ms, launches) of one tile-kernel kind since the last read."""
    ms, n = c_double(0), c_int64(0)
    _check(lib().dq_kernel_time(kind, ctypes.byref(ms), ctypes.byref(n)), "dq_kernel_time")
    return ms.value, n.value


def launch_count() -> int:
    """Kernels this library has launched in the process so far."""
    return lib().dq_launch_count()


def last_device_status(stream=None) -> int:
    """Synchronise and return (and clear) the device flags as a dq status code."""
    return lib().dq_last_device_status(_stream(stream))
