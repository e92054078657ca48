#!/usr/bin/env python
"""Benchmark of the dual-scale solver hot path on B200.

One step = one full DualQuant solve of every linear layer of the workload
(T block-coordinate-descent iterations plus the final pack pass, all in one
batched launch sequence; `--graph` replays it as a CUDA graph instead)
followed by the activation rescale + quantize of the workload's activation
batch with the solved b of the first linear (q_proj).

Metric: solver weight-elements per second per BCD iteration, i.e.
(sum of rows*cols) * T / step time; the step time also includes the final
pack pass and the activation kernel, so the figure is conservative.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME]
    python bench.py --impl reference ...      # the fp64 CPU oracle arm

With N > 1 (torchrun, one rank per GPU) every rank solves a different decoder
of the same model (weak scaling); no collective touches the data path, only
the max-over-ranks of the timings.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import re
import glob
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

DEFAULT_CONFIG = "llama31_70b_decoder_mxfp4_g32"
METRIC = "solver weight-elements/s per BCD iteration"
UNIT = "weight-elements/s"
L2_BYTES = 126e6          # B200 L2 capacity (126 MB)


def _args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--config", default=DEFAULT_CONFIG)
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-rows", type=int, default=256,
                   help="rows of q_proj in the oracle's bounded sample")
    p.add_argument("--only", type=int, default=-1,
                   help="profiling case: keep only this linear of the decoder")
    p.add_argument("--T", type=int, default=-1, help="profiling case: iterations override")
    p.add_argument("--no-act", action="store_true", help="profiling case: skip activations")
    p.add_argument("--decoders", type=int, default=-1,
                   help="profiling case: solve only this many of the workload's decoders")
    p.add_argument("--tokens", type=int, default=32768, help="w4a4_gemm: activation rows")
    p.add_argument("--graph", action="store_true",
                   help="solve by replaying a CUDA graph of the batched solve "
                        "(dq_graph_solve_batched); the dominant kernel is then event-timed in a "
                        "direct-call step after the timed region")
    p.add_argument("--method", default="dualquant", choices=["dualquant", "two_level", "w4a4_gemm"],
                   help="two_level: the two-level absmax quantization of the same weights "
                        "and activations instead of the solve")
    return p.parse_args()


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "measured"
    except OSError:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}, "fallback"


def _code_only(text):
    """C++ source without its comments and blank lines (a change to a comment
    changes no kernel)."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    out = []
    for line in text.splitlines():
        line = re.sub(r"//.*$", "", line).rstrip()
        if line.strip():
            out.append(line)
    return "\n".join(out)


def _src_hash():
    """Hash of the code (comments left out) of the sources that fix the tile
    kernels and their launch geometry (the device header, the launch header
    and the per-format tile units); the host API, the GEMM and the two-level
    kernel do not change their traffic."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "dual_scale_solver_b200", "csrc")
    files = [os.path.join(csrc, "dq_device.cuh"), os.path.join(csrc, "dq_launch.h")]
    files += sorted(glob.glob(os.path.join(csrc, "dq_tiles_c*.cu")))
    for p in files:
        with open(p, encoding="utf-8") as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def _traffic(kind_name):
    """ncu DRAM bytes per launch for the kernel, if a committed capture of the
    current source exists (profiles/traffic.json); else None."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            t = json.load(f)
    except OSError:
        return None
    e = t.get(kind_name)
    if not e or e.get("src_hash") != _src_hash():
        return None
    return e.get("bytes_per_launch_full")


class Clocks:
    """nvidia-smi sampling (every 50 ms) of SM clock and throttle reasons; the
    samples whose timestamps fall inside the host-side window around the timed
    loop (mark("t0") before it, mark("t1") after its final synchronize) are the
    ones reported (window "timed"); a window too short to hold one sample
    reports those within 0.25 s of it (window "near")."""

    Q = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.t0 = self.t1 = None

    def mark(self, which):
        setattr(self, which, datetime.datetime.now())

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        rows = []
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f")
                rows.append((ts, float(f[2]), float(f[3]),
                             [n for n, v in zip(names, f[6:10]) if v.lower() == "active"]))
            except ValueError:
                continue
        window = "all"
        if self.t0 is not None and self.t1 is not None:
            inside = [r for r in rows if self.t0 <= r[0] <= self.t1]
            pad = datetime.timedelta(seconds=0.25)
            near = [r for r in rows if self.t0 - pad <= r[0] <= self.t1 + pad]
            if inside:
                rows, window = inside, "timed"
            elif near:
                rows, window = near, "near"
        sm = [r[1] for r in rows]
        mx = [r[2] for r in rows]
        reasons = sorted({n for r in rows for n in r[3]})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(sm), "window": window}


# --------------------------------------------------------------------------- #
# CPU oracle (baseline leg and reference arm)
# --------------------------------------------------------------------------- #

def _oracle_sample(wl, rows, decoder=0):
    import numpy as np
    import synth
    import oracle as O
    W = synth.weight(wl, decoder, 0, rows=rows).double().numpy()
    fmt = O.preset(wl.fmt, wl.group)
    return W, fmt, np, O


def _oracle_iteration(W, fmt, np, O, a, b, ts):
    """One BCD iteration of the oracle from (a, b): row update, re-quantize,
    column update, re-quantize."""
    Qh, _, _ = O.qhat(W, a, b, fmt, ts)
    a, _ = O.row_update(W, Qh, b, fmt)
    Qh, _, _ = O.qhat(W, a, b, fmt, ts)
    b, _ = O.col_update(W, Qh, a, fmt)
    return a, b


def host_cores() -> int:
    return len(os.sched_getaffinity(0))


# Worker side of the all-cores oracle timing (spawned processes: numpy and
# the oracle only).  Each worker holds its own row sample.
_W_SAMPLE = None


def _worker_init(sample, wl_fmt, wl_group):
    global _W_SAMPLE
    import numpy as np
    import oracle as O
    W = np.asarray(sample, dtype=np.float64)
    fmt = O.preset(wl_fmt, wl_group)
    _W_SAMPLE = (W, fmt, O.tensor_scale(W, fmt))


def _worker_window(start_at, seconds):
    """Whole BCD iterations of the oracle on this worker's sample from
    `start_at` (wall clock) for about `seconds`; returns (elements x
    iterations, elapsed seconds)."""
    import numpy as np
    import oracle as O
    W, fmt, ts = _W_SAMPLE
    while time.time() < start_at:
        time.sleep(0.001)
    a, b = np.ones(W.shape[0]), np.ones(W.shape[1])
    its, t0 = 0, time.perf_counter()
    while True:
        a, b = _oracle_iteration(W, fmt, np, O, a, b, ts)
        its += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            return W.size * its, el


def _worker_iteration(_):
    """One BCD iteration of the oracle on this worker's sample from a = b = 1."""
    import numpy as np
    import oracle as O
    W, fmt, ts = _W_SAMPLE
    _oracle_iteration(W, fmt, np, O, np.ones(W.shape[0]), np.ones(W.shape[1]), ts)
    return W.size


class OraclePool:
    """One spawned process per host core (os.sched_getaffinity), each with
    its own seeded row sample of the workload: the first `rows` rows of
    q_proj of decoder k for worker k (i.i.d. draws of the same shape and
    distribution).  Spawned, not forked, so that it is safe after CUDA use."""

    def __init__(self, wl, rows, n=None):
        import multiprocessing as mp
        self.n = n or host_cores()
        self.rows = rows
        os.environ.setdefault("OMP_NUM_THREADS", "1")
        os.environ.setdefault("OPENBLAS_NUM_THREADS", "1")
        ctx = mp.get_context("spawn")
        samples = [_oracle_sample(wl, rows, decoder=k)[0].astype("float32") for k in range(self.n)]
        self.shape = samples[0].shape
        self.pool = [ctx.Pool(1, initializer=_worker_init, initargs=(samples[k], wl.fmt, wl.group))
                     for k in range(self.n)]

    def window(self, seconds):
        """Aggregate rate (elements x iterations / s) of all workers running
        iterations over the same wall-clock window."""
        start_at = time.time() + 1.0
        res = [p.apply_async(_worker_window, (start_at, seconds)) for p in self.pool]
        out = [r.get() for r in res]
        return sum(w / el for w, el in out), out

    def step(self):
        """One iteration on every worker's sample at once; returns elements."""
        res = [p.apply_async(_worker_iteration, (0,)) for p in self.pool]
        return sum(r.get() for r in res)

    def close(self):
        for p in self.pool:
            p.close()
            p.join()


def cpu_baseline(wl, rows, min_seconds=10.0):
    """The oracle on the host cores: one thread on a bounded sample, then one
    process per core over a common window, each on its own sample."""
    W, fmt, np, O = _oracle_sample(wl, rows)
    ts = O.tensor_scale(W, fmt)
    a, b = np.ones(W.shape[0]), np.ones(W.shape[1])
    its, t0 = 0, time.perf_counter()
    while True:
        a, b = _oracle_iteration(W, fmt, np, O, a, b, ts)
        its += 1
        el = time.perf_counter() - t0
        if el >= min_seconds or its >= 50:
            break
    single = W.size * its / el
    pool = OraclePool(wl, rows)
    try:
        value, parts = pool.window(min_seconds)
    finally:
        pool.close()
    its_all = sum(w for w, _ in parts) // W.size
    sample = (f"the fp64 numpy oracle, whole BCD iterations (row update, re-quantize, column "
              f"update, re-quantize) on the first {rows} rows of q_proj "
              f"({W.shape[0]}x{W.shape[1]}, {wl.fmt} G{wl.group}): {pool.n} processes, one "
              f"per host core, each on its own decoder's sample, {its_all} iterations in "
              f"{min_seconds:.0f} s; one thread alone: {its} iterations on decoder 0 in "
              f"{el:.1f} s ({single:.3g} el/s/iter)")
    return {"value": value, "unit": UNIT, "cores": pool.n, "kind": "oracle", "sample": sample,
            "single_thread_value": single}


def run_reference(args, wl, rank, world):
    if rank != 0:
        return 0
    pool = OraclePool(wl, args.cpu_rows)
    try:
        for _ in range(args.warmup):
            pool.step()
        t0 = time.perf_counter()
        el_total = 0
        for _ in range(args.steps):
            el_total += pool.step()
        el = time.perf_counter() - t0
    finally:
        pool.close()
    value = el_total / el
    sample = (f"each step one BCD iteration of the fp64 numpy oracle on each of {pool.n} "
              f"row samples at once ({pool.n} processes, one per host core; sample k: the "
              f"first {args.cpu_rows} rows of decoder k's {wl.linears[0].name}, "
              f"{pool.shape[0]}x{pool.shape[1]}, {wl.fmt} G{wl.group})")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": el / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "sample_rows": args.cpu_rows, "processes": pool.n},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": pool.n, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------- #
# Multi-GPU plumbing (weak scaling, no collective on the data path)
# --------------------------------------------------------------------------- #

def decoders_of(rank: int, per_rank: int) -> list:
    """Decoders that rank `rank` solves: every rank its own block of
    `per_rank` seeded decoders (the workload's decoder count), so per-GPU work
    is fixed as the number of GPUs grows."""
    return list(range(rank * per_rank, (rank + 1) * per_rank))


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank timing over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as tdist
    if not (tdist.is_available() and tdist.is_initialized()) or tdist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    tdist.all_reduce(t, op=tdist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(elements_per_rank: int, T: int, world: int, ms_per_step: float) -> float:
    """Weight-elements per second per BCD iteration over all ranks."""
    return world * elements_per_rank * T / (ms_per_step / 1e3)


# --------------------------------------------------------------------------- #
# GPU arm
# --------------------------------------------------------------------------- #

def run_ours(args, wl, rank, world, local_rank):
    import torch
    import synth
    import dual_scale_solver_b200 as dq
    from dual_scale_solver_b200 import build

    dist = world > 1
    if dist:
        import torch.distributed as tdist
        from datetime import timedelta
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    build.build()

    # weak scaling: rank r solves its own block of decoders (seeded per decoder)
    idx = [args.only] if args.only >= 0 else range(len(wl.linears))
    n_dec = wl.decoders if args.decoders < 0 else min(args.decoders, wl.decoders)
    Ws = [synth.weight(wl, d, i, device=dev) for d in decoders_of(rank, n_dec) for i in idx]
    fmt = dq.format_preset(wl.fmt, wl.group)
    act = None if args.no_act else wl.act
    X = synth.activation(wl, device=dev) if act else None
    fmt_act = dq.format_preset(act["fmt"], act["group"]) if act else None
    T = wl.T if args.T < 0 else args.T
    E = sum(W.numel() for W in Ws)
    ws = dq.workspace([tuple(W.shape) for W in Ws], fmt, dev)
    outs = None
    act_out = None
    graph = None
    stream = torch.cuda.current_stream(dev)

    def step(direct=False):
        nonlocal outs, act_out, graph
        if args.graph and not direct:
            if graph is None:
                graph = dq.solve_dual_scale_batched_graph(Ws, fmt, T, ws=ws, outs=outs)
                outs = graph.outs
            graph.launch(stream=stream)
        else:
            outs = dq.solve_dual_scale_batched(Ws, fmt, T, ws=ws, outs=outs)
        if X is not None:
            if act_out is None:
                act_out = dq.act_rescale_quant(X, outs[0]["b"], fmt_act)
            else:
                dq.act_rescale_quant(X, outs[0]["b"], fmt_act, codes=act_out[0], gscales=act_out[1])

    def barrier():
        if dist:
            tdist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if dq.last_device_status() != 0:
        raise RuntimeError("device status flags raised during warm-up")

    clocks = Clocks(local_rank)
    barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    time.sleep(0.3)
    # The dominant tile kernel is event-timed inside the timed region, in its
    # last step only: an event pair around a launch separates it from its
    # neighbours (no overlap of its start with the previous kernel's tail),
    # so the other steps run without events.
    # power-of-two group and outer scales (the MX family): one-pass iterations
    fused_fmt = fmt.group_scale == dq.DQ_SCALE_E8M0 and fmt.outer_scale == dq.DQ_SCALE_E8M0
    dom_kinds = (4,) if fused_fmt else (0, 1)
    for k in range(5):
        dq.kernel_time(k)                     # clear
    n0 = dq.launch_count()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    clocks.mark("t0")
    e0.record(stream)
    for i in range(args.steps):
        if i == args.steps - 1:
            dq.kernel_timing(True, kinds=dom_kinds)
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    clocks.mark("t1")
    barrier()
    ms = e0.elapsed_time(e1)
    launches = dq.launch_count() - n0
    kt = {k: dq.kernel_time(k) for k in range(5)}
    dq.kernel_timing(False)
    clk = clocks.stop()
    # per-kind breakdown: one more step, untimed, with every tile kind timed
    # (direct calls: graph replays take no timing events)
    dq.kernel_timing(True)
    step(direct=True)
    torch.cuda.synchronize(dev)
    kb = {k: dq.kernel_time(k) for k in range(5)}
    dq.kernel_timing(False)
    if graph is not None:
        graph.close()
    ms = max_over_ranks(ms, dev)

    ms_step = ms / args.steps
    value = whole_job_rate(E, T, world, ms_step)
    in_bytes = sum(W.numel() * W.element_size() for W in Ws) + (
        X.numel() * X.element_size() if X is not None else 0)

    # dominant tile kernel and its roofline (HBM: it streams W once per launch)
    names = {0: "row_stats", 1: "col_stats", 2: "pack", 3: "act_quant", 4: "fused_row_col_stats"}
    # (graph replays: the dominant kernel's launches are timed in the direct step)
    kt_dom = kb if args.graph else kt
    dom = max(dom_kinds, key=lambda k: kt_dom[k][0])
    tot_ms, nl = kt_dom[dom]
    avg_s = tot_ms / max(nl, 1) / 1e3
    rows_sum = sum(W.shape[0] for W in Ws)
    cols_sum = sum(W.shape[1] for W in Ws)
    alg_bytes = E * Ws[0].element_size() + 4 * (rows_sum + cols_sum)
    peaks, which = _peaks()
    peak = float(peaks["hbm_gbs"])
    achieved = alg_bytes / avg_s / 1e9
    roofline = {"bound": "hbm", "kernel": names[dom], "achieved": achieved, "peak": peak,
                "unit": "GB/s", "frac": achieved / peak, "peak_source": which,
                "traffic": _traffic(names[dom]), "algorithmic_bytes_per_launch": alg_bytes,
                "avg_launch_ms": avg_s * 1e3,
                "kernel_ms_per_step": {names[k]: kb[k][0] for k in kb},
                "kernel_ms_per_step_from": "one extra step after the timed region, every tile kind event-timed"}
    roofline["avg_launch_ms_from"] = (
        "the direct-call step after the timed region (graph replays take no events)" if args.graph else
        f"the last of the {args.steps} timed steps: its {nl} launches of this kernel, CUDA events on the "
        "launch stream (the other timed steps run without events)")

    # end-to-end: host buffers in, results out, every step.  The weights go
    # through the host-streamed solve (group g+1 of consecutive matrices
    # crosses the bus while group g is solved and group g-1's results come
    # back), largest first so that the last, small matrices leave a short tail; the activation
    # batch is copied on a stream of its own and quantized with q_proj's b
    # once the solves are done.  The step is bound by the bus: 2.25 GB in and
    # 0.6 GB out.
    e2e = None
    if not args.no_e2e:
        order = sorted(range(len(Ws)), key=lambda i: -Ws[i].numel())
        hW = [Ws[i].to("cpu").pin_memory() for i in order]
        q_pos = order.index(0)
        hX = X.to("cpu").pin_memory() if X is not None else None
        dX = torch.empty_like(X) if X is not None else None
        h2d = sum(w.numel() * w.element_size() for w in hW) + (
            hX.numel() * hX.element_size() if hX is not None else 0)
        x_stream = torch.cuda.Stream(dev)
        _, d2h_stream = dq.copy_streams(dev)
        ws_h = dq.workspace([tuple(W.shape) for W in Ws], fmt, dev)
        staging = [torch.empty_like(Ws[i]) for i in order]
        host_outs = dev_outs = act_h = None

        def e2e_step():
            nonlocal host_outs, dev_outs, act_out, act_h
            if dX is not None:
                x_stream.wait_stream(stream)          # the previous step's activation pass
                with torch.cuda.stream(x_stream):
                    dX.copy_(hX, non_blocking=True)
            host_outs, dev_outs = dq.solve_dual_scale_batched_host(
                hW, fmt, T, outs=host_outs, dev_outs=dev_outs, staging=staging, ws=ws_h,
                stream=stream, wait_out=False)
            if dX is not None:
                stream.wait_stream(x_stream)
                dq.act_rescale_quant(dX, dev_outs[q_pos]["b"], fmt_act, codes=act_out[0],
                                     gscales=act_out[1])
                if act_h is None:
                    act_h = [torch.empty(r.shape, dtype=r.dtype, pin_memory=True) for r in act_out]
                d2h_stream.wait_stream(stream)
                with torch.cuda.stream(d2h_stream):
                    for h, d in zip(act_h, act_out):
                        h.copy_(d, non_blocking=True)
            # the step's copies back run on while the next step's inputs come in
            # (the library orders each call after the copies back it depends on);
            # the timed region ends after the last step's copies back
            n = sum(v.numel() * v.element_size() for o in host_outs for v in o.values()
                    if v is not None)
            return n + (sum(v.numel() * v.element_size() for v in act_h) if act_h else 0)

        d2h = e2e_step()
        torch.cuda.synchronize(dev)
        barrier()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(args.steps):
            e2e_step()
        stream.wait_stream(d2h_stream)
        f1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        ems = max_over_ranks(f0.elapsed_time(f1), dev)
        e2e = {"value": whole_job_rate(E, T, world, ems / args.steps), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": ems / args.steps}

    if dq.last_device_status() != 0:
        raise RuntimeError("device status flags raised during timing")

    if args.only >= 0 or args.T >= 0 or args.no_act or args.decoders >= 0:
        wl_name = (f"{wl.name} (profiling subset: only={args.only} T={T} act={act is not None} "
                   f"decoders={n_dec})")
    else:
        wl_name = wl.name
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": wl_name, "matrices": len(Ws), "elements_per_gpu": E, "T": T,
                   "format": f"{wl.fmt} G{wl.group}",
                   "activation": (f"{act['tokens']}x{act['K']} bf16 -> {act['fmt']} G{act['group']}"
                                  if act else None),
                   "l2": ("inputs larger than L2 (no flush needed)" if in_bytes > L2_BYTES else
                          f"inputs ({in_bytes / 1e6:.1f} MB) fit in L2 and stay resident across "
                          "steps (not flushed)"),
                   "launch": "CUDA graph replay" if args.graph else "direct calls",
                   "parallelism": f"{world} independent decoders" if world > 1 else "1 GPU"},
        "roofline": roofline,
        "gpu_launches": launches,
        "clocks": clk,
        "e2e": e2e,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl, args.cpu_rows)
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def run_two_level(args, wl, rank, world, local_rank):
    """Two-level absmax quantization of the workload's weights (codes and
    scales) and of its activation batch (codes, scales and the float32
    reconstruction), one step = all of it, 1 GPU per rank (weak scaling)."""
    import torch
    import synth
    import dual_scale_solver_b200 as dq
    from dual_scale_solver_b200 import build

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    build.build()
    D = 512
    Ws = [synth.weight(wl, d, i, device=dev) for d in decoders_of(rank, wl.decoders)
          for i in range(len(wl.linears))]
    X = synth.activation(wl, device=dev) if wl.act and not args.no_act else None
    stream = torch.cuda.current_stream(dev)
    E = sum(W.numel() for W in Ws) + (X.numel() if X is not None else 0)

    def step(time_w=None):
        if time_w:
            time_w[0].record(stream)
        for W in Ws:
            dq.two_level_quant(W, D, qdq=False)
        if time_w:
            time_w[1].record(stream)
        if X is not None:
            dq.two_level_quant(X, D, qdq=True)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    clocks = Clocks(local_rank)
    clocks.start()
    time.sleep(0.3)
    n0 = dq.launch_count()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    clocks.mark("t0")
    e0.record(stream)
    for k in range(args.steps):
        step(ev[k])
    e1.record(stream)
    torch.cuda.synchronize(dev)
    clocks.mark("t1")
    ms = max_over_ranks(e0.elapsed_time(e1), dev) / args.steps
    launches = dq.launch_count() - n0
    clk = clocks.stop()
    w_ms = sum(a.elapsed_time(b) for a, b in ev) / args.steps
    Ew = sum(W.numel() for W in Ws)
    rows_nb = sum(W.shape[0] * -(-W.shape[1] // D) for W in Ws)
    alg = Ew * 2 + Ew // 2 + Ew // 32 + 4 * rows_nb        # read W, write codes + scales
    peaks, which = _peaks()
    peak = float(peaks["hbm_gbs"])
    achieved = alg / (w_ms / 1e3) / 1e9
    unit = "quantized elements/s"
    e2e = None
    if not args.no_e2e:
        hW = [W.to("cpu").pin_memory() for W in Ws]
        dW = [torch.empty_like(W) for W in Ws]
        outs = [(torch.empty(W.shape[0], W.shape[1] // 2, dtype=torch.uint8, pin_memory=True),
                 torch.empty(W.shape[0], W.shape[1] // 32, dtype=torch.uint8, pin_memory=True))
                for W in Ws]
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(args.steps):
            for h, d, (hc, hs) in zip(hW, dW, outs):
                d.copy_(h, non_blocking=True)
                c, si, so, _ = dq.two_level_quant(d, D, qdq=False)
                hc.copy_(c, non_blocking=True)
                hs.copy_(si, non_blocking=True)
        f1.record(stream)
        torch.cuda.synchronize(dev)
        ems = max_over_ranks(f0.elapsed_time(f1), dev) / args.steps
        e2e = {"value": world * Ew / (ems / 1e3), "unit": unit,
               "h2d_bytes_per_step": sum(h.numel() * h.element_size() for h in hW),
               "d2h_bytes_per_step": sum(c.numel() + s.numel() for c, s in outs),
               "ms_per_step": ems, "scope": "weights only"}
    if dq.last_device_status() != 0:
        raise RuntimeError("device status flags raised during timing")
    line = {
        "metric": "two-level absmax quantized elements/s", "value": world * E / (ms / 1e3),
        "unit": unit, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic",
        "config": {"workload": f"{wl.name} weights + activations, two-level absmax (outer "
                               f"{D}-column blocks, inner MXFP4 G32)",
                   "elements_per_gpu": E, "l2": "inputs larger than L2 (no flush needed)",
                   "parallelism": f"{world} independent decoders" if world > 1 else "1 GPU"},
        "roofline": {"bound": "hbm", "kernel": "two_level (weights: codes + scales)",
                     "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "peak_source": which, "traffic": None, "algorithmic_bytes_per_step": alg,
                     "weights_ms_per_step": w_ms},
        "gpu_launches": launches, "clocks": clk, "e2e": e2e,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def run_gemm(args, wl, rank, world, local_rank):
    """The inference step after the solve: every linear of the workload's
    decoder(s) as a block-scaled W4A4 GEMM (MXFP4 x MXFP4 with E8M0 scales;
    NVFP4 x NVFP4 with E4M3 scales and the weights' tensor scale for an NVFP4
    workload) on a batch of `tokens` activation rows; the weights' codes,
    scales, tensor scale and a come
    from the solve, the activations' codes and scales from the activation
    quantizer (one batch per input width)."""
    import torch
    import synth
    import dual_scale_solver_b200 as dq
    from dual_scale_solver_b200 import build

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    build.build()
    nv = wl.fmt == "nvfp4"
    fmt = dq.format_preset("nvfp4" if nv else "mxfp4")
    # (--decoders caps the decoders per rank: the float32 outputs of all
    # linears of the 32-decoder sets at 32768 tokens exceed the device memory)
    n_dec = wl.decoders if args.decoders < 0 else min(args.decoders, wl.decoders)
    Ws = [synth.weight(wl, d, i, device=dev) for d in decoders_of(rank, n_dec)
          for i in range(len(wl.linears))]
    outs = dq.solve_dual_scale_batched(Ws, fmt, wl.T)
    M = args.tokens
    acts = {}
    for W in Ws:                                  # one quantized activation batch per width K
        K = W.shape[1]
        if K not in acts:
            X = synth.normal(synth.stream_key(70, K), M * K, device=dev).view(M, K).to(torch.bfloat16)
            acts[K] = dq.act_rescale_quant(X, torch.ones(K, device=dev), fmt)
            del X
    res = [torch.empty(M, W.shape[0], dtype=torch.float32, device=dev) for W in Ws]
    del Ws
    stream = torch.cuda.current_stream(dev)
    # the GEMM reads group scales as scale tiles: the weights' once after the
    # solve, the activation batches' once per batch
    wtiles = [dq.scale_tiles(o["gscales"], group=fmt.group) for o in outs]
    acts = {K: (cx, dq.scale_tiles(sx, group=fmt.group)) for K, (cx, sx) in acts.items()}

    def step():
        for o, r, sw in zip(outs, res, wtiles):
            cx, sx = acts[2 * o["codes"].shape[1]]
            dq.w4a4_gemm(cx, sx, o["codes"], sw, o["a"], fmt, out=r, tiled=True,
                         tensor_scale=o["tensor_scale"] if nv else None)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    clocks = Clocks(local_rank)
    clocks.start()
    time.sleep(0.3)
    n0 = dq.launch_count()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    clocks.mark("t0")
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    clocks.mark("t1")
    ms = max_over_ranks(e0.elapsed_time(e1), dev) / args.steps
    launches = dq.launch_count() - n0
    clk = clocks.stop()
    if dq.last_device_status() != 0:
        raise RuntimeError("device status flags raised during timing")
    flops = sum(2.0 * M * o["codes"].shape[0] * 2 * o["codes"].shape[1] for o in outs)
    peaks, which = _peaks()
    # FP4 dense peak = the measured bf16 GEMM peak x the nominal fp4/bf16 ratio (9 / 2.25);
    # a timed region of more than half a second of back-to-back products runs
    # under the power cap, so it is held against the sustained bf16 figure
    sustained = ms * args.steps > 500.0 and "bf16_tflops_sustained" in peaks
    peak_key = "bf16_tflops_sustained" if sustained else "bf16_tflops"
    peak = float(peaks.get(peak_key, 1590.0)) * 4.0
    tflops = flops / (ms / 1e3) / 1e12
    line = {
        "metric": ("W4A4 GEMM TFLOP/s (NVFP4 x NVFP4, E4M3 scales per 16, fp32 accumulate)" if nv
                   else "W4A4 GEMM TFLOP/s (MXFP4 x MXFP4, E8M0 scales, fp32 accumulate)"),
        "value": world * tflops, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "fp4 (e2m1)", "data": "synthetic",
        "config": {"workload": f"{wl.name}: its {len(outs)} linears x {M} tokens",
                   "flops_per_step": flops, "tile": "256 x 256 per CTA pair (tcgen05 cta_group::2), K tile 256, 6-stage ring (M, N multiples of 256; else 128 x 256 or 128 x 128 per CTA)",
                   "l2": "operands larger than L2 (no flush needed)",
                   "parallelism": f"{world} independent decoders" if world > 1 else "1 GPU"},
        "roofline": {"bound": "tensor", "achieved": tflops, "peak": peak, "unit": "TFLOP/s",
                     "frac": tflops / peak,
                     "peak_source": f"{which} {'sustained' if sustained else 'burst'} bf16 x 4 "
                                    f"(nominal fp4/bf16 ratio; timed region {ms * args.steps / 1e3:.2f} s)",
                     "traffic": None},
        "gpu_launches": launches, "clocks": clk, "e2e": None,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def main():
    args = _args()
    import synth
    wl = synth.WORKLOADS[args.config]
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, wl, rank, world)
    if world > 1:
        import torch
        import torch.distributed as tdist
        from datetime import timedelta
        torch.cuda.set_device(local_rank)
        tdist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                 device_id=torch.device("cuda", local_rank))
    try:
        if args.method == "two_level":
            return run_two_level(args, wl, rank, world, local_rank)
        if args.method == "w4a4_gemm":
            return run_gemm(args, wl, rank, world, local_rank)
        return run_ours(args, wl, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as tdist
            tdist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
