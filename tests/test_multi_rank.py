"""The multi-GPU plumbing of bench.py on CPU: world size 2 over gloo.

The solve shards across GPUs by decoder (every rank solves its own decoder;
no collective touches the data path); only the step times meet in a max
reduction.  These tests run that logic on two CPU processes.
"""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        import synth
        wl = synth.WORKLOADS["llama31_70b_decoder_mxfp4_g32"]
        ds = bench.decoders_of(rank, 3)
        shards = [None] * world
        dist.all_gather_object(shards, ds)
        # this rank's matrix (a reduced-size slice of its first decoder's k_proj)
        w = synth.weight(wl, ds[0], 1, rows=4, cols=64)
        ws = [None] * world
        dist.all_gather_object(ws, w)
        # per-rank step times meet in a max
        ms = 10.0 + 5.0 * rank
        mx = bench.max_over_ranks(ms)
        rate = bench.whole_job_rate(1000, 15, world, mx)
        q.put((rank, shards, [x.clone() for x in ws], mx, rate))
    finally:
        dist.destroy_process_group()


def test_two_ranks_shard_by_decoder_and_reduce_timing():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    for rank, shards, ws, mx, rate in res:
        assert shards == [[0, 1, 2], [3, 4, 5]]       # disjoint decoder blocks
        assert not torch.equal(ws[0], ws[1])          # different seeded weights
        assert mx == 15.0                             # the slowest rank's time
        assert rate == 2 * 1000 * 15 / (15.0 / 1e3)   # whole-job throughput


def test_reference_arm_runs_on_rank_zero_only(capsys):
    sys.path.insert(0, ROOT)
    import bench
    import synth

    class A:
        steps, warmup, cpu_rows, gpus = 1, 0, 8, 2

    wl = synth.WORKLOADS["llama31_70b_decoder_mxfp4_g32"]
    assert bench.run_reference(A, wl, rank=1, world=2) == 0
    assert capsys.readouterr().out == ""
    assert bench.run_reference(A, wl, rank=0, world=2) == 0
    import json
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["value"] > 0
