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


# --------------------------------------------------------------------------- #
# One matrix with its rows sharded over the ranks (dual_scale_solver_b200.sharded)
# --------------------------------------------------------------------------- #

class NpShard:
    """CPU stand-in of sharded.RowShard with the same interface: the oracle's
    quantizer and closed forms, the column statistics as float64 partial sums
    per block of 16 rows (fixed order), summed over the blocks in order."""

    ROW_BLOCK = 16

    def __init__(self, W, row0, rows_total, fmt, a0=None):
        import numpy as np
        import oracle as O
        self.np, self.O = np, O
        self.W = W.double().numpy()
        self.row0, self.rows_total, self.fmt = row0, rows_total, fmt
        self.row_block = self.ROW_BLOCK
        assert row0 % self.row_block == 0
        self.a = np.ones(self.W.shape[0]) if a0 is None else a0.double().numpy().copy()
        self.ts = 1.0

    def tensor_scale(self):
        return self.O.tensor_scale(self.W, self.fmt) if self.W.size else 1.0

    def row_step(self, b):
        b = b.double().numpy()
        Qh, _, _ = self.O.qhat(self.W, self.a, b, self.fmt, self.ts)
        mse = self.O.mse(self.W, Qh, self.a, b) * self.W.shape[0] / self.rows_total
        self.a, _ = self.O.row_update(self.W, Qh, b, self.fmt)
        return torch.tensor([mse], dtype=torch.float64)

    def col_partials(self, b):
        np = self.np
        b = b.double().numpy()
        Qh, _, _ = self.O.qhat(self.W, self.a, b, self.fmt, self.ts)
        S = self.a[:, None] * Qh
        rows = self.W.shape[0]
        nrb = -(-rows // self.row_block)
        parts = np.zeros((nrb, self.W.shape[1], 2))
        for k in range(nrb):
            blk = slice(k * self.row_block, (k + 1) * self.row_block)
            for i in range(blk.start, min(blk.stop, rows)):        # rows in order
                parts[k, :, 0] += self.W[i] * S[i]
                parts[k, :, 1] += S[i] * S[i]
        mse = self.O.mse(self.W, Qh, self.a, b) * rows / self.rows_total
        return torch.from_numpy(parts), torch.tensor([mse], dtype=torch.float64)

    def col_finalize(self, parts):
        np = self.np
        P, E = np.zeros(parts.shape[1]), np.zeros(parts.shape[1])
        for k in range(parts.shape[0]):                            # blocks in order
            P += parts[k, :, 0].numpy()
            E += parts[k, :, 1].numpy()
        pos = E > 0
        x = np.where(pos, P / np.where(pos, E, 1.0), 1.0)
        return torch.from_numpy(np.where(pos, self.O.project_outer(x, self.fmt), 1.0))

    def pack(self, b):
        c, s = self.O.quantize(self.O.inner(self.W, self.a, b.double().numpy()), self.fmt, self.ts)
        return torch.from_numpy(c), torch.from_numpy(s)


class LocalExchange:
    """One rank: the exchanges are the identity."""

    def all_gather_rows(self, t, counts):
        return t

    def all_reduce_sum(self, t):
        return t

    def all_reduce_max(self, t):
        return t


def _sharded_matrix():
    import numpy as np
    rng = np.random.default_rng(11)
    W = rng.standard_t(4, (80, 96)) * 0.02
    W[:, [5, 50]] *= 10
    W[33] = 0.0
    return torch.from_numpy(W).to(torch.bfloat16).double()


def _sharded_worker(rank, world, port, name, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle as O
        from dual_scale_solver_b200 import sharded
        W = _sharded_matrix()
        starts = [0, 48, 80]                 # shards start on multiples of the row block
        r0, r1 = starts[rank], starts[rank + 1]
        out = sharded.solve_rows_sharded(W[r0:r1], starts, rank, O.preset(name, 16), 3,
                                         sharded.TorchExchange(), shard_type=NpShard)
        q.put((rank, {k: (v.clone() if torch.is_tensor(v) else v) for k, v in out.items()}))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("name", ["int4_bf16", "nvfp4", "mxint4"])
def test_rows_sharded_over_two_ranks_equal_one_rank(name):
    # The row-sharded solve's exchange (column partial slabs all-gathered in
    # rank order and finalized in a fixed order; MSE shares and tensor scales
    # all-reduced) gives on two gloo ranks exactly what one rank gives.
    sys.path.insert(0, ROOT)
    import oracle as O
    from dual_scale_solver_b200 import sharded
    W = _sharded_matrix()
    one = sharded.solve_rows_sharded(W, [0, 80], 0, O.preset(name, 16), 3, LocalExchange(),
                                     shard_type=NpShard)
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_sharded_worker, args=(r, world, port, name, q))
             for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    two = res[0]
    for r in range(world):
        assert torch.equal(res[r]["b"], one["b"])                 # the same b on every rank
        assert res[r]["tensor_scale"] == one["tensor_scale"]
        assert torch.allclose(res[r]["mse_trace"], one["mse_trace"], rtol=1e-13, atol=0)
        assert torch.allclose(res[r]["mse_half"], one["mse_half"], rtol=1e-13, atol=0)
    a = torch.cat([torch.as_tensor(res[0]["a"]), torch.as_tensor(res[1]["a"])])
    assert torch.equal(a, torch.as_tensor(one["a"]))
    assert torch.equal(torch.cat([res[0]["codes"], res[1]["codes"]]), one["codes"])
    # and it is the oracle's solve (whose column sums run over all rows at once)
    r = O.solve(W.numpy(), O.preset(name, 16), 3)
    assert torch.allclose(two["mse_trace"], torch.from_numpy(r["mse_trace"]), rtol=1e-12, atol=0)
    assert torch.equal(one["b"], torch.from_numpy(r["b"]))
