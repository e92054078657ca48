"""Solve of one matrix whose rows are sharded over several ranks (one process
per GPU), with one exchange per iteration.

DualQuant's closed-form updates (daiwk note, "核心公式", eq. (2)): the row
update of row i reads only row i (given b), the column update of column j
sums over every row.  So with the rows split across ranks, each iteration is

* the row half-step on each rank's own rows (local, `row_update`);
* the column statistics of each rank's rows as partial sums per row block
  (`col_partials`), exchanged by an all-gather of the slabs in rank (= row)
  order, and finalized by every rank from all of them in the fixed
  summation order of the unsharded column update (`col_finalize`): every
  rank holds the same b, bit for bit the unsharded solve's b when every
  shard starts on a multiple of the matrix's column row block;
* the MSE trace: each rank's shard MSE weighted by its rows, summed over
  the ranks (an all-reduce of one number per half-step).

The NVFP4 tensor scale (a power of two rounded up from amax(W)) is the
largest of the shards' tensor scales, which is the tensor scale of the
whole matrix.  Every step runs in the library's kernels; this module only
orders the calls and the exchanges.
"""
from __future__ import annotations

import torch

from . import (col_finalize, col_partials, col_row_block, quantize, row_update,
               solve_dual_scale)


class TorchExchange:
    """The exchanges over a torch.distributed process group (NCCL for CUDA
    tensors, gloo for CPU tensors)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)

    def all_gather_rows(self, t: torch.Tensor, counts) -> torch.Tensor:
        """Concatenation along dim 0 of every rank's t (rank order); rank r
        holds counts[r] rows, padded to the largest for the exchange."""
        n = max(counts)
        pad = torch.zeros((n,) + tuple(t.shape[1:]), dtype=t.dtype, device=t.device)
        pad[:t.shape[0]] = t
        parts = [torch.empty_like(pad) for _ in range(self.world)]
        self.dist.all_gather(parts, pad, group=self.group)
        return torch.cat([p[:c] for p, c in zip(parts, counts)], dim=0)

    def all_reduce_sum(self, t: torch.Tensor) -> torch.Tensor:
        self.dist.all_reduce(t, op=self.dist.ReduceOp.SUM, group=self.group)
        return t

    def all_reduce_max(self, t: torch.Tensor) -> torch.Tensor:
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX, group=self.group)
        return t


class RowShard:
    """Rows [row0, row0 + rows) of a rows_total x cols matrix on this device,
    with their row scales a; b is the matrix's (the same on every rank)."""

    def __init__(self, W, row0, rows_total, fmt, a0=None):
        self.W, self.row0, self.rows_total, self.fmt = W, row0, rows_total, fmt
        rows, cols = W.shape
        self.row_block = col_row_block(rows_total, cols, W.dtype)
        if row0 % self.row_block:
            raise ValueError(f"shard start {row0} is not a multiple of the row block "
                             f"{self.row_block}")
        self.a = (torch.ones(rows, dtype=torch.float32, device=W.device) if a0 is None
                  else a0.to(torch.float32).clone())
        self.ts = 1.0

    def tensor_scale(self) -> float:
        """This shard's tensor scale (a solve of no iterations computes it)."""
        if not self.fmt.tensor_scale_auto or self.W.shape[0] == 0:
            return 1.0
        return float(solve_dual_scale(self.W, self.fmt, 0, half=False)["tensor_scale"].item())

    def row_step(self, b):
        """a <- the row update from (a, b); returns this shard's MSE of the
        state before it times its share of the rows."""
        a, _, mse = row_update(self.W, self.fmt, self.a, b, self.ts)
        self.a = a
        return mse * (self.W.shape[0] / self.rows_total)

    def col_partials(self, b):
        """The column partial sums of this shard's rows at (a, b) and its
        share of the MSE of that state."""
        parts, mse = col_partials(self.W, self.fmt, self.a, b, self.row_block, self.ts)
        return parts, mse * (self.W.shape[0] / self.rows_total)

    def col_finalize(self, parts):
        return col_finalize(parts, self.fmt)[0]

    def pack(self, b):
        """Codes and group scales of this shard at (a, b)."""
        return quantize(self.W, self.fmt, self.a, b, self.ts)


def solve_rows_sharded(W_shard, row_starts, rank, fmt, T, exchange, a0=None, b0=None,
                       shard_type=RowShard):
    """T iterations of the dual-scale solve of a matrix whose rows
    [row_starts[r], row_starts[r + 1]) live on rank r (row_starts[-1] = all
    rows; every start a multiple of `col_row_block(rows, cols)`).  Returns
    this rank's a, codes and group scales, the common b and tensor scale, and
    the MSE traces of the whole matrix (mse_trace[T + 1], mse_half[T])."""
    rows_total, cols = row_starts[-1], W_shard.shape[1]
    sh = shard_type(W_shard, row_starts[rank], rows_total, fmt, a0)
    counts = [-(-(row_starts[r + 1] - row_starts[r]) // sh.row_block)
              for r in range(len(row_starts) - 1)]
    dev = W_shard.device
    ts = torch.tensor([sh.tensor_scale()], dtype=torch.float32, device=dev)
    sh.ts = float(exchange.all_reduce_max(ts).item())
    b = (torch.ones(cols, dtype=torch.float32, device=dev) if b0 is None
         else b0.to(torch.float32).clone())
    trace, half = [], []
    for _ in range(T):
        trace.append(exchange.all_reduce_sum(sh.row_step(b)))
        parts, mse = sh.col_partials(b)
        half.append(exchange.all_reduce_sum(mse))
        b = sh.col_finalize(exchange.all_gather_rows(parts, counts))
    # the MSE of the final state: the column statistics of (a, b) carry it
    _, mse = sh.col_partials(b)
    trace.append(exchange.all_reduce_sum(mse))
    codes, gscales = sh.pack(b)
    return dict(a=sh.a, b=b, codes=codes, gscales=gscales, tensor_scale=sh.ts,
                mse_trace=torch.cat(trace), mse_half=torch.cat(half) if half else torch.zeros(0))
