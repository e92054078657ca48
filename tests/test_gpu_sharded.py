"""The row-sharded solve (dual_scale_solver_b200.sharded) on one GPU: the
shards of one matrix run in lockstep in this process, their column partial
slabs concatenated in row order as the all-gather of a multi-GPU run would,
and the result must be the unsharded solve's bit for bit (a, b, codes,
group scales).  The MSE trace agrees within 1e-6 relative: the row errors
of these 4-bit formats come from the row sums (sum W^2 - 2 a sum W R + a^2
sum R^2), the same per row in both, summed in another grouping.  For MXFP4
the unsharded solve's one-pass iterations form them from their a = 1 sums
(float32 sums of terms about 100 times the error), so there the trace
agrees within 2e-5."""
import numpy as np
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


def _weights(rows, cols, key):
    w = synth.student_t4(synth.stream_key(89, key, rows, cols), rows * cols).view(rows, cols) * 0.02
    idx = synth.distinct_indices(synth.stream_key(88, key, cols), cols, max(1, cols // 100))
    w[:, idx] *= 10
    return w.to(torch.bfloat16).cuda()


@pytest.mark.parametrize("name,G", [("int4_bf16", 64), ("nvfp4", 16), ("mxfp4", 32),
                                    ("mxint4_bf16outer", 32)])
@pytest.mark.parametrize("nshards", [2, 3])
def test_row_shards_equal_the_unsharded_solve(name, G, nshards):
    from dual_scale_solver_b200 import sharded
    fl = lib_format(name, G)
    rows, cols, T = 1536, 2240, 3
    W = _weights(rows, cols, key=nshards)
    rb = dq.col_row_block(rows, cols)
    assert rows // rb >= 6                              # shards span several row blocks
    # shard starts on multiples of the row block; the last shard is ragged
    starts = [0] + [((k * rows) // nshards) // rb * rb for k in range(1, nshards)] + [rows]
    shards = [sharded.RowShard(W[s0:s1], s0, rows, fl) for s0, s1 in zip(starts, starts[1:])]
    ts = max(sh.tensor_scale() for sh in shards)
    for sh in shards:
        sh.ts = ts
    b = torch.ones(cols, device="cuda")
    trace = []
    for _ in range(T):
        trace.append(sum(sh.row_step(b) for sh in shards))
        parts = torch.cat([sh.col_partials(b)[0] for sh in shards])
        b = shards[0].col_finalize(parts)
    trace.append(sum(sh.col_partials(b)[1] for sh in shards))
    packs = [sh.pack(b) for sh in shards]
    o = dq.solve_dual_scale(W, fl, T)
    torch.cuda.synchronize()
    assert dq.last_device_status() == 0
    assert float(o["tensor_scale"].item()) == ts
    assert torch.equal(torch.cat([sh.a for sh in shards]), o["a"])
    assert torch.equal(b, o["b"])
    assert torch.equal(torch.cat([p[0] for p in packs]), o["codes"])
    assert torch.equal(torch.cat([p[1] for p in packs]), o["gscales"])
    tr = torch.cat(trace).cpu().numpy()
    rtol = 2e-5 if name == "mxfp4" else 1e-6
    assert np.allclose(tr, o["mse_trace"].cpu().numpy(), rtol=rtol, atol=0)


def test_col_partials_refuse_a_row_block_below_the_shards_own():
    W = _weights(512, 1024, key=9)
    fl = dq.format_preset("int4_bf16")
    rb = dq.col_row_block(512, 1024)
    a = torch.ones(512, device="cuda")
    b = torch.ones(1024, device="cuda")
    with pytest.raises(dq.DqError):
        dq.col_partials(W, fl, a, b, rb // 2)
    parts, _ = dq.col_partials(W, fl, a, b, rb)
    b1, _ = dq.col_finalize(parts, fl)
    b2, _, _ = dq.col_update(W, fl, a, b)
    torch.cuda.synchronize()
    assert torch.equal(b1, b2)


def test_row_shards_of_a_wide_tall_matrix_equal_the_unsharded_solve():
    # 256 x 1,310,720: alone it makes more than 8 waves of column-pass tiles,
    # so its tiles take at least 64 rows per warp (a "tall" geometry);
    # dq_col_row_block and the step entry points take the same choice as
    # the unsharded solve, and the two-shard solve stays bit-identical.
    from dual_scale_solver_b200 import sharded
    fl = lib_format("int4_bf16", 64)
    rows, cols, T = 256, 1310720, 2
    W = _weights(rows, cols, key=5)
    rb = dq.col_row_block(rows, cols)
    assert rb == 64                                     # 64 rows per warp, 1 warp row
    starts = [0, 128, rows]
    shards = [sharded.RowShard(W[s0:s1], s0, rows, fl) for s0, s1 in zip(starts, starts[1:])]
    b = torch.ones(cols, device="cuda")
    for _ in range(T):
        for sh in shards:
            sh.row_step(b)
        parts = torch.cat([sh.col_partials(b)[0] for sh in shards])
        b = shards[0].col_finalize(parts)
    o = dq.solve_dual_scale(W, fl, T)
    torch.cuda.synchronize()
    assert dq.last_device_status() == 0
    assert torch.equal(torch.cat([sh.a for sh in shards]), o["a"])
    assert torch.equal(b, o["b"])
