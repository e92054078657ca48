"""The batched solve captured as a CUDA graph (dq_graph_solve_batched):
replays give the same bits as direct calls."""
import pytest
import torch

import dual_scale_solver_b200 as dq
import synth

pytestmark = pytest.mark.gpu

KEYS = ("codes", "gscales", "a", "b", "tensor_scale", "mse_trace")


def _weights(name, shapes, seed=0):
    wl = synth.WORKLOADS[name]
    return [synth.weight(wl, seed, i, device="cuda", rows=r, cols=c) for i, (r, c) in enumerate(shapes)]


def _same(o, r, half=False):
    for k in KEYS + (("mse_half",) if half else ()):
        assert torch.equal(o[k], r[k]), k


@pytest.mark.parametrize("name, fmt, shapes", [
    ("llama31_70b_decoder_mxfp4_g32", "mxfp4", [(512, 1024), (96, 2048), (300, 512)]),
    ("llama31_8b_nvfp4_g16", "nvfp4", [(256, 512), (64, 1024)]),
    ("llama31_8b_int4_g64", "int4_bf16", [(300, 2240)]),
])
def test_graph_replay_equals_direct_solve(name, fmt, shapes):
    fl = dq.format_preset(fmt, 0)
    Ws = _weights(name, shapes)
    T = 4
    g = dq.solve_dual_scale_batched_graph(Ws, fl, T, half=True)
    before = dq.launch_count()
    g.launch()
    torch.cuda.synchronize()
    assert dq.launch_count() - before == g.launches > 0
    ref = dq.solve_dual_scale_batched(Ws, fl, T, half=True)
    torch.cuda.synchronize()
    for o, r in zip(g.outs, ref):
        _same(o, r, half=True)
    g.close()


def test_graph_reads_the_weights_at_replay_time():
    fl = dq.format_preset("mxfp4")
    shapes = [(256, 1024), (128, 2048)]
    Ws = _weights("llama31_70b_decoder_mxfp4_g32", shapes, seed=0)
    g = dq.solve_dual_scale_batched_graph(Ws, fl, 3)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        g.launch(stream=s)
        first = [{k: v.clone() for k, v in o.items() if v is not None} for o in g.outs]
        new = _weights("llama31_70b_decoder_mxfp4_g32", shapes, seed=1)
        for W, N in zip(Ws, new):
            W.copy_(N)
        g.launch(stream=s)
    s.synchronize()
    ref = dq.solve_dual_scale_batched(new, fl, 3)
    torch.cuda.synchronize()
    for o, r, f in zip(g.outs, ref, first):
        _same(o, r)
        assert not torch.equal(o["codes"], f["codes"])
    g.close()


def test_graph_uploads_its_table_on_every_replay():
    # another batched solve in the same workspace overwrites the work table;
    # the next replay still solves the graph's own matrices
    fl = dq.format_preset("mxint4")
    A = _weights("smollm2_135m_mxint4_g32", [(576, 576), (192, 576), (1536, 576)])
    B = _weights("smollm2_135m_mxint4_g32", [(576, 1536), (576, 576)], seed=3)
    shapes = [tuple(W.shape) for W in A] + [tuple(W.shape) for W in B]
    ws = dq.workspace(shapes, fl, "cuda")
    g = dq.solve_dual_scale_batched_graph(A, fl, 5, ws=ws)
    g.launch()
    dq.solve_dual_scale_batched(B, fl, 5, ws=ws)
    g.launch()
    torch.cuda.synchronize()
    ref = dq.solve_dual_scale_batched(A, fl, 5)
    torch.cuda.synchronize()
    for o, r in zip(g.outs, ref):
        _same(o, r)
    g.close()
    g.close()                                    # closing twice is harmless
    with pytest.raises(dq.DqError):
        g.launch()


def test_graph_rejects_bad_arguments_without_capturing():
    fl = dq.format_preset("mxfp4")
    W = _weights("llama31_70b_decoder_mxfp4_g32", [(64, 96)])   # 96 % 32 == 0
    ok = dq.solve_dual_scale_batched_graph(W, fl, 1)
    ok.close()
    bad = torch.zeros(64, 80, dtype=torch.bfloat16, device="cuda")  # 80 % 32 != 0
    with pytest.raises(dq.DqError):
        dq.solve_dual_scale_batched_graph([bad], fl, 1, ws=torch.empty(1 << 20, dtype=torch.uint8,
                                                                        device="cuda"),
                                          outs=[dict(codes=torch.empty(64 * 40, dtype=torch.uint8, device="cuda"),
                                                     gscales=torch.empty(64 * 3, dtype=torch.uint8, device="cuda"),
                                                     a=torch.empty(64, device="cuda"),
                                                     b=torch.empty(80, device="cuda"),
                                                     tensor_scale=torch.empty(1, device="cuda"),
                                                     mse_trace=torch.empty(2, dtype=torch.float64, device="cuda"))])
    # the stream and the library are still usable
    o = dq.solve_dual_scale_batched(W, fl, 1)
    torch.cuda.synchronize()
    assert dq.last_device_status() == 0
    assert o[0]["codes"].numel() > 0
