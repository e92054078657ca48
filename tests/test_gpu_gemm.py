"""Block-scaled W4A4 GEMM on the tensor cores against the oracle's float64
product of the decoded operands (eq. (1) of the daiwk note: X W^T ~= (X D_b)
Qhat^T D_a).

Bar: the products of E2M1 codes and E8M0 scales are exact in float32, so the
only error is the float32 accumulation over K terms and the final scaling:
|gpu - ref| <= (K + 1) 2^-24 sum_k |x_k w_k| |a_n| for every element."""
import numpy as np
import pytest
import torch

import oracle as O
import synth
from _helpers import np64

pytestmark = pytest.mark.gpu

dq = pytest.importorskip("dual_scale_solver_b200")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from dual_scale_solver_b200 import build
    build.build()


FO = O.preset("mxfp4")


def _random_operand(rows, K, key, e_lo=118, e_hi=134):
    g = torch.Generator().manual_seed(key)
    codes = torch.randint(0, 256, (rows, K // 2), generator=g, dtype=torch.uint8)
    scales = torch.randint(e_lo, e_hi, (rows, K // 32), generator=g, dtype=torch.uint8)
    return codes, scales


def _reference(cx, sx, cw, sw, a, rows=None):
    """Oracle product (float64) and the per-element error bound, optionally on
    a subset of output rows."""
    cxn, sxn = cx.cpu().numpy(), sx.cpu().numpy()
    if rows is not None:
        cxn, sxn = cxn[rows], sxn[rows]
    x_c, x_s = O.decode_codes(cxn, FO), O.decode_scales(sxn, FO)
    w_c, w_s = O.decode_codes(cw.cpu().numpy(), FO), O.decode_scales(sw.cpu().numpy(), FO)
    an = np64(a)
    ref = O.w4a4_gemm(x_c, x_s, w_c, w_s, an, FO)
    absx = np.abs(O.dequantize(x_c, x_s, FO))
    absw = np.abs(O.dequantize(w_c, w_s, FO))
    K = x_c.shape[1]
    bound = (K + 1) * 2.0 ** -24 * (absx @ absw.T) * np.abs(an)[None, :]
    return ref, bound


# (256, 256, 256), (512, 768, 1024), (768, 512, 2048): CTA pairs on 256 x 256
# tiles; (128, 128, 256), (384, 256, 2048): one CTA per 128 x 256 tile;
# (256, 384, 1024): 128 x 128 tiles
@pytest.mark.parametrize("M,N,K", [(128, 128, 256), (256, 384, 1024), (384, 256, 2048),
                                   (256, 256, 256), (512, 768, 1024), (768, 512, 2048)])
def test_w4a4_gemm_random_operands(M, N, K):
    cx, sx = _random_operand(M, K, 1 + M)
    cw, sw = _random_operand(N, K, 2 + N)
    a = torch.tensor(np.ldexp(1.0, np.random.default_rng(K).integers(-3, 4, N)), dtype=torch.float32)
    out = dq.w4a4_gemm(cx.cuda(), sx.cuda(), cw.cuda(), sw.cuda(), a.cuda())
    torch.cuda.synchronize()
    assert dq.last_device_status() == 0
    ref, bound = _reference(cx, sx, cw, sw, a)
    err = np.abs(np64(out) - ref)
    assert np.all(err <= bound), (err.max(), np.unravel_index(np.argmax(err - bound), err.shape))


def test_w4a4_gemm_zero_and_single_code():
    M, N, K = 128, 128, 512
    cx = torch.zeros(M, K // 2, dtype=torch.uint8)
    sx = torch.full((M, K // 32), 127, dtype=torch.uint8)
    cw = torch.zeros(N, K // 2, dtype=torch.uint8)
    sw = torch.full((N, K // 32), 127, dtype=torch.uint8)
    cx[5, 100] = 0x02                                   # x[5, 200] = 1.0 (E2M1 code 2)
    cw[7, 100] = 0x70                                   # w[7, 201] = 6.0 (high nibble)
    cw[9, 100] = 0x07                                   # w[9, 200] = 6.0
    a = torch.ones(N)
    out = dq.w4a4_gemm(cx.cuda(), sx.cuda(), cw.cuda(), sw.cuda(), a.cuda()).cpu()
    want = torch.zeros(M, N)
    want[5, 9] = 6.0
    assert torch.equal(out, want)


def test_w4a4_gemm_after_solve_and_activation_quant():
    # the pipeline the pages describe: solve W, quantize X D_b, multiply
    wl = synth.WORKLOADS["llama31_70b_decoder_mxfp4_g32"]
    fl = dq.format_preset("mxfp4")
    W = synth.weight(wl, 0, 1, device="cuda", rows=512, cols=2048)        # k_proj-like
    o = dq.solve_dual_scale(W, fl, 5)
    X = synth.activation(wl, device="cuda", tokens=256)[:, :2048].contiguous()
    cx, sx = dq.act_rescale_quant(X, o["b"], fl)
    out = dq.w4a4_gemm(cx, sx, o["codes"], o["gscales"], o["a"])
    torch.cuda.synchronize()
    assert dq.last_device_status() == 0
    ref, bound = _reference(cx, sx, o["codes"], o["gscales"], o["a"])
    assert np.all(np.abs(np64(out) - ref) <= bound)
    # and the W4A4 product is the quantized model of X W^T (activations with
    # outlier channels x30: about a quarter of the norm is quantization error)
    exact = np64(X) @ np64(W).T
    assert np.linalg.norm(np64(out) - exact) < 0.35 * np.linalg.norm(exact)


def test_w4a4_gemm_large_k_sampled_rows():
    M, N, K = 512, 1024, 8192
    cx, sx = _random_operand(M, K, 11)
    cw, sw = _random_operand(N, K, 12)
    a = torch.ones(N)
    out = dq.w4a4_gemm(cx.cuda(), sx.cuda(), cw.cuda(), sw.cuda(), a.cuda())
    torch.cuda.synchronize()
    rows = np.sort(synth.distinct_indices(synth.stream_key(88, M), M, 24).numpy())
    ref, bound = _reference(cx, sx, cw, sw, a, rows=rows)
    assert np.all(np.abs(np64(out)[rows] - ref) <= bound)


def _tiles_expected(S):
    """Scale tiles written out from their definition: chunk (row block rb, K
    block kc) of 512 bytes, scale k of row r at (r % 32) * 16 + (r // 32) * 4 + k."""
    rows, nk = S.shape
    out = np.zeros((rows // 128, nk // 4, 512), dtype=np.uint8)
    for rb in range(rows // 128):
        for kc in range(nk // 4):
            for r in range(128):
                for k in range(4):
                    out[rb, kc, (r % 32) * 16 + (r // 32) * 4 + k] = S[rb * 128 + r, 4 * kc + k]
    return out.reshape(-1)


@pytest.mark.parametrize("rows,K", [(128, 128), (384, 1024)])
def test_scale_tiles_layout(rows, K):
    _, S = _random_operand(rows, K, 40 + rows, e_lo=0, e_hi=256)
    t = dq.scale_tiles(S.cuda(), K).cpu().numpy()
    assert np.array_equal(t, _tiles_expected(S.numpy()))


def test_w4a4_gemm_pretiled_scales_equal_row_major():
    M, N, K = 256, 512, 1024
    cx, sx = _random_operand(M, K, 31)
    cw, sw = _random_operand(N, K, 32)
    a = torch.ones(N).cuda()
    cx, sx, cw, sw = cx.cuda(), sx.cuda(), cw.cuda(), sw.cuda()
    y0 = dq.w4a4_gemm(cx, sx, cw, sw, a)
    y1 = dq.w4a4_gemm(cx, dq.scale_tiles(sx), cw, dq.scale_tiles(sw), a, tiled=True)
    torch.cuda.synchronize()
    assert dq.last_device_status() == 0
    assert torch.equal(y0, y1)


def test_w4a4_gemm_pair_tile_placement():
    # a 256 x 256 tile is split over two CTAs: rows 128..255 of the output and
    # rows 128..255 of the weights live in the second one
    M, N, K = 256, 256, 512
    cx = torch.zeros(M, K // 2, dtype=torch.uint8)
    sx = torch.full((M, K // 32), 127, dtype=torch.uint8)
    cw = torch.zeros(N, K // 2, dtype=torch.uint8)
    sw = torch.full((N, K // 32), 127, dtype=torch.uint8)
    cx[200, 150] = 0x02                                 # x[200, 300] = 1.0
    sx[200, 9] = 128                                    # its group scale 2
    cw[130, 150] = 0x07                                 # w[130, 300] = 6.0
    cx[5, 100] = 0x02                                   # x[5, 200] = 1.0
    cw[250, 100] = 0x06                                 # w[250, 200] = 4.0
    a = torch.ones(N)
    a[250] = 0.5
    out = dq.w4a4_gemm(cx.cuda(), sx.cuda(), cw.cuda(), sw.cuda(), a.cuda()).cpu()
    want = torch.zeros(M, N)
    want[200, 130] = 12.0
    want[5, 250] = 2.0
    assert torch.equal(out, want)


@pytest.mark.parametrize("M,N", [(256, 256), (128, 128)])       # CTA pair, single CTA
def test_w4a4_gemm_stalled_pipeline_reports_timeout(M, N):
    # the producer leaves the first K tile unloaded: the MMA thread's bounded
    # wait runs out, the kernel returns and raises the timeout flag; the
    # context stays usable
    K = 512
    cx, sx = _random_operand(M, K, 51)
    cw, sw = _random_operand(N, K, 52)
    a = torch.ones(N)
    args = (cx.cuda(), sx.cuda(), cw.cuda(), sw.cuda(), a.cuda())
    assert dq.last_device_status() == 0
    dq.lib().dq_test_stall_next_gemm()
    dq.w4a4_gemm(*args)
    assert dq.last_device_status() == -11
    out = dq.w4a4_gemm(*args)
    torch.cuda.synchronize()
    assert dq.last_device_status() == 0
    ref, bound = _reference(cx, sx, cw, sw, a)
    assert np.all(np.abs(np64(out) - ref) <= bound)
