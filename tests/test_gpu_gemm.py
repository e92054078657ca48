"""Block-scaled W4A4 GEMM on the tensor cores against the oracle's float64
product of the decoded operands (eq. (1) of the daiwk note: X W^T ~= (X D_b)
Qhat^T D_a), in MXFP4 (E8M0 scales per 32) and NVFP4 (E4M3 scales per 16
and the weights' tensor scale; news article, "适配 MXFP4 与 NVFP4 块结构").

Bar: the products of E2M1 codes and E8M0 or E4M3 scales are exact in
float32 (at most 2 + 4 significant bits per operand), so the only error is
the float32 accumulation over K terms and the final scaling:
|gpu - ref| <= (K + 1) 2^-24 sum_k |x_k w_k| |a_n| ts for every element."""
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


# --------------------------------------------------------------------------- #
# NVFP4: E4M3 scales per 16 elements, the weights' tensor scale
# --------------------------------------------------------------------------- #

FNV = O.preset("nvfp4")


def _random_operand_nv(rows, K, key):
    # E4M3 scales between 2^-3 and 2^3 (bytes 0x20 .. 0x57, sign bit clear)
    g = torch.Generator().manual_seed(key)
    codes = torch.randint(0, 256, (rows, K // 2), generator=g, dtype=torch.uint8)
    scales = torch.randint(0x20, 0x58, (rows, K // 16), generator=g, dtype=torch.uint8)
    return codes, scales


def _reference_nv(cx, sx, cw, sw, a, ts, rows=None):
    cxn, sxn = cx.cpu().numpy(), sx.cpu().numpy()
    if rows is not None:
        cxn, sxn = cxn[rows], sxn[rows]
    x_c, x_s = O.decode_codes(cxn, FNV), O.decode_scales(sxn, FNV)
    w_c, w_s = O.decode_codes(cw.cpu().numpy(), FNV), O.decode_scales(sw.cpu().numpy(), FNV)
    an = np64(a)
    ref = O.w4a4_gemm(x_c, x_s, w_c, w_s, an, FNV, ts)
    absx = np.abs(O.dequantize(x_c, x_s, FNV))
    absw = np.abs(O.dequantize(w_c, w_s, FNV, ts))
    K = x_c.shape[1]
    bound = (K + 1) * 2.0 ** -24 * (absx @ absw.T) * np.abs(an)[None, :]
    return ref, bound


@pytest.mark.parametrize("M,N,K", [(128, 128, 256), (256, 384, 1024), (384, 256, 2048),
                                   (256, 256, 256), (512, 768, 1024), (768, 512, 2048)])
def test_w4a4_gemm_nvfp4_random_operands(M, N, K):
    cx, sx = _random_operand_nv(M, K, 61 + M)
    cw, sw = _random_operand_nv(N, K, 62 + N)
    a = torch.tensor(np.ldexp(1.0, np.random.default_rng(K).integers(-3, 4, N)), dtype=torch.float32)
    ts = 2.0 ** -9
    tsd = torch.tensor([ts], dtype=torch.float32, device="cuda")
    fl = dq.format_preset("nvfp4")
    out = dq.w4a4_gemm(cx.cuda(), sx.cuda(), cw.cuda(), sw.cuda(), a.cuda(), fl, tensor_scale=tsd)
    torch.cuda.synchronize()
    assert dq.last_device_status() == 0
    ref, bound = _reference_nv(cx, sx, cw, sw, a, ts)
    err = np.abs(np64(out) - ref)
    assert np.all(err <= bound), (err.max(), np.unravel_index(np.argmax(err - bound), err.shape))


@pytest.mark.parametrize("M,N", [(128, 128), (256, 256)])         # single CTA, CTA pair
def test_w4a4_gemm_nvfp4_block_placement(M, N):
    # Scales apply per 16 elements of K: x[5, 200] = 1 with its block's scale
    # 2 and w[9, 200] = 6 with its block's scale 1.5 (block 12 of 16), then
    # x[5, 216] = 1.5 and w[9, 216] = 1 in block 13 with scale 1; a_9 = 2,
    # ts = 1/4: out[5, 9] = (1*2*6*1.5 + 1.5*1) * 2 / 4 = 9.75.  (Scales read
    # per 32 elements would give 3.75.)  Row M-1 of x and row N-1 of w repeat
    # the pattern (with a_{N-1} = 2), so the four crossings are 9.75 and the
    # rest 0; row M-1 and column N-1 live in the second CTA of a pair.
    K = 512
    cx = torch.zeros(M, K // 2, dtype=torch.uint8)
    sx = torch.full((M, K // 16), 0x38, dtype=torch.uint8)        # E4M3 1.0
    cw = torch.zeros(N, K // 2, dtype=torch.uint8)
    sw = torch.full((N, K // 16), 0x38, dtype=torch.uint8)
    for m, n in [(5, 9), (M - 1, N - 1)]:
        cx[m, 100] = 0x02                                 # x[m, 200] = 1.0
        sx[m, 12] = 0x40                                  # 2.0
        cw[n, 100] = 0x07                                 # w[n, 200] = 6.0
        sw[n, 12] = 0x3C                                  # 1.5
        cx[m, 108] = 0x03                                 # x[m, 216] = 1.5
        cw[n, 108] = 0x02                                 # w[n, 216] = 1.0
    a = torch.ones(N)
    a[9] = 2.0
    a[N - 1] = 2.0
    tsd = torch.tensor([0.25], device="cuda")
    out = dq.w4a4_gemm(cx.cuda(), sx.cuda(), cw.cuda(), sw.cuda(), a.cuda(),
                       dq.format_preset("nvfp4"), tensor_scale=tsd).cpu()
    want = torch.zeros(M, N)
    for m in (5, M - 1):
        for n in (9, N - 1):
            want[m, n] = 9.75
    assert torch.equal(out, want)


@pytest.mark.parametrize("rows,K", [(128, 64), (384, 1024)])
def test_scale_tiles_layout_group16(rows, K):
    _, S = _random_operand_nv(rows, K, 70 + rows)
    t = dq.scale_tiles(S.cuda(), K, group=16).cpu().numpy()
    assert np.array_equal(t, _tiles_expected(S.numpy()))


def test_w4a4_gemm_nvfp4_after_solve_and_activation_quant():
    # the NVFP4 pipeline: solve W (E4M3 group scales with the tensor scale),
    # quantize X D_b to NVFP4 (tensor scale 1), multiply
    wl = synth.WORKLOADS["llama31_8b_nvfp4_g16"]
    fl = dq.format_preset("nvfp4")
    W = synth.weight(wl, 0, 1, device="cuda", rows=512, cols=2048)
    o = dq.solve_dual_scale(W, fl, 5)
    X = synth.activation(wl, device="cuda", tokens=256)[:, :2048].contiguous()
    cx, sx = dq.act_rescale_quant(X, o["b"], fl)
    out = dq.w4a4_gemm(cx, sx, o["codes"], o["gscales"], o["a"], fl,
                       tensor_scale=o["tensor_scale"])
    torch.cuda.synchronize()
    assert dq.last_device_status() == 0
    ts = float(o["tensor_scale"].item())
    assert ts != 1.0
    ref, bound = _reference_nv(cx, sx, o["codes"], o["gscales"], o["a"], ts)
    assert np.all(np.abs(np64(out) - ref) <= bound)
    exact = np64(X) @ np64(W).T
    assert np.linalg.norm(np64(out) - exact) < 0.35 * np.linalg.norm(exact)
