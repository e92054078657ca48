"""The C-ABI library loads, exports every symbol include/dq.h declares, and
validates arguments on the host (no kernel launches; runs without a GPU)."""
import ctypes
import os
import re

import pytest

import dual_scale_solver_b200 as dq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "dq.h")).read()
    return sorted(set(re.findall(r"^DQ_API\s+[^(]*?\b(dq_\w+)\s*\(", src, flags=re.M)))


@pytest.fixture(scope="module", autouse=True)
def built():
    from dual_scale_solver_b200 import build
    build.build()


def test_exports_match_header():
    names = _declared()
    assert len(names) == 29
    assert sorted(dq.EXPORTS) == names
    L = dq.lib()
    for n in names:
        assert hasattr(L, n), n


def test_version_and_errors():
    assert "sm_100a" in dq.version()
    assert dq.lib().dq_strerror(-2).decode().startswith("invalid shape")


@pytest.mark.parametrize("name,codes,gs,os_,G,auto", [
    ("int4_bf16", 0, 0, 0, 64, 0), ("mxint4", 0, 1, 1, 32, 0),
    ("mxfp4", 1, 1, 1, 32, 0), ("nvfp4", 1, 2, 0, 16, 1),
    ("mxint8", 2, 1, 1, 32, 0), ("mxfp8_e4m3", 3, 1, 1, 32, 0), ("mxfp8_e5m2", 4, 1, 1, 32, 0),
    ("mxfp6_e2m3", 5, 1, 1, 32, 0), ("mxfp6_e3m2", 6, 1, 1, 32, 0),
    ("mxint4_bf16outer", 0, 1, 0, 32, 0), ("mxfp4_bf16outer", 1, 1, 0, 32, 0)])
def test_presets(name, codes, gs, os_, G, auto):
    f = dq.format_preset(name)
    assert (f.codes, f.group_scale, f.outer_scale, f.group, f.tensor_scale_auto) == (codes, gs, os_, G, auto)
    assert dq.format_preset(name, 32).group == 32


@pytest.mark.parametrize("name,per_row", [
    ("int4_bf16", 32), ("mxfp4", 32), ("nvfp4", 32), ("mxint8", 64), ("mxfp8_e4m3", 64),
    ("mxfp8_e5m2", 64), ("mxfp6_e2m3", 48), ("mxfp6_e3m2", 48)])
def test_code_bytes(name, per_row):
    # 64 columns: 4-bit codes 32 bytes, 8-bit 64, 6-bit 48 (four codes per 3 bytes)
    f = dq.format_preset(name)
    assert dq.code_bytes(f, 3, 64) == 3 * per_row
    assert dq.lib().dq_code_bytes(ctypes.byref(f), 3, 65) == -1
    # the float element formats need E8M0 group and outer scales
    bad = dq.dq_format(f.codes, 32, 0, 0, 0)
    if f.codes >= 2:
        assert dq.lib().dq_code_bytes(ctypes.byref(bad), 3, 64) == -1


def test_bad_preset_and_group():
    with pytest.raises(dq.DqError) as e:
        dq.format_preset("fp8")
    assert e.value.status == -3
    with pytest.raises(dq.DqError):
        dq.format_preset("mxfp4", 48)


def test_workspace_size_and_shape_checks():
    f = dq.format_preset("mxfp4")
    n1 = dq.workspace_size([(8192, 8192)], f)
    n2 = dq.workspace_size([(8192, 8192), (1024, 8192)], f)
    assert 0 < n1 < n2
    # per-tile column partials stay small next to the matrix (8 B per column
    # per 128-row tile: 1/32 of its bf16 bytes, plus row partials)
    assert n1 < 0.04 * 8192 * 8192 * 2
    with pytest.raises(dq.DqError) as e:
        dq.workspace_size([(16, 40)], f)            # 40 % 32 != 0
    assert e.value.status == -2
    assert dq.workspace_size([], f) > 0 or dq.workspace_size([], f) == 256


def test_host_side_argument_errors():
    L = dq.lib()
    f = dq.format_preset("int4_bf16")
    bad = dq.dq_format(0, 48, 0, 0, 0)
    # bad format, shape and missing pointers are refused before any launch
    assert L.dq_quantize(None, 1, 4, 64, ctypes.byref(bad), None, None, 1.0, None, None, None) == -3
    assert L.dq_quantize(None, 1, 4, 65, ctypes.byref(f), None, None, 1.0, None, None, None) == -2
    assert L.dq_quantize(None, 1, 4, 64, ctypes.byref(f), None, None, 1.0, None, None, None) == -1
    assert L.dq_quantize(None, 7, 4, 64, ctypes.byref(f), None, None, 1.0, None, None, None) == -1
    # misaligned input pointer
    assert L.dq_quantize(ctypes.c_void_p(8), 1, 4, 64, ctypes.byref(f), None, None, 1.0,
                         ctypes.c_void_p(16), ctypes.c_void_p(16), None) == -9
    # empty shapes are valid no-ops
    assert L.dq_quantize(None, 1, 0, 64, ctypes.byref(f), None, None, 1.0, None, None, None) == 0
    # a solve without workspace
    assert L.dq_solve_dual_scale(ctypes.c_void_p(256), 1, 4, 64, ctypes.byref(f), 3, None, None,
                                 ctypes.c_void_p(256), ctypes.c_void_p(256), ctypes.c_void_p(256),
                                 ctypes.c_void_p(256), ctypes.c_void_p(256), None, None, None, 0,
                                 None) == -7
    # tensor_scale_auto only with E4M3 group scales
    assert L.dq_workspace_size(0, None, None, ctypes.byref(dq.dq_format(1, 32, 1, 1, 1)),
                               ctypes.byref(ctypes.c_size_t())) == -3
    assert L.dq_solve_dual_scale_batched(-1, None, 1, ctypes.byref(f), 1, None, 0, None) == -1


def test_two_level_argument_errors():
    L = dq.lib()
    f = dq.format_preset("mxfp4")
    nv = dq.format_preset("nvfp4")
    args = lambda fmt, D, cols: (None, 1, 4, cols, D, ctypes.byref(fmt), None, None, None, None, None)
    assert L.dq_two_level_quant(*args(nv, 512, 64)) == -3          # inner must be MXFP4
    assert L.dq_two_level_quant(*args(f, 384, 64)) == -1           # block size
    assert L.dq_two_level_quant(*args(f, 512, 48)) == -2           # cols % 32
    assert L.dq_two_level_quant(*args(f, 512, 64)) == -1           # null pointers
    assert L.dq_two_level_quant(None, 1, 0, 64, 512, ctypes.byref(f), None, None, None, None,
                                None) == 0                         # empty: nothing to do


def test_w4a4_gemm_argument_errors():
    L = dq.lib()
    f = dq.format_preset("mxfp4")
    nv = dq.format_preset("nvfp4")
    mxi = dq.format_preset("mxint4")
    nv32 = dq.format_preset("nvfp4", 32)
    args = lambda fmt, M, N, K: (None, None, None, None, None, None, M, N, K, ctypes.byref(fmt),
                                 None, None)
    assert L.dq_w4a4_gemm(*args(mxi, 128, 128, 256)) == -3         # E2M1 codes only
    assert L.dq_w4a4_gemm(*args(nv32, 128, 128, 256)) == -3        # NVFP4 blocks of 16 only
    assert L.dq_w4a4_gemm(*args(f, 100, 128, 256)) == -2           # M % 128
    assert L.dq_w4a4_gemm(*args(nv, 128, 128, 320)) == -2          # K % 256
    assert L.dq_w4a4_gemm(*args(f, 128, 128, 256)) == -1           # null pointers
    assert L.dq_w4a4_gemm(*args(nv, 128, 128, 256)) == -1
    assert L.dq_w4a4_gemm(*args(f, 0, 128, 256)) == 0              # empty
    p = ctypes.c_void_p(256)                                       # never dereferenced
    assert L.dq_w4a4_gemm(p, p, p, p, p, ctypes.c_void_p(258), 128, 128, 256, ctypes.byref(nv),
                          p, None) == -9                           # tensor_scale alignment


def test_scale_tiles_argument_errors():
    L = dq.lib()
    assert L.dq_scale_tiles(None, 100, 256, 32, None, None) == -2   # rows % 128
    assert L.dq_scale_tiles(None, 128, 96, 32, None, None) == -2    # K % 128
    assert L.dq_scale_tiles(None, 128, 96, 16, None, None) == -2    # K % 64
    assert L.dq_scale_tiles(None, 128, 256, 64, None, None) == -1   # G 16 or 32 only
    assert L.dq_scale_tiles(None, 128, 256, 32, None, None) == -1   # null pointers
    assert L.dq_scale_tiles(None, 0, 256, 16, None, None) == 0      # empty
    assert L.dq_scale_tiles(ctypes.c_void_p(16), 128, 128, 32, ctypes.c_void_p(24),
                            None) == -9                             # alignment


def test_host_solve_argument_errors():
    L = dq.lib()
    f = dq.format_preset("mxfp4")
    h, d = (dq.dq_matrix * 1)(), (dq.dq_matrix * 1)()
    h[0].rows, h[0].cols, d[0].rows, d[0].cols = 4, 64, 4, 64
    call = lambda n, fmt, hh, dd: L.dq_solve_dual_scale_batched_host(n, hh, dd, 1, ctypes.byref(fmt),
                                                                     3, None, 0, None, None, None)
    assert call(-1, f, h, d) == -1                                  # n < 0
    assert call(0, f, h, d) == 0                                    # nothing to do
    d[0].cols = 96
    assert call(1, f, h, d) == -2                                   # host / device shapes differ
    d[0].cols = 64
    assert call(1, f, h, d) == -1                                   # no W
    bad = dq.dq_format(9, 32, 1, 1, 0)
    assert call(1, bad, h, d) == -3                                 # format


def test_graph_argument_errors():
    # dq_graph_solve_batched checks its arguments before any CUDA call
    L = dq.lib()
    f = dq.format_preset("mxfp4")
    m = (dq.dq_matrix * 1)()
    m[0].rows, m[0].cols = 4, 64
    h = ctypes.c_void_p(123)
    call = lambda n, fmt, mm, out: L.dq_graph_solve_batched(n, mm, 1, ctypes.byref(fmt), 3, None, 0, out)
    assert call(1, f, m, None) == -1                                # no out
    assert call(0, f, m, ctypes.byref(h)) == -1 and h.value is None  # empty batch; *out cleared
    assert call(-1, f, m, ctypes.byref(h)) == -1                    # n < 0
    assert call(1, f, m, ctypes.byref(h)) == -1                     # no W
    bad = dq.dq_format(9, 32, 1, 1, 0)
    assert call(1, bad, m, ctypes.byref(h)) == -3                   # format
    m[0].cols = 48
    assert call(1, f, m, ctypes.byref(h)) == -2                     # cols % G
    assert L.dq_graph_launch(None, None) == -1                      # no graph
    assert L.dq_graph_launches(None) == 0
    assert L.dq_graph_destroy(None) == 0                            # no-op


def test_sharded_column_entry_points_argument_errors():
    L = dq.lib()
    f = dq.format_preset("int4_bf16")
    assert L.dq_col_row_block(-1, 64, 1) == -1
    assert L.dq_col_row_block(64, 64, 7) == -1
    assert L.dq_col_row_block(14336, 4096, 1) == 256        # 256 rows per warp, 1 warp row
    # a matrix whose column pass alone makes 8 waves of tiles takes at least
    # 64 rows per warp (the "tall" geometry); a smaller one 16
    assert L.dq_col_row_block(256, 1310720, 1) == 64         # 1 warp row, 64 rows per warp
    assert L.dq_col_row_block(1536, 2240, 1) == 128          # 8 warp rows, 16 rows per warp
    assert L.dq_col_row_block(100, 4096, 1) % 1 == 0 and L.dq_col_row_block(100, 4096, 1) > 0
    p = ctypes.c_void_p(256)                                 # never dereferenced
    ws = ctypes.c_void_p(1 << 20)
    # row block not a multiple of the warp rows / too large / null partials
    assert L.dq_col_partials(p, 1, 64, 100 * 64, ctypes.byref(f), 1.0, p, p, 0, p, None, ws,
                             1 << 30, None) == -2
    assert L.dq_col_partials(p, 1, 64, 64, ctypes.byref(f), 1.0, p, p, 3, p, None, ws,
                             1 << 30, None) == -2
    assert L.dq_col_partials(p, 1, 64, 64, ctypes.byref(f), 1.0, p, p, 64, None, None, ws,
                             1 << 30, None) == -1
    assert L.dq_col_partials(p, 1, 64, 64, ctypes.byref(f), 2.0, p, p, 64, p, None, ws,
                             1 << 30, None) == -1              # ts != 1 without a tensor scale
    assert L.dq_col_row_block(64, 64, 1) == 128              # 16 rows per warp, 8 warp rows
    assert L.dq_col_partials(p, 1, 64, 64, ctypes.byref(f), 1.0, p, p, 64, p, None, ws,
                             1 << 30, None) == -2              # below the shard's own row block
    assert L.dq_col_partials(p, 1, 64, 64, ctypes.byref(f), 1.0, p, p, 128, p, None, None,
                             0, None) == -7                    # workspace
    # finalize: columns not a multiple of the group size, null output
    assert L.dq_col_finalize(p, 4, 63, ctypes.byref(f), p, None, None) == -2
    assert L.dq_col_finalize(p, 4, 66, ctypes.byref(f), p, None, None) == -2
    assert L.dq_col_finalize(p, 4, 64, ctypes.byref(f), None, None, None) == -1
    assert L.dq_col_finalize(None, 0, 0, ctypes.byref(f), None, None, None) == 0
