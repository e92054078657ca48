"""fp64 CPU oracle of the DualQuant dual-scale solver.

TEST INFRASTRUCTURE ONLY.  This package restates the method from the DualQuant
pages in plain numpy float64 so that the CUDA library can be checked against
it.  It shares no code with the library, and the library never imports it:
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may use it.

Every function carries a ``parity`` status in the test suite; all of them are
pinned by the tests listed in the design notes (closed forms, brute force,
library casts, hand-derived cases).
"""
from .formats import *          # noqa: F401,F403
from .solver import (Format, PRESETS, QMAX, CODE_BITS, preset, project_group_scale, project_outer,  # noqa: F401
                     round_codes, tensor_scale, quantize, dequantize, inner, qhat, mse,
                     row_update, col_update, solve, act_rescale_quant, encode_codes,
                     encode_scales, decode_codes, decode_scales, two_level_quant,
                     MXFP4_MAX_NORMAL, w4a4_gemm)
