"""The oracle's and the library's constants against the values the DualQuant
pages print (tests/golden/page_constants.txt, each line with its source).
No GPU."""
import os

import numpy as np

import oracle as O
import synth

HERE = os.path.dirname(os.path.abspath(__file__))


def _golden():
    out = {}
    for line in open(os.path.join(HERE, "golden", "page_constants.txt")):
        line = line.split("#")[0].strip()
        if line:
            k, v = (x.strip() for x in line.split("="))
            out[k] = float(v)
    return out


G = _golden()


def test_int4_codebook():
    q = np.arange(-20, 21, 0.5)
    c = O.round_int4(q)
    assert c.min() == G["int4_codebook_min"] and c.max() == G["int4_codebook_max"]
    assert O.preset("mxint4").qmax == G["int4_codebook_max"]


def test_e8m0_exponent_range():
    lo, hi = int(G["e8m0_exponent_min"]), int(G["e8m0_exponent_max"])
    assert O.e8m0_ceil(np.array([2.0 ** -140]))[0] == 2.0 ** lo
    assert O.e8m0_ceil(np.array([2.0 ** 140]))[0] == 2.0 ** hi
    assert O.e8m0_nearest(np.array([2.0 ** -140, 2.0 ** 140])).tolist() == [2.0 ** lo, 2.0 ** hi]
    assert O.decode_e8m0(O.encode_e8m0(np.array([2.0 ** lo, 2.0 ** hi]))).tolist() == [2.0 ** lo, 2.0 ** hi]


def test_block_sizes_and_defaults():
    assert O.preset("mxfp4").group == G["mxfp4_block"]
    assert O.preset("mxint4").group == G["column_group"]
    assert O.preset("nvfp4").group == G["nvfp4_block"]
    assert (O.preset("nvfp4").gscale, O.preset("mxfp4").gscale) == ("e4m3", "e8m0")
    assert synth.BASE_SEED == G["seed"]
    toy = synth.WORKLOADS["toy256x512_int4_g32"]
    assert toy.T == G["iterations"] and toy.group == G["column_group"]
    assert synth.WORKLOADS["llama31_70b_decoder_mxfp4_g32"].T == G["iterations"]


def test_two_level_constants():
    assert O.MXFP4_MAX_NORMAL == G["mxfp4_max_normal"] == O.E2M1_GRID.max()
    # a block whose max is 6 * 2^k gets the outer scale 2^k
    D = int(G["dual_block_size"])
    X = np.zeros((1, D))
    X[0, 3] = G["mxfp4_max_normal"] * 2.0 ** -5
    _, _, S, _ = O.two_level_quant(X, D, O.preset("mxfp4"))
    assert S[0, 0] == 2.0 ** -5


def test_library_two_level_default_block():
    import inspect
    import dual_scale_solver_b200 as dq
    assert inspect.signature(dq.two_level_quant).parameters["dual_block"].default == G["dual_block_size"]
