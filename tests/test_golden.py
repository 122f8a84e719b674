"""Oracle against the frozen fixtures written by tests/golden/make_golden.py."""
import os

import numpy as np

from oracle import starkv_oracle as O
from starkv_inputs import workloads as W

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_tiny_decode_matches_fixture():
    L = W.host_layer(W.workload(1), 0)
    out = O.decode_explicit(L["q"], L["B_K"], L["B_V"], L["k_cache"], L["v_cache"],
                            L["tables"], L["seq_lens"], L["scale"])
    want = np.loadtxt(os.path.join(GOLDEN, "tiny_decode_out.txt"))
    np.testing.assert_allclose(out.reshape(want.shape), want, rtol=1e-14, atol=0)


def test_tiny_append_codes_match_fixture():
    La = W.host_layer(W.custom("append", 31, W.LayerShape(4, 64, 16, 64), [37, 100, 0, 15]), 0)
    cK, cV = O.compress(La["k"], La["v"], La["A_K"], La["A_V"])
    want = np.loadtxt(os.path.join(GOLDEN, "tiny_append_codes.txt"))
    np.testing.assert_allclose(np.concatenate([cK.reshape(len(cK), -1), cV], axis=1), want,
                               rtol=1e-14, atol=1e-300)
