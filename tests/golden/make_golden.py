"""Writes the oracle's outputs on the tiny workload as text fixtures.

The pages print no worked example of the method, so these fixtures are not
page values: they freeze the pinned fp64 oracle's result on the seeded tiny
workload (4 heads, head_dim 64, K rank 16, V rank 64, batch 2, lengths 37 and
100) so that any later change to the oracle's arithmetic shows up as a diff.
Run from the repository root:  python tests/golden/make_golden.py
"""
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from oracle import starkv_oracle as O          # noqa: E402
from starkv_inputs import workloads as W       # noqa: E402


def main():
    wl = W.workload(1)
    L = W.host_layer(wl, 0)
    out = O.decode_explicit(L["q"], L["B_K"], L["B_V"], L["k_cache"], L["v_cache"],
                            L["tables"], L["seq_lens"], L["scale"])
    np.savetxt(os.path.join(HERE, "tiny_decode_out.txt"), out.reshape(-1, out.shape[-1]),
               fmt="%.17e", header="oracle decode_explicit, tiny workload, rows = (b, h), cols = d")
    sh = W.LayerShape(4, 64, 16, 64)
    wa = W.custom("append", 31, sh, [37, 100, 0, 15], append=True)
    La = W.host_layer(wa, 0)
    cK, cV = O.compress(La["k"], La["v"], La["A_K"], La["A_V"])
    np.savetxt(os.path.join(HERE, "tiny_append_codes.txt"),
               np.concatenate([cK.reshape(len(cK), -1), cV], axis=1), fmt="%.17e",
               header="oracle compress: per row b, c_K[b] (H*r values) then c_V[b] (R values)")


if __name__ == "__main__":
    main()
