"""The allocation-free decode entry point against the regular one (GPU).

starkv_paged_decode_static serves callers that cannot allocate device memory
while decoding (an engine whose KV pool already holds nearly all GPU memory, a
C host without an allocator for scratch): its scratch is a fixed device array
inside the library.  Its output must match starkv_paged_decode on the same
inputs, call after call, within the decode tolerance used by the other tests
(max |diff| <= 2e-3, relative L2 <= 1e-3); oversized problems are refused.
This file sorts last so that a stop-at-first-failure run has run every other
test before it.
"""
import numpy as np
import pytest
import torch

import rank_compressed_kv_star_b200 as S
from starkv_inputs import device as D, workloads as W

pytestmark = pytest.mark.gpu

STATIC_BYTES = 64 << 20


@pytest.fixture(scope="module", autouse=True)
def _built(cuda_ok):
    from rank_compressed_kv_star_b200 import build
    build.build()
    build.build_inputs()
    S.load_library()


def _regular(L, desc, B, T):
    wsb = S.starkv_decode_workspace_bytes(desc, B, T)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    out = torch.empty((B, L["H"], L["d"]), dtype=torch.float16, device="cuda")
    S.starkv_paged_decode(desc, B, T, L["q"], L["B_K"], L["B_V"], L["k_cache"], L["v_cache"],
                          L["tables"], L["seq_lens"], L["scale"], ws, wsb, out)
    torch.cuda.synchronize()
    return out.float().cpu().numpy()


@pytest.mark.parametrize("case", ["tiny", "heads32"])
def test_static_scratch_decode_matches_regular_twice(case):
    if case == "tiny":
        wl = W.workload(1)
    else:
        wl = W.custom("static", 808, W.LayerShape(32, 128, 64, 2048), [300, 17, 1, 128], append=False)
    L = D.device_layer(wl, 0)
    desc = S.layer_desc(L["H"], L["d"], L["r"], L["R"], L["nb"], L["tables"].shape[1])
    B, T = wl.batch, wl.max_seq_len
    assert S.starkv_decode_workspace_bytes(desc, B, T) <= STATIC_BYTES
    ref = _regular(L, desc, B, T)
    for _ in range(2):
        out = torch.full((B, L["H"], L["d"]), float("nan"), dtype=torch.float16, device="cuda")
        S.starkv_paged_decode_static(desc, B, T, L["q"], L["B_K"], L["B_V"], L["k_cache"],
                                     L["v_cache"], L["tables"], L["seq_lens"], L["scale"], out)
        torch.cuda.synchronize()
        got = out.float().cpu().numpy()
        assert np.isfinite(got).all()
        assert np.abs(got - ref).max() <= 2e-3
        assert np.linalg.norm(got - ref) <= 1e-3 * np.linalg.norm(ref)


def test_static_scratch_refuses_oversized_problem():
    desc = S.layer_desc(32, 128, 64, 2048, 40000, 512)
    assert S.starkv_decode_workspace_bytes(desc, 64, 8192) > STATIC_BYTES
    fake = 1 << 20
    st = S.starkv_paged_decode_static(desc, 64, 8192, fake, fake, fake, fake, fake, fake, fake,
                                      0.1, fake, check=False)
    assert S.STATUS[st] == "STARKV_ERR_WORKSPACE"
