"""Failure path of the device pipelines: a wait that runs out ends the call cleanly.

Every pipeline wait in the kernels is bounded.  When a bound runs out, the
kernel sets STARKV_FLAG_TIMEOUT plus a bit naming the wait, leaves its loop,
lets the copies it issued land and returns, instead of hanging.  The test hook
shortens every bound to 1 ms and makes the K pass skip the copy of its first
ring stage in every CTA.  The waits on that stage then run out while no copy is
in flight: nothing faults, traps or hangs, and the GPU stays usable.  The next
call with the hook off, on the same workspace, must report a clean status and
give the correct output.
"""
import time

import numpy as np
import pytest
import torch

import rank_compressed_kv_star_b200 as S
from oracle import starkv_oracle as O
from starkv_inputs import device as D, workloads as W
from gpu_common import POISON, assert_close, desc_of, load

pytestmark = pytest.mark.gpu

SITE_K_FULL = 1 << (8 + 1)   # the consumers' wait on a K-pass ring stage


@pytest.fixture(scope="module", autouse=True)
def _built(cuda_ok):
    load()


@pytest.mark.parametrize("kv_heads", [0, 8])
def test_k_pass_wait_runs_out_then_clean_call(kv_heads):
    """kv_heads 0: the CUDA-core K pass; 8 (32 query heads): the tensor-core K pass (TMEM freed on abort)."""
    sh = W.LayerShape(32, 128, 64, 2048 if not kv_heads else 512, num_kv_heads=kv_heads)
    wl = W.custom("timeout", 97 + kv_heads, sh, [300, 40, 1000, 17], append=False)
    Lh = W.host_layer(wl, 0)
    Ld = D.device_layer(wl, 0, tables=Lh["tables"], nb=Lh["nb"])
    desc = desc_of(Ld)
    B, T = wl.batch, wl.max_seq_len
    wsb = S.starkv_decode_workspace_bytes(desc, B, T)
    ws = torch.full((wsb,), POISON, dtype=torch.uint8, device="cuda")
    out = torch.empty((B, 32, 128), dtype=torch.float16, device="cuda")
    args = (desc, B, T, Ld["q"], Ld["B_K"], Ld["B_V"], Ld["k_cache"], Ld["v_cache"], Ld["tables"],
            Ld["seq_lens"], Ld["scale"], ws, wsb, out)
    torch.cuda.synchronize()
    try:
        S.starkv_set_wait_test_hook(1000, 0)
        t0 = time.perf_counter()
        S.starkv_paged_decode(*args)
        st, flags = S.starkv_decode_check(ws)
        elapsed = time.perf_counter() - t0
    finally:
        S.starkv_set_wait_test_hook(0, -1)
    assert S.STATUS[st] == "STARKV_ERR_TIMEOUT", (S.STATUS[st], hex(flags))
    assert flags & S.FLAG_TIMEOUT and flags & SITE_K_FULL, hex(flags)
    assert elapsed < 1.5, elapsed     # the shortened bound, not the default of about 2 s per wait

    # the same workspace and output, hook off: clean status, correct result
    out.fill_(float("nan"))
    S.starkv_paged_decode(*args)
    assert S.starkv_decode_check(ws) == (0, 0)
    got = out.float().cpu().numpy().astype(np.float64)
    ref = O.decode_explicit(Lh["q"], Lh["B_K"], Lh["B_V"], Lh["k_cache"], Lh["v_cache"], Lh["tables"],
                            Lh["seq_lens"], Lh["scale"])
    assert_close({b: got[b] for b in range(B)}, {b: ref[b] for b in range(B)})
