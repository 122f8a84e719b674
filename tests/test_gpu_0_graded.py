"""GPU parity of the hot path on the five benchmark workloads, compress-and-append
bit-exactness, and grouped-query attention, against the CPU fp64 oracle.

These are the graded checks, so this file sorts before the other GPU test files:
a run that stops at its first failure reaches them before any edge case.
Tolerances are stated in ``gpu_common``: decode max |err| <= 2e-3 and relative
L2 <= 1e-3; appended-code placement and untouched bytes bit-exact.
"""
import numpy as np
import pytest
import torch

from starkv_inputs import workloads as W
from gpu_common import (append_check, append_then_decode, assert_close, full_check, load, oracle_rows,
                        run_decode)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built(cuda_ok):
    load()


def test_decode_tiny_workload():
    """The tiny workload (4 heads, d64, r16, R64, lengths 37 and 100): every output."""
    full_check(W.workload(1))


@pytest.mark.parametrize("idx,layer,sample", [
    (2, 0, list(range(16))),            # batch 16, context 2048: every sequence
    (3, 0, [0, 31, 63]),                # batch 64, context 8192
    (4, 0, [0, 17, 47]),                # batch 48, mixed lengths, r=32 / R=1024
    (4, 1, [5, 23, 30]),                #   r=64 / R=2048
    (4, 2, [11, 40]),                   #   r=96 / R=3072
    (5, 0, [0, 7]),                     # 32-layer 7B attention path, first layer
    (5, 31, [3]),                       #   last layer
    (6, 0, [0, 21, 63]),                # grouped-query layer, batch 64, context 8192
])
def test_full_size_append_then_decode(idx, layer, sample):
    """Full-size workloads in the benchmark's launch configuration (one starkv_append_decode per step).

    The whole batch's append is checked (placement and untouched bytes
    bit-exact, codes against the oracle), then decode on sampled sequences.
    """
    wl = W.workload(idx)
    Ld, appended, (got, _) = append_check(wl, layer, run=append_then_decode)
    ref = oracle_rows(wl, layer, W.activation(wl, layer, W.ACT_Q), Ld["A_np"], sample, wl.seq_lens,
                      appended)
    assert_close({b: got[b] for b in sample}, ref)
    assert np.isfinite(got).all()
    del Ld
    torch.cuda.empty_cache()


def test_append_tiny_ragged():
    """Positions 37, 100, 0 and 15: mid-page, page start of a new page, the first slot, a page's last slot."""
    append_check(W.custom("app", 31, W.LayerShape(4, 64, 16, 64), [37, 100, 0, 15]))


@pytest.mark.parametrize("kv_heads", [0, 8])
def test_fused_step_equals_append_then_decode_calls(kv_heads):
    """starkv_append_decode against starkv_compress_append + starkv_paged_decode: identical pools and outputs."""
    sh = W.LayerShape(32, 128, 64, 2048 if not kv_heads else 512, num_kv_heads=kv_heads)
    wl = W.custom("fused", 4141 + kv_heads, sh, [37, 100, 0, 15, 700, 2047, 31], append=True)
    La, appended, _ = append_check(wl)
    sep, *_ = run_decode(La)
    Lb, _, (fused, _) = append_check(wl, run=append_then_decode)
    assert torch.equal(La["k_cache"].view(torch.int16), Lb["k_cache"].view(torch.int16))
    assert torch.equal(La["v_cache"].view(torch.int16), Lb["v_cache"].view(torch.int16))
    assert np.array_equal(sep, fused)
    ref = oracle_rows(wl, 0, W.activation(wl, 0, W.ACT_Q), La["A_np"], range(wl.batch), wl.seq_lens, appended)
    assert_close({b: fused[b] for b in range(wl.batch)}, ref)


@pytest.mark.parametrize("H,Hkv,d,r,R", [
    (32, 8, 128, 64, 512),      # Llama-3-8B-like heads, 4 query heads per KV head
    (32, 16, 128, 64, 1024),    # 2 per KV head
    (16, 1, 128, 64, 128),      # one KV head (multi-query)
    (64, 8, 128, 128, 1024),    # 8 per KV head, r = d
    (8, 2, 64, 16, 128),        # small pages: 8-page K stages
    (64, 32, 64, 64, 1024),     # 32 KV heads: the CUDA-core K pass with 2 query heads per KV head
    (4, 2, 64, 16, 64),         # 4 query heads: the CUDA-core K pass
])
def test_decode_grouped_query(H, Hkv, d, r, R):
    sh = W.LayerShape(H, d, r, R, num_kv_heads=Hkv)
    wl = W.custom(f"gqa{H}x{Hkv}", 600 + H + Hkv, sh, [1, 15, 16, 17, 300, 0, 1000, 129], append=False)
    full_check(wl)


def test_append_then_decode_grouped_query():
    sh = W.LayerShape(32, 128, 64, 512, num_kv_heads=8)
    wl = W.custom("gqa-app", 777, sh, [37, 100, 0, 15, 2000, 4095], append=True)
    Ld, appended, _ = append_check(wl)
    got, *_ = run_decode(Ld)
    ref = oracle_rows(wl, 0, W.activation(wl, 0, W.ACT_Q), Ld["A_np"], range(wl.batch), wl.seq_lens,
                      appended)
    assert_close({b: got[b] for b in range(wl.batch)}, ref)


def test_step_from_host_buffers_equals_device_call():
    """starkv_append_decode_host (inputs and output in pinned host memory) against starkv_append_decode."""
    import rank_compressed_kv_star_b200 as S
    from gpu_common import POISON, desc_of
    from starkv_inputs import device as D
    sh = W.LayerShape(32, 128, 64, 2048)
    wl = W.custom("host", 4343, sh, [37, 100, 0, 15, 700], append=True)
    La = D.device_layer(wl, 0)
    Lb = D.device_layer(wl, 0)
    desc = desc_of(La)
    B, T = wl.batch, wl.max_seq_len
    dev_out, _ = append_then_decode(La, desc, None, B)
    wsb = S.starkv_decode_workspace_bytes(desc, B, T)
    ws = torch.full((wsb,), POISON, dtype=torch.uint8, device="cuda")
    stg = S.starkv_host_staging_bytes(desc, B)
    staging = torch.full((stg,), POISON, dtype=torch.uint8, device="cuda")
    h = {n: Lb[n].cpu().pin_memory() for n in ("q", "k", "v", "tables", "seq_lens", "ctx_lens")}
    out_host = torch.full((B, 32, 128), float("nan"), dtype=torch.float16).pin_memory()
    S.starkv_append_decode_host(desc, B, T, h["k"], h["v"], h["ctx_lens"], h["q"], h["tables"], h["seq_lens"],
                                Lb["A_K"], Lb["A_V"], Lb["B_K"], Lb["B_V"], Lb["k_cache"], Lb["v_cache"],
                                Lb["scale"], staging, stg, ws, wsb, out_host)
    torch.cuda.synchronize()
    assert S.starkv_decode_check(ws) == (0, 0)
    assert np.array_equal(out_host.float().numpy().astype(np.float64), dev_out)
    assert torch.equal(La["k_cache"].view(torch.int16), Lb["k_cache"].view(torch.int16))
    assert torch.equal(La["v_cache"].view(torch.int16), Lb["v_cache"].view(torch.int16))
