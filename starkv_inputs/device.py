"""Device copies of the seeded inputs (tests and benchmark only).

Large pools are generated on the GPU by the device twin of the host generator
(``gen_cuda.cu``, bit-identical by construction and by test), then written to
their paged slots with torch indexing.  Small tensors (activations,
projections, block tables) come from the host generator.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

from . import gen, workloads as W

_HERE = os.path.dirname(os.path.abspath(__file__))
GEN_LIB_PATH = os.path.join(_HERE, "libstarkv_inputs.so")
_gen = None


def gen_lib():
    global _gen
    if _gen is None:
        if not os.path.exists(GEN_LIB_PATH):
            raise OSError(f"{GEN_LIB_PATH} missing; run python -m rank_compressed_kv_star_b200.build")
        lib = ctypes.CDLL(GEN_LIB_PATH)
        lib.starkv_gen_codes.argtypes = [ctypes.c_uint64, ctypes.c_int64, ctypes.c_int32, ctypes.c_int64,
                                         ctypes.c_void_p, ctypes.c_int32, ctypes.c_float, ctypes.c_void_p,
                                         ctypes.c_void_p]
        lib.starkv_gen_codes.restype = ctypes.c_int
        _gen = lib
    return _gen


def gen_codes(key: int, n_rows: int, row_len: int, spectrum: torch.Tensor | None,
              out: torch.Tensor, row_offset: int = 0):
    """Fills ``out`` (fp16, contiguous, n_rows*row_len elements) on its device."""
    assert out.dtype == torch.float16 and out.is_contiguous() and out.numel() >= n_rows * row_len
    spec_ptr = spectrum.data_ptr() if spectrum is not None else None
    spec_len = spectrum.numel() if spectrum is not None else 0
    st = gen_lib().starkv_gen_codes(key & ((1 << 64) - 1), n_rows, row_len, row_offset, spec_ptr,
                                    spec_len, float(gen.IH4_SCALE), out.data_ptr(),
                                    torch.cuda.current_stream().cuda_stream)
    if st != 0:
        raise RuntimeError(f"starkv_gen_codes failed ({st})")


def slot_rows(table_row: np.ndarray, n_tokens: int, t0: int = 0) -> np.ndarray:
    t = np.arange(t0, t0 + n_tokens)
    return table_row[t // W.BLOCK_SIZE].astype(np.int64) * W.BLOCK_SIZE + t % W.BLOCK_SIZE


def device_layer(wl: W.Workload, layer: int, device="cuda", tables=None, nb=None,
                 fill_nan: bool = True):
    """All inputs of one layer on the device, pools filled with the seeded codes.

    Same content as :func:`workloads.host_layer`: the ``ctx_lens[b]`` context
    tokens of every sequence hold generated codes; every other slot is fp16 NaN.
    """
    sh = wl.layers[layer]
    H, d, r, R = sh.num_heads, sh.head_dim, sh.k_rank, sh.v_rank
    Hkv = sh.kv_heads
    if tables is None:
        tables, nb, _ = W.block_tables(wl.seed, wl.seq_lens, wl.max_blocks_per_seq, wl.decoy_frac)
    k_cache = torch.empty((nb, W.BLOCK_SIZE, Hkv, r), dtype=torch.float16, device=device)
    v_cache = torch.empty((nb, W.BLOCK_SIZE, R), dtype=torch.float16, device=device)
    if fill_nan:
        k_cache.fill_(float("nan"))
        v_cache.fill_(float("nan"))
    kspec = torch.from_numpy(W.k_spectrum(sh)).to(device)
    vspec = torch.from_numpy(W.v_spectrum(sh)).to(device)
    kflat = k_cache.view(nb * W.BLOCK_SIZE, Hkv * r)
    vflat = v_cache.view(nb * W.BLOCK_SIZE, R)
    tmax = int(wl.ctx_lens.max()) if wl.batch else 0
    tk = torch.empty(max(tmax, 1) * Hkv * r, dtype=torch.float16, device=device)
    tv = torch.empty(max(tmax, 1) * R, dtype=torch.float16, device=device)
    for b in range(wl.batch):
        T = int(wl.ctx_lens[b])
        if T == 0:
            continue
        gen_codes(W.code_key(wl, layer, W.POOL_K, b), T, Hkv * r, kspec, tk)
        gen_codes(W.code_key(wl, layer, W.POOL_V, b), T, R, vspec, tv)
        rows = torch.from_numpy(slot_rows(tables[b], T)).to(device)
        kflat.index_copy_(0, rows, tk[:T * Hkv * r].view(T, Hkv * r))
        vflat.index_copy_(0, rows, tv[:T * R].view(T, R))
    A_K, A_V, B_K, B_V = W.projections(wl, layer)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
    return dict(
        H=H, Hkv=Hkv, d=d, r=r, R=R, nb=nb, tables_np=tables,
        tables=dev(tables.astype(np.int32)),
        ctx_lens=dev(wl.ctx_lens.astype(np.int32)), seq_lens=dev(wl.seq_lens.astype(np.int32)),
        k_cache=k_cache, v_cache=v_cache,
        q=dev(W.activation(wl, layer, W.ACT_Q)), k=dev(W.activation(wl, layer, W.ACT_K)),
        v=dev(W.activation(wl, layer, W.ACT_V)),
        A_K=dev(A_K), A_V=dev(A_V), B_K=dev(B_K), B_V=dev(B_V),
        A_np=(A_K, A_V, B_K, B_V), scale=float(1.0 / np.sqrt(d)),
    )
