"""Python binding of libstarkv (STAR-KV paged low-rank decode on sm_100a).

Argument marshalling only: every function forwards to the C entry point of the
same name in ``libstarkv.so`` (declared in ``include/starkv.h``).  Tensor
arguments may be torch tensors (their ``data_ptr()`` is passed) or raw integer
device addresses; ``stream`` may be a ``torch.cuda.Stream``, a raw
``cudaStream_t`` integer or ``None`` (the current torch stream).  There is no
fallback: if the shared library cannot be loaded, importing the functions
raises.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libstarkv.so")

STATUS = {
    0: "STARKV_OK", 1: "STARKV_ERR_INVALID_ARG", 2: "STARKV_ERR_UNSUPPORTED",
    3: "STARKV_ERR_WORKSPACE", 4: "STARKV_ERR_CUDA", 5: "STARKV_ERR_DEVICE_CHECK",
    6: "STARKV_ERR_TIMEOUT",
}
FLAG_BAD_BLOCK_ID, FLAG_BAD_SEQ_LEN, FLAG_TIMEOUT = 1, 2, 4

EXPORTED = (
    "starkv_compress_append", "starkv_compress_store", "starkv_decode_workspace_bytes",
    "starkv_paged_decode", "starkv_append_decode", "starkv_append_decode_host", "starkv_host_staging_bytes",
    "starkv_paged_decode_profiled", "starkv_paged_decode_static",
    "starkv_decode_check", "starkv_decode_workspace_layout", "starkv_status_string",
    "starkv_rank_from_spectrum", "starkv_version", "starkv_kv_bytes_per_token", "starkv_num_blocks",
    "starkv_prefill_workspace_bytes", "starkv_paged_prefill", "starkv_set_wait_test_hook",
)


class StarkvError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {STATUS.get(status, status)}")
        self.status = status


class LayerDesc(ctypes.Structure):
    _fields_ = [("num_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("k_rank", ctypes.c_int32), ("v_rank", ctypes.c_int32),
                ("block_size", ctypes.c_int32), ("num_blocks", ctypes.c_int32),
                ("max_blocks_per_seq", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32)]


class WorkspaceLayout(ctypes.Structure):
    _fields_ = [("total_bytes", ctypes.c_size_t), ("status_off", ctypes.c_size_t),
                ("prefix_off", ctypes.c_size_t), ("qt_off", ctypes.c_size_t),
                ("logits_off", ctypes.c_size_t), ("mpart_off", ctypes.c_size_t),
                ("lpart_off", ctypes.c_size_t),
                ("zpart_off", ctypes.c_size_t),
                ("t_pad", ctypes.c_int32), ("k_ctas", ctypes.c_int32), ("k_slots", ctypes.c_int32),
                ("v_ctas", ctypes.c_int32), ("v_slots", ctypes.c_int32),
                ("n_rranges", ctypes.c_int32), ("r_range", ctypes.c_int32),
                ("k_tensor", ctypes.c_int32), ("qth_off", ctypes.c_size_t)]


def layer_desc(num_heads, head_dim, k_rank, v_rank, num_blocks, max_blocks_per_seq,
               block_size=16, num_kv_heads=0) -> LayerDesc:
    """``num_kv_heads`` 0 means multi-head attention (as many KV heads as query heads)."""
    return LayerDesc(num_heads, head_dim, k_rank, v_rank, block_size, num_blocks,
                     max_blocks_per_seq, num_kv_heads)


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Loads libstarkv.so (raises OSError when it is missing: no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise OSError(f"libstarkv.so not found at {path}; build it with "
                      "`python -m rank_compressed_kv_star_b200.build`")
    lib = ctypes.CDLL(path)
    P, I32, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    DP = ctypes.POINTER(LayerDesc)
    lib.starkv_compress_append.argtypes = [DP, I32, P, P, P, P, P, P, P, P, P, P]
    lib.starkv_compress_append.restype = ctypes.c_int
    lib.starkv_compress_store.argtypes = [DP, I32, P, P, P, P, P, P, P, P, P]
    lib.starkv_compress_store.restype = ctypes.c_int
    lib.starkv_decode_workspace_bytes.argtypes = [DP, I32, I32]
    lib.starkv_decode_workspace_bytes.restype = SZ
    lib.starkv_paged_decode.argtypes = [DP, I32, I32, P, P, P, P, P, P, P, ctypes.c_float,
                                        P, SZ, P, P]
    lib.starkv_paged_decode.restype = ctypes.c_int
    lib.starkv_append_decode.argtypes = [DP, I32, I32, P, P, P, P, P, P, P, P, P, P, P, P, ctypes.c_float,
                                         P, SZ, P, P, P]
    lib.starkv_append_decode.restype = ctypes.c_int
    lib.starkv_host_staging_bytes.argtypes = [DP, I32]
    lib.starkv_host_staging_bytes.restype = SZ
    lib.starkv_append_decode_host.argtypes = [DP, I32, I32, P, P, P, P, P, P, P, P, P, P, P, P, ctypes.c_float,
                                              P, SZ, P, SZ, P, P, P]
    lib.starkv_append_decode_host.restype = ctypes.c_int
    lib.starkv_paged_decode_profiled.argtypes = [DP, I32, I32, P, P, P, P, P, P, P, ctypes.c_float,
                                                 P, SZ, P, P, ctypes.POINTER(P)]
    lib.starkv_paged_decode_profiled.restype = ctypes.c_int
    lib.starkv_paged_decode_static.argtypes = [DP, I32, I32, P, P, P, P, P, P, P, ctypes.c_float, P, P]
    lib.starkv_prefill_workspace_bytes.argtypes = [DP, I32, I32, I32]
    lib.starkv_prefill_workspace_bytes.restype = ctypes.c_size_t
    lib.starkv_paged_prefill.argtypes = [DP, I32, I32, I32, P, P, P, P, P, P, P, P, ctypes.c_float, P,
                                         ctypes.c_size_t, P, P]
    lib.starkv_paged_prefill.restype = ctypes.c_int
    lib.starkv_paged_decode_static.restype = ctypes.c_int
    lib.starkv_decode_check.argtypes = [P, P, ctypes.POINTER(ctypes.c_int32)]
    lib.starkv_decode_check.restype = ctypes.c_int
    lib.starkv_decode_workspace_layout.argtypes = [DP, I32, I32, ctypes.POINTER(WorkspaceLayout)]
    lib.starkv_decode_workspace_layout.restype = ctypes.c_int
    lib.starkv_status_string.argtypes = [ctypes.c_int]
    lib.starkv_status_string.restype = ctypes.c_char_p
    lib.starkv_rank_from_spectrum.argtypes = [ctypes.POINTER(ctypes.c_double), I32, ctypes.c_double]
    lib.starkv_rank_from_spectrum.restype = I32
    I64 = ctypes.c_int64
    IP = ctypes.POINTER(ctypes.c_int32)
    lib.starkv_kv_bytes_per_token.argtypes = [I32, IP, IP, IP]
    lib.starkv_kv_bytes_per_token.restype = I64
    lib.starkv_num_blocks.argtypes = [I64, I64, I32]
    lib.starkv_num_blocks.restype = I64
    lib.starkv_set_wait_test_hook.argtypes = [ctypes.c_uint32, I32]
    lib.starkv_set_wait_test_hook.restype = ctypes.c_int
    lib.starkv_version.argtypes = []
    lib.starkv_version.restype = I32
    _lib = lib
    return lib


def _desc_ref(desc):
    return ctypes.byref(desc) if desc is not None else None


def _ptr(x) -> int | None:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s) -> int | None:
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(status: int, where: str):
    if status != 0:
        raise StarkvError(status, where)


def starkv_compress_append(desc: LayerDesc, batch: int, k, v, A_K, A_V, block_tables, positions,
                           k_cache, v_cache, stream=None, check: bool = True, status=None) -> int:
    """``status``: optional device int32 word that skipped targets flag (never cleared by the call)."""
    st = load_library().starkv_compress_append(
        _desc_ref(desc), batch, _ptr(k), _ptr(v), _ptr(A_K), _ptr(A_V), _ptr(block_tables),
        _ptr(positions), _ptr(k_cache), _ptr(v_cache), _ptr(status), _stream(stream))
    if check:
        _check(st, "starkv_compress_append")
    return st


def starkv_compress_store(desc: LayerDesc, n_tokens: int, k, v, A_K, A_V, slot_mapping, k_cache,
                          v_cache, stream=None, check: bool = True, status=None) -> int:
    st = load_library().starkv_compress_store(
        _desc_ref(desc), n_tokens, _ptr(k), _ptr(v), _ptr(A_K), _ptr(A_V), _ptr(slot_mapping),
        _ptr(k_cache), _ptr(v_cache), _ptr(status), _stream(stream))
    if check:
        _check(st, "starkv_compress_store")
    return st


def starkv_decode_workspace_bytes(desc: LayerDesc, batch: int, max_seq_len: int) -> int:
    return int(load_library().starkv_decode_workspace_bytes(_desc_ref(desc), batch, max_seq_len))


def starkv_decode_workspace_layout(desc: LayerDesc, batch: int, max_seq_len: int) -> WorkspaceLayout:
    out = WorkspaceLayout()
    _check(load_library().starkv_decode_workspace_layout(_desc_ref(desc), batch, max_seq_len,
                                                         ctypes.byref(out)),
           "starkv_decode_workspace_layout")
    return out


def starkv_paged_decode(desc: LayerDesc, batch: int, max_seq_len: int, q, B_K, B_V, k_cache,
                        v_cache, block_tables, seq_lens, scale: float, workspace,
                        workspace_bytes: int, out, stream=None, check: bool = True) -> int:
    st = load_library().starkv_paged_decode(
        _desc_ref(desc), batch, max_seq_len, _ptr(q), _ptr(B_K), _ptr(B_V), _ptr(k_cache),
        _ptr(v_cache), _ptr(block_tables), _ptr(seq_lens), float(scale), _ptr(workspace),
        int(workspace_bytes), _ptr(out), _stream(stream))
    if check:
        _check(st, "starkv_paged_decode")
    return st


def starkv_append_decode(desc: LayerDesc, batch: int, max_seq_len: int, k, v, A_K, A_V, positions, q, B_K,
                         B_V, k_cache, v_cache, block_tables, seq_lens, scale: float, workspace,
                         workspace_bytes: int, out, stream=None, check: bool = True, append_status=None) -> int:
    """compress-append of the new tokens then paged decode, in one call (one launch fewer per kernel pair)."""
    st = load_library().starkv_append_decode(
        _desc_ref(desc), batch, max_seq_len, _ptr(k), _ptr(v), _ptr(A_K), _ptr(A_V), _ptr(positions), _ptr(q),
        _ptr(B_K), _ptr(B_V), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), _ptr(seq_lens), float(scale),
        _ptr(workspace), int(workspace_bytes), _ptr(out), _ptr(append_status), _stream(stream))
    if check:
        _check(st, "starkv_append_decode")
    return st


def starkv_host_staging_bytes(desc: LayerDesc, batch: int) -> int:
    return int(load_library().starkv_host_staging_bytes(_desc_ref(desc), batch))


def starkv_append_decode_host(desc: LayerDesc, batch: int, max_seq_len: int, k_host, v_host, positions_host,
                              q_host, block_tables_host, seq_lens_host, A_K, A_V, B_K, B_V, k_cache, v_cache,
                              scale: float, staging, staging_bytes: int, workspace, workspace_bytes: int,
                              out_host, stream=None, check: bool = True, append_status=None) -> int:
    """The step from host buffers (``*_host``: pinned CPU tensors or addresses); copies run in the call."""
    st = load_library().starkv_append_decode_host(
        _desc_ref(desc), batch, max_seq_len, _ptr(k_host), _ptr(v_host), _ptr(positions_host), _ptr(q_host),
        _ptr(block_tables_host), _ptr(seq_lens_host), _ptr(A_K), _ptr(A_V), _ptr(B_K), _ptr(B_V),
        _ptr(k_cache), _ptr(v_cache), float(scale), _ptr(staging), int(staging_bytes), _ptr(workspace),
        int(workspace_bytes), _ptr(out_host), _ptr(append_status), _stream(stream))
    if check:
        _check(st, "starkv_append_decode_host")
    return st


def starkv_prefill_workspace_bytes(desc: LayerDesc, n_seqs: int, n_rows: int, max_seq_len: int) -> int:
    return int(load_library().starkv_prefill_workspace_bytes(_desc_ref(desc), n_seqs, n_rows, max_seq_len))


def starkv_paged_prefill(desc: LayerDesc, n_seqs: int, n_rows: int, max_seq_len: int, q, B_K, B_V,
                         k_cache, v_cache, block_tables, starts, row_offsets, scale: float, workspace,
                         workspace_bytes: int, out, stream=None, check: bool = True) -> int:
    st = load_library().starkv_paged_prefill(
        _desc_ref(desc), n_seqs, n_rows, max_seq_len, _ptr(q), _ptr(B_K), _ptr(B_V), _ptr(k_cache),
        _ptr(v_cache), _ptr(block_tables), _ptr(starts), _ptr(row_offsets), float(scale),
        _ptr(workspace), int(workspace_bytes), _ptr(out), _stream(stream))
    if check:
        _check(st, "starkv_paged_prefill")
    return st


def starkv_paged_decode_profiled(desc: LayerDesc, batch: int, max_seq_len: int, q, B_K, B_V,
                                 k_cache, v_cache, block_tables, seq_lens, scale: float, workspace,
                                 workspace_bytes: int, out, stage_events, stream=None,
                                 check: bool = True) -> int:
    """``stage_events``: five ``torch.cuda.Event`` (or raw cudaEvent_t ints / None)."""
    raw = [None if e is None else (e if isinstance(e, int) else e.cuda_event) for e in stage_events]
    assert len(raw) == 5
    arr = (ctypes.c_void_p * 5)(*raw)
    st = load_library().starkv_paged_decode_profiled(
        _desc_ref(desc), batch, max_seq_len, _ptr(q), _ptr(B_K), _ptr(B_V), _ptr(k_cache),
        _ptr(v_cache), _ptr(block_tables), _ptr(seq_lens), float(scale), _ptr(workspace),
        int(workspace_bytes), _ptr(out), _stream(stream), arr)
    if check:
        _check(st, "starkv_paged_decode_profiled")
    return st


def starkv_paged_decode_static(desc: LayerDesc, batch: int, max_seq_len: int, q, B_K, B_V, k_cache,
                               v_cache, block_tables, seq_lens, scale: float, out, stream=None,
                               check: bool = True) -> int:
    """Decode with the library's fixed device scratch (no workspace argument)."""
    st = load_library().starkv_paged_decode_static(
        _desc_ref(desc), batch, max_seq_len, _ptr(q), _ptr(B_K), _ptr(B_V), _ptr(k_cache),
        _ptr(v_cache), _ptr(block_tables), _ptr(seq_lens), float(scale), _ptr(out), _stream(stream))
    if check:
        _check(st, "starkv_paged_decode_static")
    return st


def starkv_decode_check(workspace, stream=None) -> tuple[int, int]:
    """Returns (status, flags) after synchronising the stream."""
    flags = ctypes.c_int32(0)
    st = load_library().starkv_decode_check(_ptr(workspace), _stream(stream), ctypes.byref(flags))
    return st, flags.value


def starkv_set_wait_test_hook(wait_limit_us: int, drop_k_stage: int, check: bool = True) -> int:
    """Test hook: shorten every device wait bound (0 = default) and drop one K-pass stage (-1 = off)."""
    st = load_library().starkv_set_wait_test_hook(int(wait_limit_us), int(drop_k_stage))
    if check:
        _check(st, "starkv_set_wait_test_hook")
    return st


def starkv_status_string(status: int) -> str:
    return load_library().starkv_status_string(status).decode()


def starkv_rank_from_spectrum(s, tau: float) -> int:
    vals = [float(x) for x in s]
    arr = (ctypes.c_double * len(vals))(*vals) if vals else None
    return int(load_library().starkv_rank_from_spectrum(arr, len(vals), float(tau)))


def starkv_kv_bytes_per_token(num_heads, k_ranks, v_ranks) -> int:
    """Compressed cache bytes per token over the layers (one entry per layer)."""
    n = len(num_heads)
    arr = lambda xs: (ctypes.c_int32 * n)(*[int(x) for x in xs]) if n else None
    return int(load_library().starkv_kv_bytes_per_token(n, arr(num_heads), arr(k_ranks), arr(v_ranks)))


def starkv_num_blocks(budget_bytes: int, bytes_per_token: int, block_size: int = 16) -> int:
    return int(load_library().starkv_num_blocks(int(budget_bytes), int(bytes_per_token), block_size))


def starkv_version() -> int:
    return int(load_library().starkv_version())
