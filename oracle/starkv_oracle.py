"""CPU fp64 oracle of STAR-KV paged low-rank decode and compress-and-append.

TEST INFRASTRUCTURE.  Only the test-suite, the smoke check and the benchmark's
CPU-baseline leg may import this module.  The product path (the C-ABI library
and its Python binding) never calls it and shares no code with it.

What it computes (written from the method's description, not from any code):

* STAR-KV replaces the full-dimension K/V cache by a per-layer low-rank
  projection, head-wise for K and joint across heads for V, stored in a
  compressed paged format (Proxima README on wpnews.pro, "Low-rank KV Cache
  Compression for vLLM", opening method paragraph; same sentence on the
  tenosra.com/proxima landing page, first paragraph).
* Head-wise K: per head h, the code is ``c_K[h] = k_h . A_K[h]`` with
  ``A_K[h]`` of shape (head_dim x r); the head's key is recovered as
  ``k_hat_h = c_K[h] . B_K[h]`` with ``B_K[h]`` of shape (r x head_dim).
* Joint V: ``c_V = v . A_V`` with ``v`` the concatenation of all heads'
  values (H*head_dim) and ``A_V`` of shape (H*head_dim x R); values are
  recovered as ``v_hat = c_V . B_V`` with ``B_V`` of shape (R x H*head_dim).
* Paged format: pages of ``block_size = 16`` tokens (README, KV-cache block
  paragraph: "block size 16"), addressed through a per-sequence block table;
  pages of one sequence may be anywhere in the pool (botdigit.com PagedAttention
  explainer, "How Dynamic KV-Cache Compaction Works", block-level management).
  Token ``t`` of sequence ``b`` lives in slot ``t % 16`` of physical page
  ``block_table[b][t // 16]``.
* Decode: single-token attention of the new query over the sequence's cached
  tokens, textbook softmax with scale ``1/sqrt(head_dim)``.

* Grouped-query attention: the README lists Qwen, Mistral, Gemma and Llama-3
  support (wpnews.pro README, status paragraph), families whose layers have
  fewer KV heads than query heads.  Reading taken: K and V are compressed per
  *KV* head (head-wise A_K[j] for each of the Hkv KV heads, joint A_V over the
  Hkv*head_dim concatenated values), and query head ``h`` attends with KV head
  ``h // (H / Hkv)`` (consecutive query heads share a KV head).  With
  ``Hkv == H`` everything below is plain multi-head attention.

Readings where the pages are silent (also listed in the design notes):
K page layout ``[num_blocks][16][H][r]``, V page layout ``[num_blocks][16][R]``
(token-major inside a page, one block table shared by both pools);
``positions[b]`` is the length before the append; slots at or past
``seq_lens[b]`` are never read; ``seq_lens[b] == 0`` gives a zero output row.

Everything is evaluated in float64 on exactly the fp16 inputs the GPU sees.
"""
from __future__ import annotations

import numpy as np

BLOCK_SIZE = 16


# ------------------------------------------------------------------ heads

def kv_head(h: int, num_heads: int, num_kv_heads: int) -> int:
    """KV head that query head ``h`` reads (consecutive groups of H/Hkv heads)."""
    if num_heads % num_kv_heads:
        raise ValueError("query heads must be a multiple of KV heads")
    return h // (num_heads // num_kv_heads)


# ------------------------------------------------------------------ paging

def slot_of(table_row: np.ndarray, pos: int, block_size: int = BLOCK_SIZE):
    """Physical (page, slot) of logical token ``pos`` (paged format above)."""
    return int(table_row[pos // block_size]), int(pos % block_size)


def gather(cache: np.ndarray, table_row: np.ndarray, T: int) -> np.ndarray:
    """Logical ``[T][...]`` rows of one sequence, walking its block table, in fp64."""
    out = np.empty((T,) + cache.shape[2:], dtype=np.float64)
    for t in range(T):
        page, slot = slot_of(table_row, t)
        out[t] = cache[page, slot]
    return out


# --------------------------------------------------------------- compression

def compress(k: np.ndarray, v: np.ndarray, A_K: np.ndarray, A_V: np.ndarray):
    """Codes of new tokens.

    k, v: ``[B][Hkv][d]``; A_K ``[Hkv][d][r]`` (head-wise); A_V ``[Hkv*d][R]``
    (joint).  Returns fp64 ``c_K [B][Hkv][r]`` and ``c_V [B][R]``.
    """
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    A_K = np.asarray(A_K, dtype=np.float64)
    A_V = np.asarray(A_V, dtype=np.float64)
    B, H, d = k.shape
    c_K = np.empty((B, H, A_K.shape[2]))
    for h in range(H):
        c_K[:, h, :] = k[:, h, :] @ A_K[h]          # head-wise: k_h . A_K[h]
    c_V = v.reshape(B, H * d) @ A_V                 # joint: concat(v_h) . A_V
    return c_K, c_V


def compress_append(k, v, A_K, A_V, tables, positions, k_cache, v_cache):
    """Compress-and-append one new token per sequence.

    Codes are computed in fp64, rounded to fp16 (round to nearest even) and
    written to slot ``positions[b] % 16`` of page
    ``tables[b][positions[b] // 16]`` in both pools.  Returns
    ``(c_K, c_V, new_k_cache, new_v_cache)`` with the fp64 codes and updated
    copies of the pools (inputs are not modified).
    """
    c_K, c_V = compress(k, v, A_K, A_V)
    kc = np.array(k_cache, copy=True)
    vc = np.array(v_cache, copy=True)
    for b in range(len(positions)):
        page, slot = slot_of(tables[b], int(positions[b]))
        kc[page, slot] = c_K[b].astype(np.float16)
        vc[page, slot] = c_V[b].astype(np.float16)
    return c_K, c_V, kc, vc


def compress_store(k, v, A_K, A_V, slot_mapping, k_cache, v_cache, block_size=BLOCK_SIZE):
    """Compress rows and store their fp16 codes at flat slots ``page*16 + offset``.

    Returns ``(c_K, c_V, new_k_cache, new_v_cache)`` (inputs not modified).
    """
    c_K, c_V = compress(k, v, A_K, A_V)
    kc = np.array(k_cache, copy=True)
    vc = np.array(v_cache, copy=True)
    for i, sl in enumerate(slot_mapping):
        page, off = divmod(int(sl), block_size)
        kc[page, off] = c_K[i].astype(np.float16)
        vc[page, off] = c_V[i].astype(np.float16)
    return c_K, c_V, kc, vc


# ------------------------------------------------------------ decompression

def decompress_k(c_K_seq: np.ndarray, B_K: np.ndarray) -> np.ndarray:
    """``k_hat[t, j, :] = c_K[t, j, :] . B_K[j]`` per KV head j; returns ``[T][Hkv][d]``."""
    B_K = np.asarray(B_K, dtype=np.float64)
    T, H, _ = c_K_seq.shape
    out = np.empty((T, H, B_K.shape[2]))
    for h in range(H):
        out[:, h, :] = c_K_seq[:, h, :] @ B_K[h]
    return out


def decompress_v(c_V_seq: np.ndarray, B_V: np.ndarray) -> np.ndarray:
    """``v_hat[t, :] = c_V[t, :] . B_V``; returns ``[T][Hkv*d]``."""
    return c_V_seq @ np.asarray(B_V, dtype=np.float64)


# ---------------------------------------------------------------- attention

def softmax(a: np.ndarray) -> np.ndarray:
    """Textbook softmax over the last axis: exp(a - max a) / sum."""
    e = np.exp(a - a.max(axis=-1, keepdims=True))
    return e / e.sum(axis=-1, keepdims=True)


def attention_head(q_h: np.ndarray, k_h: np.ndarray, v_h: np.ndarray, scale: float):
    """One head of single-query attention: ``softmax(scale * K q) . V``."""
    if k_h.shape[0] == 0:
        return np.zeros(v_h.shape[1])
    p = softmax(scale * (k_h @ q_h))
    return p @ v_h


# ------------------------------------------------------------------- decode

def decode_explicit(q, B_K, B_V, k_cache, v_cache, tables, seq_lens, scale):
    """Definition of decode: decompress K and V explicitly, then attend.

    For every sequence: walk the block table, gather the codes of its
    ``seq_lens[b]`` tokens, rebuild ``k_hat``/``v_hat`` per KV head and run
    textbook softmax attention per query head with its KV head.  Returns
    fp64 ``[B][H][d]`` (H query heads; Hkv = ``B_K.shape[0]``).
    """
    q = np.asarray(q, dtype=np.float64)
    Bsz, H, d = q.shape
    Hkv = np.shape(B_K)[0]
    out = np.zeros((Bsz, H, d))
    for b in range(Bsz):
        T = int(seq_lens[b])
        if T == 0:
            continue
        c_K = gather(k_cache, tables[b], T)
        c_V = gather(v_cache, tables[b], T)
        k_hat = decompress_k(c_K, B_K)
        v_hat = decompress_v(c_V, B_V).reshape(T, Hkv, d)
        for h in range(H):
            j = kv_head(h, H, Hkv)
            out[b, h] = attention_head(q[b, h], k_hat[:, j, :], v_hat[:, j, :], scale)
    return out


def attend_codes_reordered(q_b, B_K, B_V, c_K, c_V, scale, heads=None):
    """One sequence, V applied after the weighted sum of codes.

    K is still decompressed explicitly.  For V the weighted sum is taken over
    the codes first, ``z_h = sum_t p_t c_V[t]``, and then projected,
    ``o_h = z_h . B_V[:, j*d:(j+1)*d]`` with ``j`` the head's KV head
    (associativity of the matrix product; agreement with
    :func:`decode_explicit` is a pinned test).  Returns ``[len(heads)][d]`` fp64.
    """
    q_b = np.asarray(q_b, dtype=np.float64)
    B_V = np.asarray(B_V, dtype=np.float64)
    H, d = q_b.shape
    Hkv = np.shape(B_K)[0]
    heads = range(H) if heads is None else heads
    T = c_K.shape[0]
    out = np.zeros((len(heads), d))
    if T == 0:
        return out
    B_K = np.asarray(B_K, dtype=np.float64)
    for i, h in enumerate(heads):
        j = kv_head(h, H, Hkv)
        k_hat_h = c_K[:, j, :] @ B_K[j]
        p = softmax(scale * (k_hat_h @ q_b[h]))
        z = p @ c_V
        out[i] = z @ B_V[:, j * d:(j + 1) * d]
    return out


def decode_reordered(q, B_K, B_V, k_cache, v_cache, tables, seq_lens, scale):
    """Same result as :func:`decode_explicit`; cheaper for long contexts."""
    q = np.asarray(q, dtype=np.float64)
    Bsz, H, d = q.shape
    out = np.zeros((Bsz, H, d))
    for b in range(Bsz):
        T = int(seq_lens[b])
        if T == 0:
            continue
        out[b] = attend_codes_reordered(q[b], B_K, B_V, gather(k_cache, tables[b], T),
                                        gather(v_cache, tables[b], T), scale)
    return out


def decode_contiguous(q, B_K, B_V, c_K_list, c_V_list, scale):
    """Decode over per-sequence contiguous code arrays (no paging)."""
    q = np.asarray(q, dtype=np.float64)
    Bsz, H, d = q.shape
    Hkv = np.shape(B_K)[0]
    out = np.zeros((Bsz, H, d))
    for b in range(Bsz):
        c_K = np.asarray(c_K_list[b], dtype=np.float64)
        c_V = np.asarray(c_V_list[b], dtype=np.float64)
        T = c_K.shape[0]
        if T == 0:
            continue
        k_hat = decompress_k(c_K, B_K)
        v_hat = decompress_v(c_V, B_V).reshape(T, Hkv, d)
        for h in range(H):
            j = kv_head(h, H, Hkv)
            out[b, h] = attention_head(q[b, h], k_hat[:, j, :], v_hat[:, j, :], scale)
    return out


def attention_uncompressed(q, k_list, v_list, scale):
    """Plain single-query attention over full K/V ``[T][Hkv][d]`` (grouped when Hkv < H)."""
    q = np.asarray(q, dtype=np.float64)
    Bsz, H, d = q.shape
    out = np.zeros((Bsz, H, d))
    for b in range(Bsz):
        k = np.asarray(k_list[b], dtype=np.float64)
        v = np.asarray(v_list[b], dtype=np.float64)
        Hkv = k.shape[1]
        for h in range(H):
            j = kv_head(h, H, Hkv)
            out[b, h] = attention_head(q[b, h], k[:, j, :], v[:, j, :], scale)
    return out


def prefill_attention(q, B_K, B_V, k_cache, v_cache, tables, starts, chunk_lens, scale):
    """Causal attention of prefill chunks over the paged codes (chunked prefill).

    The README has STAR-KV served by dedicated kernels over the compressed
    pages (method paragraph) and gives no formula; the reading taken is the
    autoregressive one: query token ``i`` of sequence ``b`` (row
    ``sum(chunk_lens[:b]) + i`` of ``q``) attends over the sequence's tokens
    ``0 .. starts[b] + i``, whose codes (the chunk's own included) are in the
    cache.  Keys and values are decompressed explicitly as in
    :func:`decode_explicit`.  Returns fp64 ``[n_rows][H][d]``.
    """
    q = np.asarray(q, dtype=np.float64)
    n_rows, H, d = q.shape
    Hkv = np.shape(B_K)[0]
    out = np.zeros((n_rows, H, d))
    row = 0
    for b, n in enumerate(chunk_lens):
        n = int(n)
        t_end = int(starts[b]) + n
        if n == 0:
            continue
        k_hat = decompress_k(gather(k_cache, tables[b], t_end), B_K)
        v_hat = decompress_v(gather(v_cache, tables[b], t_end), B_V).reshape(t_end, Hkv, d)
        for i in range(n):
            T = int(starts[b]) + i + 1
            for h in range(H):
                j = kv_head(h, H, Hkv)
                out[row, h] = attention_head(q[row, h], k_hat[:T, j, :], v_hat[:T, j, :], scale)
            row += 1
    return out


def decode_stages(q_b, B_K, B_V, c_K, c_V, scale):
    """Intermediate quantities of one sequence in absorbed form, for diagnosis.

    With ``j = g(h)`` the query head's KV head: ``q_tilde[h] = scale * q_h .
    B_K[j]^T`` (r-vector), ``s[h, t] = q_tilde[h] . c_K[t, j]``, ``p =
    softmax_t(s)``, ``z[h] = p[h] . c_V`` and ``o[h] = z[h] . B_V[:,
    j*d:(j+1)*d]``.  The scores here are natural-log logits (no base-2 change).
    """
    q_b = np.asarray(q_b, dtype=np.float64)
    B_K = np.asarray(B_K, dtype=np.float64)
    B_V = np.asarray(B_V, dtype=np.float64)
    H, d = q_b.shape
    Hkv = B_K.shape[0]
    g = [kv_head(h, H, Hkv) for h in range(H)]
    q_tilde = np.stack([scale * (B_K[g[h]] @ q_b[h]) for h in range(H)])
    s = np.stack([c_K[:, g[h], :] @ q_tilde[h] for h in range(H)])
    p = softmax(s)
    z = p @ c_V
    o = np.stack([z[h] @ B_V[:, g[h] * d:(g[h] + 1) * d] for h in range(H)])
    return dict(q_tilde=q_tilde, s=s, p=p, z=z, o=o)


# ----------------------------------------------------------- rank selection

def rank_from_spectrum(s, tau: float) -> int:
    """Soft-threshold rank: the number of singular values strictly above ``tau``.

    "learned soft-thresholding for adaptive rank control" (README opening
    line): soft-thresholding ``max(s_i - tau, 0)`` zeroes every singular value
    at or below ``tau``, so the rank kept is ``#{i : s_i > tau}``.
    """
    s = np.asarray(s, dtype=np.float64)
    return int(np.count_nonzero(s > tau))


# ----------------------------------------------------------------- capacity

def kv_bytes_per_token(num_heads, k_ranks, v_ranks) -> int:
    """fp16 bytes one token occupies in the compressed cache, summed over layers.

    Per layer a token stores H*r head-wise K codes and R joint V codes (the
    paged format above), 2 bytes each, with H the layer's KV heads.  A
    full-rank cache is r = d, R = H*d.
    """
    return sum(2 * (h * r + R) for h, r, R in zip(num_heads, k_ranks, v_ranks))


def num_blocks(budget_bytes: int, bytes_per_token: int, block_size: int = BLOCK_SIZE) -> int:
    """Whole blocks of ``block_size`` tokens that fit in ``budget_bytes``."""
    return budget_bytes // (block_size * bytes_per_token)
