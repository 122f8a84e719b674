"""Synthetic workloads shaped like the Proxima decode-kernel benchmark.

Shapes follow the pages' kernel benchmark (32-head MHA, head_size 128, rank 64,
fp16, block size 16, batch 1-64, context 1k-32k: tenosra.com/proxima
"Decode kernel" table; wpnews.pro Show-HN text, bench_attn_step table and the
KV-cache block paragraph).  Values are synthetic and seeded; no dataset or
trained checkpoint is involved.

Everything here is input construction: sizes, seeds, block tables (random
physical page permutations with NaN decoy pages) and the seeded values of
codes, projections and activations.  The paged placement helper below only
*writes* inputs into pools the way a paged cache lays them out (token ``t`` of
sequence ``b`` lives in slot ``t % bs`` of page ``block_table[b][t // bs]``);
reading them back is the oracle's and the kernels' own business.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

from . import gen

BLOCK_SIZE = 16
POOL_K, POOL_V, ACT_Q, ACT_K, ACT_V = 0, 1, 2, 3, 4


@dataclass
class LayerShape:
    num_heads: int          # query heads
    head_dim: int
    k_rank: int
    v_rank: int
    num_kv_heads: int = 0   # 0: as many KV heads as query heads

    @property
    def kv_heads(self) -> int:
        return self.num_kv_heads or self.num_heads


@dataclass
class Workload:
    name: str
    seed: int
    batch: int
    layers: list[LayerShape]
    # context length before the step's append (one new token per sequence)
    ctx_lens: np.ndarray
    append: bool = True
    decoy_frac: float = 0.05
    notes: str = ""
    extra: dict = field(default_factory=dict)

    @property
    def seq_lens(self) -> np.ndarray:
        """Lengths seen by decode (after the append when the step has one)."""
        return self.ctx_lens + (1 if self.append else 0)

    @property
    def max_seq_len(self) -> int:
        return int(self.seq_lens.max()) if self.batch else 0

    @property
    def max_blocks_per_seq(self) -> int:
        return max(1, -(-self.max_seq_len // BLOCK_SIZE))


def _llama_layer(r: int, R: int) -> LayerShape:
    return LayerShape(num_heads=32, head_dim=128, k_rank=r, v_rank=R)


def workload(idx: int) -> Workload:
    """The five benchmark workloads (1-based), plus 6: a grouped-query layer.

    Workload 6 has Llama-3-8B attention heads (32 query heads over 8 KV heads,
    head_dim 128) compressed at the same ratios as the 7B layers (K rank 64 of
    128, V rank 512 of the 1024 concatenated KV-head dims), batch 64 at
    context 8192.
    """
    if idx == 1:
        return Workload("tiny: H4 d64 r16 R64, B2, T{37,100}", 1001, 2,
                        [LayerShape(4, 64, 16, 64)],
                        np.array([37, 100], dtype=np.int64), append=False)
    if idx == 2:
        return Workload("single layer: H32 d128 r64 R2048, B16, T2048", 1002, 16,
                        [_llama_layer(64, 2048)],
                        np.full(16, 2047, dtype=np.int64))
    if idx == 3:
        return Workload("single layer: H32 d128 r64 R2048, B64, T8192", 1003, 64,
                        [_llama_layer(64, 2048)],
                        np.full(64, 8191, dtype=np.int64))
    if idx == 4:
        rng = np.random.default_rng(1004)
        ctx = rng.integers(512, 16384 + 1, size=48).astype(np.int64)
        return Workload("continuous batching: B48, T~U[512,16384], 3 layers r{32,64,96}, R=32r",
                        1004, 48, [_llama_layer(r, 32 * r) for r in (32, 64, 96)], ctx)
    if idx == 5:
        return Workload("Llama-2-7B attention path: 32 layers, B8, T32768, r64 R2048", 1005, 8,
                        [_llama_layer(64, 2048) for _ in range(32)],
                        np.full(8, 32767, dtype=np.int64))
    if idx == 6:
        return Workload("grouped-query layer: H32 Hkv8 d128 r64 R512, B64, T8192", 1006, 64,
                        [LayerShape(32, 128, 64, 512, num_kv_heads=8)],
                        np.full(64, 8191, dtype=np.int64))
    raise ValueError(idx)


def custom(name: str, seed: int, shape: LayerShape, ctx_lens, append=True,
           n_layers: int = 1) -> Workload:
    ctx = np.asarray(ctx_lens, dtype=np.int64)
    return Workload(name, seed, len(ctx), [shape] * n_layers, ctx, append=append)


# ---------------------------------------------------------------- block tables

def block_tables(seed: int, seq_lens: np.ndarray, max_blocks: int,
                 decoy_frac: float = 0.05):
    """Random physical page assignment.

    Returns ``(tables [B][max_blocks] int32, num_blocks, decoys)``.  Every
    sequence gets ``ceil(len/16)`` distinct pages drawn from a seeded
    permutation of the pool; the pool has ``decoy_frac`` extra pages that no
    sequence owns, and table entries past a sequence's last page point at a
    decoy (a valid index whose contents are NaN).
    """
    need = [-(-int(t) // BLOCK_SIZE) for t in seq_lens]
    total = int(sum(need))
    n_decoy = max(1, int(np.ceil(total * decoy_frac)))
    nb = total + n_decoy
    rng = np.random.default_rng(seed + 7919)
    perm = rng.permutation(nb).astype(np.int32)
    owned, decoys = perm[:total], perm[total:]
    tables = np.empty((len(seq_lens), max_blocks), dtype=np.int32)
    pos = 0
    for b, n in enumerate(need):
        tables[b, :n] = owned[pos:pos + n]
        pos += n
        tables[b, n:] = decoys[rng.integers(0, len(decoys), size=max_blocks - n)]
    return tables, nb, decoys


# ----------------------------------------------------------- host-side inputs

def layer_seed(wl: Workload, layer: int) -> int:
    return wl.seed * 1000 + layer


def projections(wl: Workload, layer: int):
    """fp16 projections of one layer: A_K [Hkv][d][r], A_V [Hkv*d][R], B_K [Hkv][r][d], B_V [R][Hkv*d].

    A_K[h] and A_V are the orthonormal Q factors of seeded Gaussians, rounded
    to fp16; B is the transpose of the rounded A.
    """
    sh = wl.layers[layer]
    H, d, r, R = sh.kv_heads, sh.head_dim, sh.k_rank, sh.v_rank
    s = layer_seed(wl, layer)
    A_K = np.stack([gen.orthonormal_f64(s * 131 + h, d, r) for h in range(H)]).astype(np.float16)
    A_V = gen.orthonormal_f64(s * 131 + 977, H * d, R).astype(np.float16)
    B_K = np.ascontiguousarray(np.transpose(A_K, (0, 2, 1)))
    B_V = np.ascontiguousarray(A_V.T)
    return A_K, A_V, B_K, B_V


def activation(wl: Workload, layer: int, which: int) -> np.ndarray:
    """q ([B][H][d], query heads) or k, v ([B][Hkv][d], KV heads) of the step's new token: fp16 ~N(0,1)."""
    sh = wl.layers[layer]
    key = gen.stream_key(wl.seed, layer, which)
    heads = sh.num_heads if which == ACT_Q else sh.kv_heads
    n = heads * sh.head_dim
    return gen.codes_f16(key, wl.batch, n, None).reshape(wl.batch, heads, sh.head_dim)


def code_key(wl: Workload, layer: int, pool: int, b: int) -> int:
    return gen.stream_key(wl.seed, layer, 10 + pool, b)


def k_spectrum(sh: LayerShape) -> np.ndarray:
    return gen.spectrum_f32(sh.k_rank)


def v_spectrum(sh: LayerShape) -> np.ndarray:
    return gen.spectrum_f32(sh.v_rank)


def seq_codes(wl: Workload, layer: int, b: int, n_tokens: int, t0: int = 0):
    """Logical codes of tokens ``t0 .. t0+n_tokens-1`` of sequence ``b``.

    Returns ``(cK [n][Hkv][r], cV [n][R])`` fp16.
    """
    sh = wl.layers[layer]
    H, r, R = sh.kv_heads, sh.k_rank, sh.v_rank
    cK = gen.codes_f16(code_key(wl, layer, POOL_K, b), n_tokens, H * r, k_spectrum(sh),
                       row_offset=t0).reshape(n_tokens, H, r)
    cV = gen.codes_f16(code_key(wl, layer, POOL_V, b), n_tokens, R, v_spectrum(sh),
                       row_offset=t0)
    return cK, cV


def place_host(pool: np.ndarray, table_row: np.ndarray, codes: np.ndarray):
    """Write logical rows ``codes[t]`` into a host pool ``[NB][bs][...]``."""
    T = codes.shape[0]
    for t in range(T):
        pool[table_row[t // BLOCK_SIZE], t % BLOCK_SIZE] = codes[t]


def host_layer(wl: Workload, layer: int, tables=None, nb=None):
    """All inputs of one layer as host numpy arrays (small workloads only).

    Pools hold generated codes for the ``ctx_lens[b]`` context tokens of every
    sequence; every other slot (tails, decoys, the append targets) is fp16 NaN.
    """
    sh = wl.layers[layer]
    H, d, r, R = sh.num_heads, sh.head_dim, sh.k_rank, sh.v_rank
    Hkv = sh.kv_heads
    if tables is None:
        tables, nb, _ = block_tables(wl.seed, wl.seq_lens, wl.max_blocks_per_seq, wl.decoy_frac)
    k_cache = np.full((nb, BLOCK_SIZE, Hkv, r), np.nan, dtype=np.float16)
    v_cache = np.full((nb, BLOCK_SIZE, R), np.nan, dtype=np.float16)
    for b in range(wl.batch):
        T = int(wl.ctx_lens[b])
        cK, cV = seq_codes(wl, layer, b, T)
        place_host(k_cache, tables[b], cK)
        place_host(v_cache, tables[b], cV)
    A_K, A_V, B_K, B_V = projections(wl, layer)
    return dict(
        H=H, Hkv=Hkv, d=d, r=r, R=R, nb=nb, tables=tables,
        ctx_lens=wl.ctx_lens.astype(np.int32), seq_lens=wl.seq_lens.astype(np.int32),
        k_cache=k_cache, v_cache=v_cache,
        q=activation(wl, layer, ACT_Q), k=activation(wl, layer, ACT_K),
        v=activation(wl, layer, ACT_V),
        A_K=A_K, A_V=A_V, B_K=B_K, B_V=B_V, scale=float(1.0 / np.sqrt(d)),
    )
