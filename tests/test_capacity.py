"""Capacity arithmetic against the README's boot-log figures (no GPU)."""
import os

import numpy as np

import rank_compressed_kv_star_b200 as S
from oracle import starkv_oracle as O

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "boot_log_capacity.txt")
GIB = 1 << 30


def _boot_log():
    rows = {}
    for line in open(GOLDEN):
        if line.startswith("#") or not line.strip():
            continue
        name, gib, tokens = line.split()
        rows[name] = (float(gib), int(tokens))
    return rows


def test_uncompressed_7b_boot_log_reproduced():
    gib, tokens = _boot_log()["plain"]
    full = ([32] * 32, [128] * 32, [32 * 128] * 32)          # r = d, R = H*d: full rank
    per_tok = O.kv_bytes_per_token(*full)
    assert per_tok == 32 * 2 * 4096 * 2 == 512 * 1024          # 512 KiB per token
    assert S.starkv_kv_bytes_per_token(*full) == per_tok
    blocks = O.num_blocks(int(gib * GIB), per_tok)
    assert S.starkv_num_blocks(int(gib * GIB), per_tok, 16) == blocks
    assert blocks * 16 == tokens                               # 894 blocks = 14,304 tokens


def test_starkv_boot_logs_are_whole_blocks_of_one_token_size():
    rows = _boot_log()
    per_tok = [gib * GIB / tokens for name, (gib, tokens) in rows.items() if name != "plain"]
    for name, (_, tokens) in rows.items():
        assert tokens % 16 == 0
    # both compressed boot logs imply the same bytes per token (within the
    # two-decimal rounding of the GiB figures): about 165 KiB, 3.1x below 512 KiB
    assert abs(per_tok[0] - per_tok[1]) / per_tok[0] < 1e-3
    assert 164 * 1024 < per_tok[0] < 166 * 1024
    # a profile averaging H*r + R = 2640 codes per layer gives that size
    assert abs(O.kv_bytes_per_token([32] * 32, [40] * 32, [1360] * 32) - per_tok[0]) / per_tok[0] < 1e-3


def test_rank_profile_from_spectra_and_capacity():
    # per-layer ranks by soft-thresholding synthetic spectra, then bytes/token
    taus = [0.2, 0.125, 0.09]
    s_k = np.arange(1, 129, dtype=np.float64) ** -0.5          # exact fp64 spectra
    s_v = np.arange(1, 4097, dtype=np.float64) ** -0.5
    r = [O.rank_from_spectrum(s_k, t) for t in taus]
    R = [O.rank_from_spectrum(s_v, t) for t in taus]
    assert r == [S.starkv_rank_from_spectrum(s_k, t) for t in taus]
    assert r == [24, 63, 123] and R == [24, 63, 123]          # i**-0.5 > tau  <=>  i < tau**-2
    b = O.kv_bytes_per_token([32] * 3, r, R)
    assert S.starkv_kv_bytes_per_token([32] * 3, r, R) == b == 2 * sum(32 * ri + Ri for ri, Ri in zip(r, R))


def test_capacity_helpers_reject_bad_input():
    assert S.starkv_kv_bytes_per_token([], [], []) == -1
    assert S.starkv_kv_bytes_per_token([32], [0], [64]) == -1
    assert S.starkv_num_blocks(-1, 10, 16) == -1
    assert S.starkv_num_blocks(100, 0, 16) == -1
    assert S.starkv_num_blocks(0, 10, 16) == 0


def test_grouped_query_cache_costs_kv_heads_only():
    """With grouped queries a token stores codes per KV head: a Llama-3-8B-shaped model (32 layers of
    8 KV heads, d = 128) costs 2 * 32 * (8*128 + 8*128) bytes per token at full rank, a quarter of
    the 32-head cost, and 2 * 32 * (8*64 + 512) at the 50% ranks of the grouped-query workload."""
    full = ([8] * 32, [128] * 32, [8 * 128] * 32)
    assert O.kv_bytes_per_token(*full) == S.starkv_kv_bytes_per_token(*full) == 2 * 32 * 2048
    assert O.kv_bytes_per_token([32] * 32, [128] * 32, [4096] * 32) == 4 * O.kv_bytes_per_token(*full)
    half = ([8] * 32, [64] * 32, [512] * 32)
    assert O.kv_bytes_per_token(*half) == S.starkv_kv_bytes_per_token(*half) == 2 * 32 * 1024
