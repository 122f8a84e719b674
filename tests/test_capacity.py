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


BLOCKS = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "block_count_table.txt")


def _block_table():
    rows = {}
    for line in open(BLOCKS):
        if line.startswith("#") or not line.strip():
            continue
        name, blocks = line.split()
        rows[name] = int(blocks)
    return rows


def test_block_count_table_756_to_2353():
    """The pages' 756 -> 2353 (3.11x) block counts in one memory budget.

    Plain blocks cost 16 tokens x 512 KiB, so 756 whole blocks pin the budget
    to [756, 757) x 8 MiB.  2353 whole STAR-KV blocks in that budget pin the
    compressed bytes per token to (756*8 MiB / (16*2354), 757*8 MiB /
    (16*2353)], about 164.4-164.7 KiB: 2631-2635 fp16 codes per layer on
    average (H*r + R), a ratio of 3.11 to the 512 KiB of the full cache, within
    0.3% of the ~165 KiB per token of the README's boot logs.  A profile that
    the kernels accept (K ranks multiples of 16, V ranks multiples of 64) falls
    in that interval and reproduces both counts through the capacity helpers.
    """
    t = _block_table()
    plain_tok = O.kv_bytes_per_token([32] * 32, [128] * 32, [4096] * 32)
    assert plain_tok == 512 * 1024
    block = 16 * plain_tok
    lo, hi = t["plain"] * block, (t["plain"] + 1) * block          # budget interval [lo, hi)
    assert O.num_blocks(lo, plain_tok) == S.starkv_num_blocks(lo, plain_tok, 16) == t["plain"]
    assert O.num_blocks(hi - 1, plain_tok) == t["plain"] and O.num_blocks(hi, plain_tok) == t["plain"] + 1
    # per-token bytes b with floor(budget / (16 b)) == 2353 for some budget in [lo, hi)
    b_min, b_max = lo / (16 * (t["starkv"] + 1)), (hi - 1) / (16 * t["starkv"])
    assert 164.4 * 1024 < b_min < b_max < 164.8 * 1024
    ratio = plain_tok / np.array([b_max, b_min])
    assert np.all(np.abs(ratio - 3.11) < 0.005)                      # the printed "3.11x"
    codes_per_layer = np.array([b_min, b_max]) / (2 * 32)
    assert 2630 < codes_per_layer[0] < codes_per_layer[1] < 2636
    boot = _boot_log()
    per_tok_boot = boot["starkv_8192"][0] * GIB / boot["starkv_8192"][1]
    assert abs(per_tok_boot - b_max) / per_tok_boot < 3e-3
    # a kernel-compatible profile: K rank 32 per head in every layer, V ranks
    # 1600 in 28 layers and 1664 in 4 (2 * (32*32*32 + 51456) = 168448 bytes)
    prof = ([32] * 32, [32] * 32, [1600] * 28 + [1664] * 4)
    per_tok = O.kv_bytes_per_token(*prof)
    assert per_tok == S.starkv_kv_bytes_per_token(*prof) == 168448
    assert b_min < per_tok <= b_max
    # budgets giving both printed counts: [lo, min(hi, 2354 * 16 * per_tok)), not empty
    both = (lo, min(hi, (t["starkv"] + 1) * 16 * per_tok))
    assert both[0] < both[1]
    for budget in (both[0], both[1] - 1):
        assert O.num_blocks(budget, plain_tok) == S.starkv_num_blocks(budget, plain_tok, 16) == t["plain"]
        assert O.num_blocks(budget, per_tok) == S.starkv_num_blocks(budget, per_tok, 16) == t["starkv"]
    assert round(t["starkv"] / t["plain"], 2) == 3.11
