"""The C-ABI library without a GPU: it loads, exports every declared entry point
and rejects bad arguments on the host before any launch."""
import ctypes
import os
import re

import numpy as np
import pytest

import rank_compressed_kv_star_b200 as S
from oracle import starkv_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from rank_compressed_kv_star_b200 import build
    build.build()
    return S.load_library()


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "starkv.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(starkv_[a-z_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_symbols()
    assert len(names) >= 8
    for n in names:
        assert hasattr(lib, n), n
    assert set(S.EXPORTED) <= set(names)


def test_status_strings_and_version(lib):
    for code, name in S.STATUS.items():
        assert S.starkv_status_string(code) == name
    assert S.starkv_version() >= 100


def test_rank_from_spectrum_matches_oracle(lib):
    rng = np.random.default_rng(0)
    for _ in range(50):
        s = np.sort(rng.random(rng.integers(0, 80)))[::-1]
        tau = float(rng.random())
        assert S.starkv_rank_from_spectrum(s, tau) == O.rank_from_spectrum(s, tau)
    assert lib.starkv_rank_from_spectrum(None, -1, 0.0) == -1
    assert S.starkv_rank_from_spectrum([1.0], float("nan")) == -1


def _desc(**kw):
    base = dict(num_heads=32, head_dim=128, k_rank=64, v_rank=2048, num_blocks=1000,
                max_blocks_per_seq=64)
    base.update(kw)
    return S.layer_desc(**base)


@pytest.mark.parametrize("kw,expect", [
    (dict(block_size=32), 2), (dict(num_heads=48), 2), (dict(head_dim=96), 2),
    (dict(k_rank=40), 2), (dict(v_rank=100), 2), (dict(num_heads=0), 1), (dict(num_blocks=0), 1),
    (dict(k_rank=272), 2), (dict(v_rank=8256), 2),
])
def test_descriptor_validation(lib, kw, expect):
    d = _desc(**kw)
    fake = 1 << 20
    st = S.starkv_paged_decode(d, 1, 16, fake, fake, fake, fake, fake, fake, fake, 0.1, fake,
                               1 << 30, fake, stream=0, check=False)
    assert st == expect
    assert S.starkv_decode_workspace_bytes(d, 1, 16) == 0
    st = S.starkv_compress_append(d, 1, fake, fake, fake, fake, fake, fake, fake, fake, stream=0,
                                  check=False)
    assert st == expect


def test_decode_argument_errors(lib):
    d = _desc()
    fake = 1 << 20
    need = S.starkv_decode_workspace_bytes(d, 4, 1024)
    assert need > 0
    args = [d, 4, 1024, fake, fake, fake, fake, fake, fake, fake, 0.1, fake, need, fake]
    def call(i, v):
        a = list(args); a[i] = v
        return S.starkv_paged_decode(*a, stream=0, check=False)
    assert call(1, -1) == 1                      # negative batch
    assert call(2, 64 * 16 + 1) == 1             # max_seq_len above table capacity
    assert call(10, 0.0) == 1 and call(10, float("inf")) == 1
    assert call(3, None) == 1                    # null q
    assert call(3, fake + 2) == 1                # misaligned q
    assert call(12, need - 1) == 3               # workspace too small
    a = list(args); a[1] = 0; a[11] = None       # empty batch without a workspace: a no-op
    assert S.starkv_paged_decode(*a, stream=0, check=False) == 0
    assert call(11, None) == 3                   # null workspace
    assert call(11, fake + 128) == 3             # workspace not 256-byte aligned
    assert S.starkv_paged_decode(None, 4, 1024, *args[3:], stream=0, check=False) == 1


def test_append_argument_errors(lib):
    d = _desc()
    fake = 1 << 20
    args = [d, 4, fake, fake, fake, fake, fake, fake, fake, fake]
    for i in range(2, 10):
        a = list(args); a[i] = None
        assert S.starkv_compress_append(*a, stream=0, check=False) == 1
    a = list(args); a[1] = -3
    assert S.starkv_compress_append(*a, stream=0, check=False) == 1
    a = list(args); a[1] = 0
    assert S.starkv_compress_append(*a, stream=0, check=False) == 0   # empty batch: no-op
    a = list(args)                                                      # misaligned status word
    assert S.starkv_compress_append(*a, stream=0, check=False, status=fake + 2) == 1


def test_workspace_layout_is_consistent(lib):
    d = _desc(max_blocks_per_seq=600, num_blocks=40000)
    lay = S.starkv_decode_workspace_layout(d, 64, 8192)
    assert lay.total_bytes == S.starkv_decode_workspace_bytes(d, 64, 8192)
    offs = [lay.status_off, lay.prefix_off, lay.qt_off, lay.logits_off, lay.mpart_off,
            lay.lpart_off, lay.zpart_off]
    assert offs == sorted(offs) and all(o % 256 == 0 for o in offs)
    assert lay.t_pad == 8192 and lay.k_slots == 64 and lay.v_slots == lay.v_ctas + 64
    assert lay.n_rranges * lay.r_range >= 2048
    assert lay.logits_off + 64 * 8192 * 32 * 4 <= lay.mpart_off
    # grows with batch and length
    assert S.starkv_decode_workspace_bytes(d, 65, 8192) > lay.total_bytes
    assert S.starkv_decode_workspace_bytes(d, 64, 8200) > lay.total_bytes


def test_compress_store_argument_errors(lib):
    d = _desc()
    fake = 1 << 20
    args = [d, 8, fake, fake, fake, fake, fake, fake, fake]
    a = list(args); a[6] = None                    # no slot mapping
    assert S.starkv_compress_store(*a, stream=0, check=False) == 1
    a = list(args); a[6] = fake + 2                # misaligned slot mapping
    assert S.starkv_compress_store(*a, stream=0, check=False) == 1
    a = list(args); a[1] = 0
    assert S.starkv_compress_store(*a, stream=0, check=False) == 0
    assert S.starkv_compress_store(_desc(block_size=8), *args[1:], stream=0, check=False) == 2


@pytest.mark.parametrize("kv,expect", [(-1, 1), (12, 2), (64, 2), (3, 2)])
def test_kv_head_count_validation(lib, kv, expect):
    d = _desc(num_kv_heads=kv)
    fake = 1 << 20
    st = S.starkv_paged_decode(d, 1, 16, fake, fake, fake, fake, fake, fake, fake, 0.1, fake,
                               1 << 30, fake, stream=0, check=False)
    assert st == expect
    assert S.starkv_decode_workspace_bytes(d, 1, 16) == 0


def test_prefill_argument_errors(lib):
    d = _desc()
    fake = 1 << 20
    need = S.starkv_prefill_workspace_bytes(d, 2, 40, 1024)
    assert need > S.starkv_decode_workspace_bytes(d, 40, 1024) > 0
    args = [d, 2, 40, 1024, fake, fake, fake, fake, fake, fake, fake, fake, 0.1, fake, need, fake]

    def call(i, v):
        a = list(args); a[i] = v
        return S.starkv_paged_prefill(*a, stream=0, check=False)
    assert call(1, -1) == 1                      # negative sequence count
    assert call(2, -5) == 1                      # negative row count
    assert call(1, 0) == 1                       # rows but no sequences
    assert call(10, None) == 1                   # null starts
    assert call(11, fake + 2) == 1               # misaligned row offsets
    assert call(14, need - 1) == 3               # workspace too small for the row arrays
    assert call(3, 64 * 16 + 1) == 1             # length bound above table capacity
    a = list(args); a[2] = 0; a[13] = None       # no rows and no workspace: a no-op
    assert S.starkv_paged_prefill(*a, stream=0, check=False) == 0
    a = list(args); a[2] = 0; a[13] = fake + 128  # no rows, misaligned workspace: refused
    assert S.starkv_paged_prefill(*a, stream=0, check=False) == 3
    assert S.starkv_prefill_workspace_bytes(d, 2, -1, 1024) == 0
    assert S.starkv_prefill_workspace_bytes(d, -1, 40, 1024) == 0


def test_wait_test_hook_rejects_bad_stage(lib):
    assert S.starkv_set_wait_test_hook(0, -2, check=False) == 1


def test_host_step_argument_errors(lib):
    """starkv_append_decode_host refuses bad arguments before it enqueues any copy."""
    d = _desc()
    fake = 1 << 20
    stg = S.starkv_host_staging_bytes(d, 4)
    ws = S.starkv_decode_workspace_bytes(d, 4, 1024)
    assert stg >= 4 * 32 * 128 * 2 * 4 and ws > 0
    args = [d, 4, 1024] + [fake] * 6 + [fake] * 6 + [0.1, fake, stg, fake, ws, fake]

    def call(i, v):
        a = list(args); a[i] = v
        return S.starkv_append_decode_host(*a, stream=0, check=False)
    # indices: 3..8 host k, v, positions, q, tables, lengths; 9..14 device A_K, A_V, B_K, B_V, pools;
    # 15 scale, 16/17 staging and its size, 18/19 workspace and its size, 20 host out
    assert call(3, None) == 1                    # no host k
    assert call(20, None) == 1                   # no host output
    assert call(17, stg - 1) == 3                # staging too small
    assert call(16, fake + 64) == 3              # staging not 256-byte aligned
    assert call(19, ws - 1) == 3                 # workspace too small
    assert call(2, 64 * 16 + 1) == 1             # length bound above table capacity
    assert call(15, float("nan")) == 1           # bad scale
    assert call(9, None) == 1 and call(13, fake + 8) == 1   # no A_K; misaligned K pool
    assert S.starkv_host_staging_bytes(_desc(block_size=8), 4) == 0
