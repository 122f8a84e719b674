"""Seeded input generator: published-definition vectors and distribution checks (no GPU)."""
import numpy as np

from starkv_inputs import gen, workloads as W


def test_splitmix64_published_sequence():
    # SplitMix64 (Steele/Lea/Flood 2014; Vigna's splitmix64.c) seeded with
    # 1234567: the first five outputs of the reference generator.
    s = 1234567
    got = [gen.mix64_int(s + i * gen.GOLDEN) for i in range(1, 6)]
    assert got == [6457827717110365317, 3203168211198807973, 9817491932198370423,
                   4593380528125082431, 16408922859458223821]
    assert gen.mix64_int(gen.GOLDEN) == 0xE220A8397B1DCDAF


def test_array_and_scalar_paths_agree():
    key = gen.stream_key(1, 2, 3)
    z = gen.normal_f32(key, 64)
    for i in range(64):
        x = gen.mix64_int(key + (i + 1) * gen.GOLDEN)
        s = sum((x >> (16 * f)) & 0xFFFF for f in range(4)) - gen.IH4_CENTER
        assert z[i] == np.float32(np.float32(s) * gen.IH4_SCALE)


def test_normal_moments_and_bounds():
    z = gen.normal_f32(gen.stream_key(42), 1 << 20).astype(np.float64)
    assert abs(z.mean()) < 5e-3
    assert abs(z.var() - 1.0) < 5e-3
    assert np.abs(z).max() <= np.sqrt(12.0) + 1e-6


def test_offsets_are_slices_of_one_stream():
    key = gen.stream_key(7, 0, 11, 3)
    spec = gen.spectrum_f32(16)
    full = gen.codes_f16(key, 40, 32, spec)
    part = gen.codes_f16(key, 9, 32, spec, row_offset=17)
    assert np.array_equal(full[17:26].view(np.uint16), part.view(np.uint16))


def test_spectrum_and_keys():
    s = gen.spectrum_f32(4)
    assert s.dtype == np.float32 and s[0] == 1.0 and s[3] == np.float32(0.5)
    assert len({gen.stream_key(1, 0, p, b) for p in range(3) for b in range(50)}) == 150


def test_block_tables_structure():
    lens = np.array([1, 16, 17, 100, 0])
    tables, nb, decoys = W.block_tables(5, lens, 8)
    need = [-(-int(t) // 16) for t in lens]
    owned = np.concatenate([tables[b, :n] for b, n in enumerate(need)])
    assert len(set(owned.tolist())) == len(owned) == sum(need)     # distinct pages
    assert set(decoys.tolist()).isdisjoint(owned.tolist())
    for b, n in enumerate(need):
        assert set(tables[b, n:].tolist()) <= set(decoys.tolist())
    assert tables.min() >= 0 and tables.max() < nb


def test_workload_shapes():
    for i in range(1, 6):
        wl = W.workload(i)
        assert wl.batch == len(wl.ctx_lens)
    wl = W.workload(4)
    assert 512 <= wl.ctx_lens.min() and wl.ctx_lens.max() <= 16384
    assert [s.k_rank for s in wl.layers] == [32, 64, 96]
    assert [s.v_rank for s in wl.layers] == [1024, 2048, 3072]
