"""Pins of the CPU oracle to facts outside itself (no GPU).

The pages print no worked example of the method, so the oracle is pinned by
what the definition and the mathematics fix: full-rank reduction to plain
attention (checked against torch's fp64 scaled-dot-product attention, a
library routine), associativity of the reordered V product, paging
invariances, hand-computable special cases, zero padding of ranks, and
pure-Python brute force on the tiny workload.  The last group plants
plausible mistakes in copies of oracle functions and checks that a pin fails.
"""
import math

import numpy as np
import pytest
import torch

from oracle import starkv_oracle as O
from starkv_inputs import gen, workloads as W


def _orth(rng, n):
    q, r = np.linalg.qr(rng.standard_normal((n, n)))
    return q * np.sign(np.diag(r))


def _paged_fp64(codes_list, tables, nb, row_shape):
    pool = np.full((nb, 16) + row_shape, np.nan)
    for b, c in enumerate(codes_list):
        for t in range(c.shape[0]):
            pool[tables[b][t // 16], t % 16] = c[t]
    return pool


def _full_rank_case(seed=5, H=4, d=16, lens=(1, 19, 40), Hkv=None):
    """Uncompressed K/V, orthogonal A (fp64), B = A^T, codes = k.A exactly.

    ``Hkv`` KV heads (default ``H``) carry K and V; q has ``H`` query heads.
    """
    Hkv = Hkv or H
    rng = np.random.default_rng(seed)
    Bsz = len(lens)
    q = rng.standard_normal((Bsz, H, d))
    k_full = [rng.standard_normal((T, Hkv, d)) for T in lens]
    v_full = [rng.standard_normal((T, Hkv, d)) for T in lens]
    A_K = np.stack([_orth(rng, d) for _ in range(Hkv)])
    A_V = _orth(rng, Hkv * d)
    B_K = np.transpose(A_K, (0, 2, 1)).copy()
    B_V = A_V.T.copy()
    cK = [np.stack([k[:, h, :] @ A_K[h] for h in range(Hkv)], axis=1) for k in k_full]
    cV = [v.reshape(v.shape[0], Hkv * d) @ A_V for v in v_full]
    tables, nb, _ = W.block_tables(seed, np.array(lens), max(1, -(-max(lens) // 16)) + 1)
    kc = _paged_fp64(cK, tables, nb, (Hkv, d))
    vc = _paged_fp64(cV, tables, nb, (Hkv * d,))
    return dict(q=q, k_full=k_full, v_full=v_full, A_K=A_K, A_V=A_V, B_K=B_K, B_V=B_V,
                cK=cK, cV=cV, tables=tables, kc=kc, vc=vc, lens=np.array(lens),
                scale=1.0 / math.sqrt(d))


def _sdpa(q, k_list, v_list, scale):
    """torch fp64 scaled-dot-product attention; grouped query heads when K/V have fewer heads."""
    out = []
    for b in range(q.shape[0]):
        qt = torch.from_numpy(q[b][:, None, :])                     # [H][1][d]
        kt = torch.from_numpy(np.transpose(k_list[b], (1, 0, 2)).copy())  # [Hkv][T][d]
        vt = torch.from_numpy(np.transpose(v_list[b], (1, 0, 2)).copy())
        gqa = kt.shape[0] != qt.shape[0]
        o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=scale,
                                                             enable_gqa=gqa)
        out.append(o[:, 0, :].numpy())
    return np.stack(out)


# ---------------------------------------------------------------- I1 full rank

def check_full_rank(decode=None):
    c = _full_rank_case()
    decode = decode or O.decode_explicit
    got = decode(c["q"], c["B_K"], c["B_V"], c["kc"], c["vc"], c["tables"], c["lens"], c["scale"])
    ref = _sdpa(c["q"], c["k_full"], c["v_full"], c["scale"])
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_full_rank_orthonormal_equals_library_attention():
    check_full_rank()


def check_full_rank_gqa(decode=None):
    """Grouped queries: 8 query heads over 2 KV heads, against torch's own GQA attention."""
    c = _full_rank_case(seed=6, H=8, Hkv=2, lens=(1, 17, 33))
    decode = decode or O.decode_explicit
    got = decode(c["q"], c["B_K"], c["B_V"], c["kc"], c["vc"], c["tables"], c["lens"], c["scale"])
    ref = _sdpa(c["q"], c["k_full"], c["v_full"], c["scale"])
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_full_rank_grouped_query_equals_library_attention():
    check_full_rank_gqa()
    check_full_rank_gqa(O.decode_reordered)


def test_grouped_query_equals_mha_with_repeated_kv_heads():
    """Hkv KV heads shared by groups of H/Hkv query heads == MHA on repeated KV heads."""
    H, Hkv = 8, 2
    G = H // Hkv
    sh = W.LayerShape(H, 32, 16, 64, num_kv_heads=Hkv)
    wl = W.custom("gqa", 91, sh, [1, 16, 45], append=False)
    L = W.host_layer(wl, 0)
    d = L["d"]
    B_K_rep = np.repeat(L["B_K"], G, axis=0)                   # [H][r][d]
    kc_rep = np.repeat(L["k_cache"], G, axis=2)                # [NB][16][H][r]
    B_V_rep = np.concatenate([L["B_V"][:, (h // G) * d:(h // G + 1) * d] for h in range(H)],
                             axis=1)                            # [R][H*d]
    got = O.decode_explicit(L["q"], L["B_K"], L["B_V"], L["k_cache"], L["v_cache"], L["tables"],
                            L["seq_lens"], L["scale"])
    want = O.decode_explicit(L["q"], B_K_rep, B_V_rep, kc_rep, L["v_cache"], L["tables"],
                             L["seq_lens"], L["scale"])
    np.testing.assert_array_equal(got, want)
    np.testing.assert_allclose(
        O.decode_reordered(L["q"], L["B_K"], L["B_V"], L["k_cache"], L["v_cache"], L["tables"],
                           L["seq_lens"], L["scale"]), want, rtol=0, atol=1e-12 * np.abs(want).max())


def check_prefill_causal_full_rank(prefill=None):
    """Chunks over a full-rank cache equal torch's attention with the causal mask of each chunk."""
    H, Hkv, d = 4, 2, 16
    starts, chunks = [0, 7, 30], [5, 9, 1]
    lens = [s + c for s, c in zip(starts, chunks)]
    c = _full_rank_case(seed=12, H=H, Hkv=Hkv, d=d, lens=tuple(lens))
    rng = np.random.default_rng(4)
    q = rng.standard_normal((sum(chunks), H, d))
    prefill = prefill or O.prefill_attention
    got = prefill(q, c["B_K"], c["B_V"], c["kc"], c["vc"], c["tables"], starts, chunks, c["scale"])
    row = 0
    for b, (s0, n) in enumerate(zip(starts, chunks)):
        T = s0 + n
        mask = torch.from_numpy(np.arange(T)[None, :] <= (s0 + np.arange(n))[:, None])      # [n][T]
        qt = torch.from_numpy(np.transpose(q[row:row + n], (1, 0, 2)).copy())                 # [H][n][d]
        kt = torch.from_numpy(np.transpose(c["k_full"][b], (1, 0, 2)).copy())                # [Hkv][T][d]
        vt = torch.from_numpy(np.transpose(c["v_full"][b], (1, 0, 2)).copy())
        ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=c["scale"],
                                                               enable_gqa=True)
        np.testing.assert_allclose(got[row:row + n], np.transpose(ref.numpy(), (1, 0, 2)), rtol=0, atol=1e-12)
        row += n


def test_prefill_causal_full_rank_equals_library_attention():
    check_prefill_causal_full_rank()


def test_prefill_single_token_chunks_equal_decode():
    wl = W.workload(1)
    L = W.host_layer(wl, 0)
    T = L["seq_lens"]
    q = L["q"]
    got = O.prefill_attention(q, L["B_K"], L["B_V"], L["k_cache"], L["v_cache"], L["tables"], T - 1,
                              [1] * wl.batch, L["scale"])
    want = O.decode_explicit(q, L["B_K"], L["B_V"], L["k_cache"], L["v_cache"], L["tables"], T, L["scale"])
    np.testing.assert_array_equal(got, want)


def test_planted_acausal_prefill_is_caught():
    """A chunk token that also sees the next token must fail the causal pin."""
    with pytest.raises(AssertionError):
        check_prefill_causal_full_rank(_leaky_prefill)


def _leaky_prefill(q, B_K, B_V, kc, vc, tables, starts, chunks, scale):
    q = np.asarray(q, float)
    n_rows, H, d = q.shape
    Hkv = np.shape(B_K)[0]
    out = np.zeros((n_rows, H, d))
    row = 0
    for b, n in enumerate(chunks):
        t_end = starts[b] + n
        k_hat = O.decompress_k(O.gather(kc, tables[b], t_end), B_K)
        v_hat = O.decompress_v(O.gather(vc, tables[b], t_end), B_V).reshape(t_end, Hkv, d)
        for i in range(n):
            T = min(t_end, starts[b] + i + 2)          # one token too many
            for h in range(H):
                j = O.kv_head(h, H, Hkv)
                out[row, h] = O.attention_head(q[row, h], k_hat[:T, j], v_hat[:T, j], scale)
            row += 1
    return out


def test_uncompressed_attention_matches_library():
    c = _full_rank_case(seed=9, lens=(3, 33))
    got = O.attention_uncompressed(c["q"], c["k_full"], c["v_full"], c["scale"])
    np.testing.assert_allclose(got, _sdpa(c["q"], c["k_full"], c["v_full"], c["scale"]),
                               rtol=0, atol=1e-13)


# -------------------------------------------------- I2 reordered / absorbed form

@pytest.mark.parametrize("idx", [1])
def test_explicit_equals_reordered_and_stages(idx):
    wl = W.workload(idx)
    L = W.host_layer(wl, 0)
    args = (L["q"], L["B_K"], L["B_V"], L["k_cache"], L["v_cache"], L["tables"],
            L["seq_lens"], L["scale"])
    e = O.decode_explicit(*args)
    r = O.decode_reordered(*args)
    np.testing.assert_allclose(r, e, rtol=0, atol=1e-12 * np.abs(e).max())
    for b in range(wl.batch):
        T = int(L["seq_lens"][b])
        st = O.decode_stages(L["q"][b], L["B_K"], L["B_V"], O.gather(L["k_cache"], L["tables"][b], T),
                             O.gather(L["v_cache"], L["tables"][b], T), L["scale"])
        np.testing.assert_allclose(st["o"], e[b], rtol=0, atol=1e-12 * np.abs(e).max())
        np.testing.assert_allclose(st["p"].sum(axis=1), 1.0, atol=1e-14)


def test_explicit_equals_reordered_midsize():
    sh = W.LayerShape(8, 32, 16, 128)
    wl = W.custom("mid", 77, sh, [1, 15, 16, 17, 250], append=False)
    L = W.host_layer(wl, 0)
    args = (L["q"], L["B_K"], L["B_V"], L["k_cache"], L["v_cache"], L["tables"],
            L["seq_lens"], L["scale"])
    e = O.decode_explicit(*args)
    np.testing.assert_allclose(O.decode_reordered(*args), e, rtol=0, atol=1e-12 * np.abs(e).max())


# ------------------------------------------------------------- I3 / I4 paging

def test_page_permutation_and_relabel_bit_identical():
    wl = W.workload(1)
    L = W.host_layer(wl, 0)
    args = (L["q"], L["B_K"], L["B_V"])
    base = O.decode_explicit(*args, L["k_cache"], L["v_cache"], L["tables"], L["seq_lens"], L["scale"])
    perm = np.random.default_rng(3).permutation(L["nb"])       # new page id of old page i = perm[i]
    kc = np.empty_like(L["k_cache"])
    vc = np.empty_like(L["v_cache"])
    kc[perm] = L["k_cache"]
    vc[perm] = L["v_cache"]
    tables = perm[L["tables"]].astype(np.int32)
    got = O.decode_explicit(*args, kc, vc, tables, L["seq_lens"], L["scale"])
    assert np.array_equal(got, base)


def check_contiguous_equals_paged(gather=None):
    wl = W.workload(1)
    L = W.host_layer(wl, 0)
    cK, cV = [], []
    for b in range(wl.batch):
        k, v = W.seq_codes(wl, 0, b, int(L["seq_lens"][b]))
        cK.append(k.astype(np.float64))
        cV.append(v.astype(np.float64))
    cont = O.decode_contiguous(L["q"], L["B_K"], L["B_V"], cK, cV, L["scale"])
    paged = O.decode_explicit(L["q"], L["B_K"], L["B_V"], L["k_cache"], L["v_cache"],
                              L["tables"], L["seq_lens"], L["scale"])
    assert np.array_equal(cont, paged)


def test_contiguous_equals_paged():
    check_contiguous_equals_paged()


def test_gather_by_hand():
    cache = np.arange(4 * 16, dtype=np.float64).reshape(4, 16, 1)   # value = page*16 + slot
    row = np.array([2, 0, 3], dtype=np.int32)
    got = O.gather(cache, row, 35)[:, 0]
    want = [2 * 16 + t for t in range(16)] + [0 * 16 + t for t in range(16)] + [3 * 16 + t for t in range(3)]
    assert got.tolist() == want


# ------------------------------------------------------------ I5 special cases

def _one_seq_case(T, seed=11, H=2, d=8, r=4, R=8):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((1, H, d))
    B_K = rng.standard_normal((H, r, d))
    B_V = rng.standard_normal((R, H * d))
    cK = rng.standard_normal((T, H, r))
    cV = rng.standard_normal((T, R))
    tables = np.arange(-(-T // 16), dtype=np.int32)[None, :]
    kc = _paged_fp64([cK], tables, tables.shape[1], (H, r))
    vc = _paged_fp64([cV], tables, tables.shape[1], (R,))
    return q, B_K, B_V, cK, cV, tables, kc, vc


def test_single_token_returns_its_value():
    q, B_K, B_V, cK, cV, tables, kc, vc = _one_seq_case(1)
    o = O.decode_explicit(q, B_K, B_V, kc, vc, tables, [1], 0.3)
    vhat = (cV[0] @ B_V).reshape(2, 8)
    assert np.array_equal(o[0], vhat)


def test_zero_query_gives_mean_value():
    q, B_K, B_V, cK, cV, tables, kc, vc = _one_seq_case(37)
    o = O.decode_explicit(np.zeros_like(q), B_K, B_V, kc, vc, tables, [37], 0.3)
    vhat = (cV @ B_V).reshape(37, 2, 8)
    np.testing.assert_allclose(o[0], vhat.mean(axis=0), rtol=0, atol=1e-14)


def test_identical_codes_give_that_value():
    q, B_K, B_V, cK, cV, tables, kc, vc = _one_seq_case(21)
    kc[:] = cK[0]
    vc[:] = cV[0]
    o = O.decode_explicit(q, B_K, B_V, kc, vc, tables, [21], 0.3)
    np.testing.assert_allclose(o[0], (cV[0] @ B_V).reshape(2, 8), rtol=0, atol=1e-14)


@pytest.mark.parametrize("delta", [-3.0, 0.0, 0.7, 12.0])
def test_two_token_logit_gap_gives_sigmoid_weights(delta):
    # identity projections (r = d, R = H*d): codes are the keys/values themselves
    H, d = 1, 4
    scale = 0.5
    q = np.zeros((1, H, d)); q[0, 0, 0] = 1.0
    k = np.zeros((2, H, d)); k[0, 0, 0] = delta / scale
    v = np.array([[[1.0, 2.0, 3.0, 4.0]], [[-1.0, 0.5, 0.0, 2.0]]])
    tables = np.array([[0]], dtype=np.int32)
    kc = _paged_fp64([k], tables, 1, (H, d))
    vc = _paged_fp64([v.reshape(2, H * d)], tables, 1, (H * d,))
    o = O.decode_explicit(q, np.eye(d)[None], np.eye(H * d), kc, vc, tables, [2], scale)
    w0 = 1.0 / (1.0 + math.exp(-delta))
    want = w0 * v[0, 0] + (1.0 - w0) * v[1, 0]
    np.testing.assert_allclose(o[0, 0], want, rtol=1e-14, atol=1e-15)


def test_empty_sequence_gives_zero_row():
    q, B_K, B_V, cK, cV, tables, kc, vc = _one_seq_case(5)
    o = O.decode_explicit(q, B_K, B_V, kc, vc, tables, [0], 0.3)
    assert np.array_equal(o, np.zeros_like(o))


# ------------------------------------------------------------ I6 zero padding

def test_zero_padding_of_ranks_leaves_output_unchanged():
    wl = W.workload(1)
    L = W.host_layer(wl, 0)
    H, d, r, R = L["H"], L["d"], L["r"], L["R"]
    base = O.decode_explicit(L["q"], L["B_K"], L["B_V"], L["k_cache"], L["v_cache"],
                             L["tables"], L["seq_lens"], L["scale"])
    B_K = np.concatenate([L["B_K"], np.zeros((H, 16, d), np.float16)], axis=1)
    B_V = np.concatenate([L["B_V"], np.zeros((16, H * d), np.float16)], axis=0)
    kc = np.concatenate([L["k_cache"], np.zeros(L["k_cache"].shape[:3] + (16,), np.float16)], axis=3)
    vc = np.concatenate([L["v_cache"], np.zeros(L["v_cache"].shape[:2] + (16,), np.float16)], axis=2)
    got = O.decode_explicit(L["q"], B_K, B_V, kc, vc, L["tables"], L["seq_lens"], L["scale"])
    np.testing.assert_allclose(got, base, rtol=0, atol=1e-13 * np.abs(base).max())


# ---------------------------------------------------------- I7 append (brute)

def test_append_brute_force_and_placement():
    sh = W.LayerShape(4, 64, 16, 64)
    wl = W.custom("append", 31, sh, [37, 100, 0, 15], append=True)
    L = W.host_layer(wl, 0)
    pos = L["ctx_lens"]
    cK, cV, kc, vc = O.compress_append(L["k"], L["v"], L["A_K"], L["A_V"], L["tables"], pos,
                                       L["k_cache"], L["v_cache"])
    k, v = L["k"].astype(float), L["v"].astype(float)
    A_K, A_V = L["A_K"].astype(float), L["A_V"].astype(float)
    for b in range(wl.batch):
        for h in range(sh.num_heads):
            for i in range(sh.k_rank):
                want = math.fsum(k[b, h, j] * A_K[h, j, i] for j in range(sh.head_dim))
                assert abs(cK[b, h, i] - want) <= 1e-13
        vflat = v[b].reshape(-1)
        for i in range(sh.v_rank):
            want = math.fsum(vflat[j] * A_V[j, i] for j in range(vflat.shape[0]))
            assert abs(cV[b, i] - want) <= 1e-13
    # exactly the target slots changed, to the fp16-rounded codes
    changed_k = np.argwhere(~((kc == L["k_cache"]) | (np.isnan(kc) & np.isnan(L["k_cache"]))).all(axis=(2, 3)))
    targets = sorted((int(L["tables"][b][pos[b] // 16]), int(pos[b] % 16)) for b in range(wl.batch))
    assert sorted(map(tuple, changed_k.tolist())) == targets
    for b in range(wl.batch):
        pg, sl = L["tables"][b][pos[b] // 16], pos[b] % 16
        assert np.array_equal(kc[pg, sl].view(np.uint16), cK[b].astype(np.float16).view(np.uint16))
        assert np.array_equal(vc[pg, sl].view(np.uint16), cV[b].astype(np.float16).view(np.uint16))
    untouched_v = vc.copy()
    for (pg, sl) in targets:
        untouched_v[pg, sl] = L["v_cache"][pg, sl]
    assert np.array_equal(untouched_v.view(np.uint16), L["v_cache"].view(np.uint16))


# ------------------------------------------------------- I8 brute force (tiny)

def _brute_decode(L):
    """Independent pure-Python evaluation of the definition (triple loops)."""
    H, d, r, R = L["H"], L["d"], L["r"], L["R"]
    q = L["q"].astype(float).tolist()
    B_K = L["B_K"].astype(float).tolist()
    B_V = L["B_V"].astype(float).tolist()
    kc, vc, tables = L["k_cache"], L["v_cache"], L["tables"]
    scale = 1.0 / math.sqrt(d)
    out = []
    for b in range(len(q)):
        T = int(L["seq_lens"][b])
        rows_k, rows_v = [], []
        for t in range(T):
            page, slot = int(tables[b][t // 16]), t % 16
            rows_k.append(kc[page, slot].astype(float).tolist())
            rows_v.append(vc[page, slot].astype(float).tolist())
        ob = []
        for h in range(H):
            logits = []
            vhat = []
            for t in range(T):
                khat = [math.fsum(rows_k[t][h][i] * B_K[h][i][j] for i in range(r)) for j in range(d)]
                logits.append(scale * math.fsum(khat[j] * q[b][h][j] for j in range(d)))
                vhat.append([math.fsum(rows_v[t][i] * B_V[i][h * d + j] for i in range(R))
                             for j in range(d)])
            mx = max(logits)
            e = [math.exp(a - mx) for a in logits]
            s = math.fsum(e)
            ob.append([math.fsum(e[t] / s * vhat[t][j] for t in range(T)) for j in range(d)])
        out.append(ob)
    return np.array(out)


def check_brute_force(decode=None):
    wl = W.workload(1)
    L = W.host_layer(wl, 0)
    decode = decode or O.decode_explicit
    got = decode(L["q"], L["B_K"], L["B_V"], L["k_cache"], L["v_cache"], L["tables"],
                 L["seq_lens"], L["scale"])
    want = _brute_decode(L)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-13 * np.abs(want).max())


def test_brute_force_tiny_workload():
    check_brute_force()


# ------------------------------------------------------------ rank selection

def test_rank_from_spectrum():
    s = gen.spectrum_f32(64).astype(np.float64)               # i**-0.5
    assert O.rank_from_spectrum(s, 0.0) == 64
    assert O.rank_from_spectrum(s, 1.0) == 0                  # strictly above
    assert O.rank_from_spectrum(s, 0.25) == 15                # i**-0.5 > 1/4  <=>  i < 16
    assert O.rank_from_spectrum(s, 0.125 + 1e-12) == 63       # i < 64
    assert O.rank_from_spectrum([], 0.5) == 0
    assert O.rank_from_spectrum([3.0, 2.0, 2.0, 1.0], 2.0) == 1


# --------------------------------------------------- planted mistakes (CPU)

def _mut_scale_by_rank(q, B_K, B_V, kc, vc, tables, seq_lens, scale):
    r = np.asarray(B_K).shape[1]
    return O.decode_explicit(q, B_K, B_V, kc, vc, tables, seq_lens, 1.0 / math.sqrt(r))


def _mut_strided_heads(q, B_K, B_V, kc, vc, tables, seq_lens, scale):
    q = np.asarray(q, float)
    Bsz, H, d = q.shape
    out = np.zeros((Bsz, H, d))
    for b in range(Bsz):
        T = int(seq_lens[b])
        k_hat = O.decompress_k(O.gather(kc, tables[b], T), B_K)
        v_hat = O.decompress_v(O.gather(vc, tables[b], T), B_V)
        for h in range(H):
            out[b, h] = O.attention_head(q[b, h], k_hat[:, h], v_hat[:, h::H], scale)
    return out


def _mut_untransposed_bk(q, B_K, B_V, kc, vc, tables, seq_lens, scale):
    return O.decode_explicit(q, np.transpose(np.asarray(B_K), (0, 2, 1)), B_V, kc, vc, tables,
                             seq_lens, scale)


def _mut_unnormalised(q, B_K, B_V, kc, vc, tables, seq_lens, scale):
    orig = O.softmax
    try:
        O.softmax = lambda a: np.exp(a - a.max(axis=-1, keepdims=True))
        return O.decode_explicit(q, B_K, B_V, kc, vc, tables, seq_lens, scale)
    finally:
        O.softmax = orig


def _mut_slot_shift(cache, table_row, T):
    out = np.empty((T,) + cache.shape[2:])
    for t in range(T):
        out[t] = cache[table_row[(t + 1) // 16], (t + 1) % 16]
    return out


@pytest.mark.parametrize("mutant,pin", [
    (_mut_scale_by_rank, check_brute_force),
    (_mut_strided_heads, check_full_rank),
    (_mut_untransposed_bk, check_full_rank),
    (_mut_unnormalised, check_brute_force),
])
def test_planted_decode_mistakes_are_caught(mutant, pin):
    with pytest.raises(AssertionError):
        pin(mutant)


def test_planted_interleaved_kv_heads_are_caught(monkeypatch):
    """Query head h reading KV head h % Hkv (interleaved groups) instead of h // G."""
    monkeypatch.setattr(O, "kv_head", lambda h, H, Hkv: h % Hkv)
    with pytest.raises(AssertionError):
        check_full_rank_gqa()


def test_planted_slot_mistake_is_caught(monkeypatch):
    monkeypatch.setattr(O, "gather", _mut_slot_shift)
    with pytest.raises((AssertionError, IndexError)):
        check_contiguous_equals_paged()


def test_slot_mapped_store_equals_block_table_append():
    sh = W.LayerShape(4, 64, 16, 64)
    wl = W.custom("store", 41, sh, [37, 100, 0, 15], append=True)
    L = W.host_layer(wl, 0)
    pos = L["ctx_lens"]
    slots = [int(L["tables"][b][pos[b] // 16]) * 16 + int(pos[b] % 16) for b in range(wl.batch)]
    a = O.compress_append(L["k"], L["v"], L["A_K"], L["A_V"], L["tables"], pos, L["k_cache"], L["v_cache"])
    s = O.compress_store(L["k"], L["v"], L["A_K"], L["A_V"], slots, L["k_cache"], L["v_cache"])
    for x, y in zip(a[2:], s[2:]):
        assert np.array_equal(x.view(np.uint16), y.view(np.uint16))


def test_grouped_query_store_equals_append_and_contiguous_equals_paged():
    """With 2 KV heads under 8 query heads: slot-mapped store == block-table append (bitwise), and
    decode over contiguous code arrays == decode through the block tables (bitwise)."""
    sh = W.LayerShape(8, 32, 16, 64, num_kv_heads=2)
    wl = W.custom("gqa-store", 43, sh, [37, 100, 0, 15], append=True)
    L = W.host_layer(wl, 0)
    pos = L["ctx_lens"]
    slots = [int(L["tables"][b][pos[b] // 16]) * 16 + int(pos[b] % 16) for b in range(wl.batch)]
    a = O.compress_append(L["k"], L["v"], L["A_K"], L["A_V"], L["tables"], pos, L["k_cache"], L["v_cache"])
    s = O.compress_store(L["k"], L["v"], L["A_K"], L["A_V"], slots, L["k_cache"], L["v_cache"])
    for x, y in zip(a[2:], s[2:]):
        assert np.array_equal(x.view(np.uint16), y.view(np.uint16))
    kc, vc = a[2], a[3]
    T = L["seq_lens"]
    paged = O.decode_explicit(L["q"], L["B_K"], L["B_V"], kc, vc, L["tables"], T, L["scale"])
    contig = O.decode_contiguous(L["q"], L["B_K"], L["B_V"],
                                 [O.gather(kc, L["tables"][b], int(T[b])) for b in range(wl.batch)],
                                 [O.gather(vc, L["tables"][b], int(T[b])) for b in range(wl.batch)], L["scale"])
    assert np.array_equal(paged, contig)
