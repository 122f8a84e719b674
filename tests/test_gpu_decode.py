"""GPU parity of the C-ABI path against the CPU fp64 oracle (B200, sm_100a):
edge cases, paging invariances, shapes, errors, chunked prefill, graphs.

The graded workloads, append bit-exactness and grouped-query parity run
first, from test_gpu_0_graded.py.  Tolerances are stated in ``gpu_common``:
decode max |err| <= 2e-3 and relative L2 <= 1e-3; paging invariances (page
permutation, identity vs shuffled table) are bit-exact.
"""
import numpy as np
import pytest
import torch

import rank_compressed_kv_star_b200 as S
from oracle import starkv_oracle as O
from starkv_inputs import device as D, gen, workloads as W
from gpu_common import (MAX_ABS, REL_L2, POISON, append_check, assert_close, desc_of, full_check, load,
                        oracle_rows, rel_l2, run_decode)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built(cuda_ok):
    load()


# ------------------------------------------------------------- generator twin

def test_device_generator_matches_host_bits():
    spec = gen.spectrum_f32(64)
    for key, rows, row_len, off in [(gen.stream_key(1, 2), 37, 64 * 4, 0),
                                    (gen.stream_key(9), 5, 2048, 123), (123456789, 3, 64, 1 << 20)]:
        out = torch.empty(rows * row_len, dtype=torch.float16, device="cuda")
        D.gen_codes(key, rows, row_len, torch.from_numpy(spec).cuda(), out, row_offset=off)
        host = gen.codes_f16(key, rows, row_len, spec, row_offset=off)
        assert np.array_equal(out.cpu().numpy().view(np.uint16), host.reshape(-1).view(np.uint16))


def test_device_pools_match_host_pools():
    wl = W.workload(1)
    Lh = W.host_layer(wl, 0)
    Ld = D.device_layer(wl, 0, tables=Lh["tables"], nb=Lh["nb"])
    assert np.array_equal(Ld["k_cache"].cpu().numpy().view(np.uint16), Lh["k_cache"].view(np.uint16))
    assert np.array_equal(Ld["v_cache"].cpu().numpy().view(np.uint16), Lh["v_cache"].view(np.uint16))


# ------------------------------------------------------------------ decode

@pytest.mark.parametrize("gqa", [False, True])
def test_decode_tiny_intermediates(gqa):
    """Logits, per-sequence maxima and softmax normaliser against the oracle's stages.

    The grouped-query case (8 query heads over 2 KV heads) runs the tensor-core K pass.
    """
    wl = (W.custom("tiny-gqa", 1011, W.LayerShape(8, 64, 16, 128, num_kv_heads=2), [37, 100, 290],
                   append=False) if gqa else W.workload(1))
    Lh = W.host_layer(wl, 0)
    Ld = D.device_layer(wl, 0, tables=Lh["tables"], nb=Lh["nb"])
    got, ws, desc = run_decode(Ld)
    lay = S.starkv_decode_workspace_layout(desc, wl.batch, wl.max_seq_len)
    assert lay.k_tensor == (1 if gqa else 0)
    wsn = ws.cpu().numpy()
    H = Lh["H"]
    f32 = lambda off, n: wsn[off:off + 4 * n].view(np.float32)
    logits = f32(lay.logits_off, wl.batch * lay.t_pad * H).reshape(wl.batch, lay.t_pad, H)
    mpart = f32(lay.mpart_off, lay.k_slots * H).reshape(lay.k_slots, H)
    lpart = f32(lay.lpart_off, lay.v_slots * H).reshape(lay.v_slots, H)
    prefix = wsn[lay.prefix_off:lay.prefix_off + 4 * (wl.batch + 1)].view(np.int32)
    P = int(prefix[-1])
    Gv = min(lay.v_ctas, P)
    assert lay.k_slots == wl.batch
    owner = lambda x, G: min(G - 1, ((x + 1) * G + P - 1) // P - 1)
    for b in range(wl.batch):
        T = int(Lh["seq_lens"][b])
        st = O.decode_stages(Lh["q"][b], Lh["B_K"], Lh["B_V"], O.gather(Lh["k_cache"], Lh["tables"][b], T),
                             O.gather(Lh["v_cache"], Lh["tables"][b], T), Lh["scale"])
        s2 = st["s"] * np.log2(np.e)             # base-2 logits [H][T]
        np.testing.assert_allclose(logits[b, :T].T, s2, rtol=0, atol=1e-4)
        M = s2.max(axis=1)
        np.testing.assert_allclose(mpart[b], M, rtol=0, atol=1e-4)
        Lsum = np.exp2(s2 - M[:, None]).sum(axis=1)
        segs = range(owner(int(prefix[b]), Gv), owner(int(prefix[b + 1]) - 1, Gv) + 1)
        Lgpu = sum(lpart[b + i] for i in segs)
        np.testing.assert_allclose(Lgpu, Lsum, rtol=2e-3)


def test_decode_ragged_multitile():
    sh = W.LayerShape(32, 128, 64, 2048)
    wl = W.custom("ragged", 2024, sh, [1, 15, 16, 17, 300, 0, 1000], append=False)
    full_check(wl)


@pytest.mark.parametrize("r,R", [(32, 1024), (96, 3072), (16, 64), (128, 512)])
def test_decode_rank_variants(r, R):
    sh = W.LayerShape(32, 128, r, R)
    wl = W.custom(f"r{r}", 300 + r, sh, [5, 33, 160, 511], append=False)
    full_check(wl)


def test_decode_largest_head_dim_and_k_rank():
    """head_dim 256 and K rank 256 (the largest the kernels take), V rank 4096, ragged lengths."""
    sh = W.LayerShape(16, 256, 256, 4096)
    wl = W.custom("d256", 256, sh, [1, 17, 100], append=False)
    full_check(wl)


def test_decode_small_heads_and_dims():
    sh = W.LayerShape(8, 64, 32, 256)
    wl = W.custom("h8", 55, sh, [3, 64, 129], append=False)
    full_check(wl)


@pytest.mark.parametrize("H,Hkv", [(64, 0), (2, 0), (1, 0), (64, 16)])
def test_decode_head_count_extremes(H, Hkv):
    """64 query heads (two 32-column TMEM blocks per R tile in the V pass's drain), 1 and 2 heads (a partly
    used quad of columns there), and 64 query heads over 16 KV heads (grouped queries at the most heads)."""
    sh = W.LayerShape(H, 64, 16, min(256, 64 * H), num_kv_heads=Hkv)   # the joint V rank is at most H * d
    wl = W.custom(f"h{H}kv{Hkv}", 640 + H + Hkv, sh, [3, 70, 300], append=False)
    full_check(wl)


def test_decode_empty_and_zero_batch():
    sh = W.LayerShape(32, 128, 64, 2048)
    wl = W.custom("empties", 7, sh, [0, 0, 40, 0], append=False)
    Lh, Ld, got, *_ = full_check(wl)
    assert np.array_equal(got[[0, 1, 3]], np.zeros_like(got[[0, 1, 3]]))
    # batch 0 and max_seq_len 0 are accepted and launch nothing / zero the output
    z = torch.zeros(0, dtype=torch.int32, device="cuda")
    run_decode(Ld, seq_lens=z, max_seq_len=0)
    zeros4 = torch.zeros(4, dtype=torch.int32, device="cuda")
    out, *_ = run_decode(Ld, seq_lens=zeros4, max_seq_len=0)
    assert np.array_equal(out, np.zeros_like(out))
    # a prefill call with no rows also leaves a clean status word in a poisoned workspace
    desc = desc_of(Ld)
    wsb = S.starkv_prefill_workspace_bytes(desc, 0, 0, 0)
    ws = torch.full((max(wsb, 256),), POISON, dtype=torch.uint8, device="cuda")
    S.starkv_paged_prefill(desc, 0, 0, 0, None, None, None, None, None, None, None, None, 0.1, ws, wsb, None)
    assert S.starkv_decode_check(ws) == (0, 0)


def test_append_flags_skipped_targets():
    """Out-of-range positions and block ids are skipped and reported; the other rows are written."""
    sh = W.LayerShape(32, 128, 64, 2048)
    wl = W.custom("skips", 96, sh, [37, 100, 5, 64], append=True)
    Ld = D.device_layer(wl, 0)
    desc = desc_of(Ld)
    before_k, before_v = Ld["k_cache"].clone(), Ld["v_cache"].clone()
    pos = Ld["ctx_lens"].clone()
    tables = Ld["tables"].clone()
    pos[1] = Ld["tables"].shape[1] * 16          # past the block table
    tables[2, 0] = Ld["nb"] + 3                  # page outside the pool
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    S.starkv_compress_append(desc, wl.batch, Ld["k"], Ld["v"], Ld["A_K"], Ld["A_V"], tables, pos,
                             Ld["k_cache"], Ld["v_cache"], status=status)
    st, flags = S.starkv_decode_check(status)
    assert S.STATUS[st] == "STARKV_ERR_DEVICE_CHECK"
    assert flags == S.FLAG_BAD_SEQ_LEN | S.FLAG_BAD_BLOCK_ID
    tab = Ld["tables_np"]
    written = [int(tab[b][wl.ctx_lens[b] // 16]) * 16 + int(wl.ctx_lens[b] % 16) for b in (0, 3)]
    kf, vf = Ld["k_cache"].view(-1, 32 * 64), Ld["v_cache"].view(-1, 2048)
    changed_k = (kf.view(torch.int16) != before_k.view(-1, 32 * 64).view(torch.int16)).any(1)
    changed_v = (vf.view(torch.int16) != before_v.view(-1, 2048).view(torch.int16)).any(1)
    assert sorted(torch.nonzero(changed_k).flatten().tolist()) == sorted(written)
    assert sorted(torch.nonzero(changed_v).flatten().tolist()) == sorted(written)
    # compress-store: a slot outside the pool is skipped and flagged the same way
    status.zero_()
    slots = torch.tensor([written[0], Ld["nb"] * 16 + 7], dtype=torch.int32, device="cuda")
    S.starkv_compress_store(desc, 2, Ld["k"][:2], Ld["v"][:2], Ld["A_K"], Ld["A_V"], slots, Ld["k_cache"],
                            Ld["v_cache"], status=status)
    assert S.starkv_decode_check(status) == (5, S.FLAG_BAD_BLOCK_ID)


def test_decode_page_permutation_bit_identical():
    sh = W.LayerShape(32, 128, 64, 2048)
    wl = W.custom("perm", 91, sh, [77, 300, 1, 129], append=False)
    Lh = W.host_layer(wl, 0)
    Ld = D.device_layer(wl, 0, tables=Lh["tables"], nb=Lh["nb"])
    base, *_ = run_decode(Ld)
    perm = torch.from_numpy(np.random.default_rng(4).permutation(Lh["nb"])).cuda()
    kc = torch.empty_like(Ld["k_cache"]); kc[perm] = Ld["k_cache"]
    vc = torch.empty_like(Ld["v_cache"]); vc[perm] = Ld["v_cache"]
    L2 = dict(Ld, k_cache=kc, v_cache=vc, tables=perm[Ld["tables"].long()].int().contiguous())
    got, *_ = run_decode(L2)
    assert np.array_equal(got, base)


def test_decode_contiguous_equals_paged():
    sh = W.LayerShape(32, 128, 64, 2048)
    wl = W.custom("contig", 92, sh, [50, 200, 33], append=False)
    Lh = W.host_layer(wl, 0)
    Ld = D.device_layer(wl, 0, tables=Lh["tables"], nb=Lh["nb"])
    shuffled, *_ = run_decode(Ld)
    # identity layout: sequence b's pages are consecutive, in order
    need = [-(-int(t) // 16) for t in wl.seq_lens]
    ident = np.zeros_like(Lh["tables"])
    start = 0
    for b, n in enumerate(need):
        ident[b, :n] = np.arange(start, start + n)
        ident[b, n:] = Lh["nb"] - 1
        start += n
    Li = D.device_layer(wl, 0, tables=ident, nb=Lh["nb"])
    got, *_ = run_decode(Li)
    assert np.array_equal(got, shuffled)


def test_decode_softmax_stress_needle():
    """Large logits and a planted token whose K code lines up with the query."""
    sh = W.LayerShape(32, 128, 64, 2048)
    wl = W.custom("needle", 93, sh, [700, 1300], append=False)
    Lh = W.host_layer(wl, 0)
    q = (Lh["q"].astype(np.float32) * 32).astype(np.float16)
    for b, t in [(0, 5), (1, 1299)]:
        pg, sl = Lh["tables"][b][t // 16], t % 16
        qt = np.stack([Lh["B_K"][h].astype(np.float64) @ q[b, h].astype(np.float64) for h in range(32)])
        Lh["k_cache"][pg, sl] = (qt / np.abs(qt).max(axis=1, keepdims=True) * 4).astype(np.float16)
    Ld = D.device_layer(wl, 0, tables=Lh["tables"], nb=Lh["nb"])
    Ld["k_cache"].copy_(torch.from_numpy(Lh["k_cache"]))
    Ld["q"] = torch.from_numpy(q).cuda()
    got, *_ = run_decode(Ld)
    ref = O.decode_explicit(q, Lh["B_K"], Lh["B_V"], Lh["k_cache"], Lh["v_cache"], Lh["tables"],
                            Lh["seq_lens"], Lh["scale"])
    assert_close({b: got[b] for b in range(2)}, {b: ref[b] for b in range(2)})


def test_decode_bad_block_id_is_flagged():
    sh = W.LayerShape(32, 128, 64, 2048)
    wl = W.custom("bad", 94, sh, [40], append=False)
    Lh = W.host_layer(wl, 0)
    Ld = D.device_layer(wl, 0, tables=Lh["tables"], nb=Lh["nb"])
    bad = Ld["tables"].clone()
    bad[0, 1] = Lh["nb"] + 5
    desc = desc_of(Ld)
    wsb = S.starkv_decode_workspace_bytes(desc, 1, 40)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    out = torch.empty((1, 32, 128), dtype=torch.float16, device="cuda")
    S.starkv_paged_decode(desc, 1, 40, Ld["q"], Ld["B_K"], Ld["B_V"], Ld["k_cache"], Ld["v_cache"],
                          bad, Ld["seq_lens"], Ld["scale"], ws, wsb, out)
    st, flags = S.starkv_decode_check(ws)
    assert S.STATUS[st] == "STARKV_ERR_DEVICE_CHECK" and flags & S.FLAG_BAD_BLOCK_ID
    # a clean call on the same workspace clears the word
    run_decode(Ld)


def test_host_side_errors_launch_nothing():
    sh = W.LayerShape(32, 128, 64, 2048)
    wl = W.custom("err", 95, sh, [40], append=False)
    Ld = D.device_layer(wl, 0)
    desc = desc_of(Ld)
    wsb = S.starkv_decode_workspace_bytes(desc, 1, 40)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    out = torch.zeros((1, 32, 128), dtype=torch.float16, device="cuda")
    args = [desc, 1, 40, Ld["q"], Ld["B_K"], Ld["B_V"], Ld["k_cache"], Ld["v_cache"], Ld["tables"],
            Ld["seq_lens"], Ld["scale"], ws, wsb, out]
    a = list(args); a[12] = wsb - 1
    assert S.starkv_paged_decode(*a, check=False) == 3
    a = list(args); a[10] = float("nan")
    assert S.starkv_paged_decode(*a, check=False) == 1
    a = list(args); a[2] = 10 ** 6
    assert S.starkv_paged_decode(*a, check=False) == 1
    torch.cuda.synchronize()
    assert torch.count_nonzero(out).item() == 0


# ------------------------------------------------------------------ append

def test_compress_store_prefill_then_decode():
    """A 600-token prompt compressed by slot mapping (three 256-row tiles), then decoded."""
    sh = W.LayerShape(32, 128, 64, 2048)
    T = 600
    wl = W.custom("prefill", 4242, sh, [T], append=False)
    tables, nb, _ = W.block_tables(wl.seed, np.array([T]), -(-T // 16) + 2)
    A_K, A_V, B_K, B_V = W.projections(wl, 0)
    key = gen.stream_key(wl.seed, 99)
    kx = gen.codes_f16(key, T, 32 * 128, None).reshape(T, 32, 128)
    vx = gen.codes_f16(key + 1, T, 32 * 128, None).reshape(T, 32, 128)
    slots = np.array([tables[0][t // 16] * 16 + t % 16 for t in range(T)], dtype=np.int32)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    kc = torch.full((nb, 16, 32, 64), float("nan"), dtype=torch.float16, device="cuda")
    vc = torch.full((nb, 16, 2048), float("nan"), dtype=torch.float16, device="cuda")
    desc = S.layer_desc(32, 128, 64, 2048, nb, tables.shape[1])
    S.starkv_compress_store(desc, T, dev(kx), dev(vx), dev(A_K), dev(A_V), dev(slots), kc, vc)
    torch.cuda.synchronize()
    cK, cV, kc_ref, vc_ref = O.compress_store(kx, vx, A_K, A_V, slots, np.full((nb, 16, 32, 64), np.nan, np.float16),
                                              np.full((nb, 16, 2048), np.nan, np.float16))
    kg, vg = kc.cpu().numpy(), vc.cpu().numpy()
    assert np.array_equal(np.isnan(kg), np.isnan(kc_ref)) and np.array_equal(np.isnan(vg), np.isnan(vc_ref))
    kgot = kg.reshape(-1, 32 * 64)[slots].astype(np.float64)
    vgot = vg.reshape(-1, 2048)[slots].astype(np.float64)
    for got, want in ((kgot, cK.reshape(T, -1)), (vgot, cV)):
        assert np.abs(got - want).max() <= MAX_ABS and rel_l2(got, want) <= REL_L2
    q = gen.codes_f16(key + 2, 1, 32 * 128, None).reshape(1, 32, 128)
    L = dict(H=32, d=128, r=64, R=2048, nb=nb, tables=dev(tables), seq_lens=dev(np.array([T], np.int32)),
             k_cache=kc, v_cache=vc, q=dev(q), B_K=dev(B_K), B_V=dev(B_V), scale=1 / np.sqrt(128))
    got, *_ = run_decode(L)
    ref = O.decode_explicit(q, B_K, B_V, kc_ref, vc_ref, tables, [T], 1 / np.sqrt(128))
    assert_close({0: got[0]}, {0: ref[0]})


@pytest.mark.parametrize("kv_heads", [0, 8])
def test_decode_independent_of_workspace_contents(kv_heads):
    """Two runs over a workspace pre-filled with 0x00 and with 0xFF (NaN) bytes agree bit for bit."""
    sh = W.LayerShape(32, 128, 64, 512, num_kv_heads=kv_heads)
    wl = W.custom("ws", 4040 + kv_heads, sh, [1, 15, 16, 17, 300, 0, 1000, 129], append=False)
    Ld = D.device_layer(wl, 0)
    desc = desc_of(Ld)
    B, T = wl.batch, wl.max_seq_len
    wsb = S.starkv_decode_workspace_bytes(desc, B, T)
    outs = []
    for fill in (0x00, 0xFF):
        ws = torch.full((wsb,), fill, dtype=torch.uint8, device="cuda")
        out = torch.full((B, Ld["H"], Ld["d"]), float("nan"), dtype=torch.float16, device="cuda")
        S.starkv_paged_decode(desc, B, T, Ld["q"], Ld["B_K"], Ld["B_V"], Ld["k_cache"], Ld["v_cache"],
                              Ld["tables"], Ld["seq_lens"], Ld["scale"], ws, wsb, out)
        st, flags = S.starkv_decode_check(ws)
        assert st == 0, (S.STATUS[st], flags)
        outs.append(out.cpu().numpy())
    assert np.array_equal(outs[0].view(np.uint16), outs[1].view(np.uint16))


def test_append_and_decode_in_cuda_graph_match_stream_launches():
    """Three layers of append + decode captured as one CUDA graph and replayed: bit-identical outputs."""
    full = W.workload(4)
    wl = W.Workload("cb-graph", full.seed, 6, full.layers, full.ctx_lens[:6])
    layers = [D.device_layer(wl, li) for li in range(3)]
    descs = [desc_of(L) for L in layers]
    B, T = wl.batch, wl.max_seq_len
    wsb = max(S.starkv_decode_workspace_bytes(dsc, B, T) for dsc in descs)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    pools = [(L["k_cache"].clone(), L["v_cache"].clone()) for L in layers]

    def run(outs):
        st = torch.cuda.current_stream()
        for L, dsc, o, (kc, vc) in zip(layers, descs, outs, pools):
            S.starkv_compress_append(dsc, B, L["k"], L["v"], L["A_K"], L["A_V"], L["tables"], L["ctx_lens"],
                                     kc, vc, stream=st)
            S.starkv_paged_decode(dsc, B, T, L["q"], L["B_K"], L["B_V"], kc, vc, L["tables"], L["seq_lens"],
                                  L["scale"], ws, wsb, o, stream=st)

    eager = [torch.empty((B, L["H"], L["d"]), dtype=torch.float16, device="cuda") for L in layers]
    run(eager)
    torch.cuda.synchronize()
    graphed = [torch.full_like(o, float("nan")) for o in eager]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run(graphed)
    g.replay()
    torch.cuda.synchronize()
    st, flags = S.starkv_decode_check(ws)
    assert st == 0, (S.STATUS[st], flags)
    for a, b in zip(eager, graphed):
        assert np.array_equal(a.cpu().numpy().view(np.uint16), b.cpu().numpy().view(np.uint16))


# ------------------------------------------------------ chunked prefill

def _prefill_check(kv_heads, starts, chunks, seed, H=32, d=128, r=64, R=None):
    R = R or (512 if kv_heads else 2048)
    sh = W.LayerShape(H, d, r, R, num_kv_heads=kv_heads)
    starts = np.asarray(starts, np.int64)
    chunks = np.asarray(chunks, np.int64)
    # every chunk's codes are in the cache: the context is start + chunk tokens
    wl = W.custom("prefill", seed, sh, starts + chunks, append=False)
    Lh = W.host_layer(wl, 0)
    Ld = D.device_layer(wl, 0, tables=Lh["tables"], nb=Lh["nb"])
    n_rows = int(chunks.sum())
    q = gen.codes_f16(gen.stream_key(seed, 77), n_rows, H * d, None).reshape(n_rows, H, d)
    offsets = np.concatenate([[0], np.cumsum(chunks)]).astype(np.int32)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    desc = desc_of(Ld)
    max_len = int((starts + chunks).max())
    wsb = S.starkv_prefill_workspace_bytes(desc, len(chunks), n_rows, max_len)
    ws = torch.full((wsb,), 0xFF, dtype=torch.uint8, device="cuda")
    out = torch.full((n_rows, H, d), float("nan"), dtype=torch.float16, device="cuda")
    S.starkv_paged_prefill(desc, len(chunks), n_rows, max_len, dev(q), Ld["B_K"], Ld["B_V"], Ld["k_cache"],
                           Ld["v_cache"], Ld["tables"], dev(starts.astype(np.int32)), dev(offsets), Ld["scale"],
                           ws, wsb, out)
    st, flags = S.starkv_decode_check(ws)
    assert st == 0, (S.STATUS[st], flags)
    got = out.float().cpu().numpy().astype(np.float64)
    ref = O.prefill_attention(q, Lh["B_K"], Lh["B_V"], Lh["k_cache"], Lh["v_cache"], Lh["tables"], starts,
                              chunks, Lh["scale"])
    assert_close({r: got[r] for r in range(n_rows)}, {r: ref[r] for r in range(n_rows)})


@pytest.mark.parametrize("kv_heads", [0, 8])
def test_prefill_chunks_causal(kv_heads):
    """A first chunk, an empty chunk, a mid-prompt chunk, a one-token chunk and a 64-token tail chunk."""
    _prefill_check(kv_heads, starts=[0, 5, 200, 1000, 37], chunks=[37, 0, 150, 1, 64], seed=6060 + kv_heads)


def test_prefill_rows_of_one_sequence_span_tiles():
    """One sequence, a 300-token chunk after 700 cached tokens: rows span several K/V partitions."""
    _prefill_check(0, starts=[700], chunks=[300], seed=6161)


def test_prefill_read_once_shapes():
    """Read-once path for every tile geometry: 8 query heads per KV head (64 virtual heads per KV
    head, 8 rows per virtual sequence, K tiles of 4 KV heads over two pages), 2 per KV head (32
    virtual heads, N = 256 tiles of 8 KV heads), 4 per KV head with odd page counts (two-page tiles
    that end on one page), and 16-row chunks of several sequences over long contexts (the
    benchmark's chunk size)."""
    _prefill_check(8, starts=[0, 333, 1500], chunks=[5, 16, 33], seed=6262, H=64, r=64, R=512)
    _prefill_check(16, starts=[0, 333, 1500, 47], chunks=[5, 16, 33, 17], seed=6265, H=32, r=64, R=1024)
    _prefill_check(8, starts=[1, 15, 16, 300, 4000], chunks=[16, 1, 16, 20, 3], seed=6266, H=32, r=32, R=512)
    _prefill_check(0, starts=[2048, 700, 1601, 16], chunks=[16, 16, 16, 16], seed=6363)


def test_prefill_row_wise_path():
    """KV heads not in groups of 8 (8 query heads over 2 KV heads): every row runs as a decode row."""
    _prefill_check(2, starts=[0, 5, 200, 37], chunks=[37, 0, 150, 64], seed=6464, H=8, d=64, r=16, R=128)


# ------------------------------------------------ grouped-query attention

def test_decode_grouped_query_equals_repeated_kv_heads_on_gpu():
    """Hkv KV heads against the same inputs repeated to H KV heads: the MHA kernels' output."""
    H, Hkv, d, r, R = 16, 4, 64, 32, 256
    G = H // Hkv
    sh = W.LayerShape(H, d, r, R, num_kv_heads=Hkv)
    wl = W.custom("gqa-rep", 808, sh, [5, 70, 333], append=False)
    Lh = W.host_layer(wl, 0)
    Ld = D.device_layer(wl, 0, tables=Lh["tables"], nb=Lh["nb"])
    got, *_ = run_decode(Ld)
    rep = dict(Ld)
    rep["Hkv"] = H
    rep["k_cache"] = Ld["k_cache"].repeat_interleave(G, dim=2).contiguous()
    rep["B_K"] = Ld["B_K"].repeat_interleave(G, dim=0).contiguous()
    rep["B_V"] = torch.cat([Ld["B_V"][:, (h // G) * d:(h // G + 1) * d] for h in range(H)], 1).contiguous()
    want, *_ = run_decode(rep)
    ref = O.decode_explicit(Lh["q"], Lh["B_K"], Lh["B_V"], Lh["k_cache"], Lh["v_cache"],
                            Lh["tables"], Lh["seq_lens"], Lh["scale"])
    assert_close({b: got[b] for b in range(wl.batch)}, {b: ref[b] for b in range(wl.batch)})
    assert_close({b: want[b] for b in range(wl.batch)}, {b: ref[b] for b in range(wl.batch)})


def test_grouped_query_descriptor_checks():
    d = S.layer_desc(32, 128, 64, 512, 100, 8, num_kv_heads=12)        # not a power of two
    assert S.starkv_decode_workspace_bytes(d, 4, 100) == 0
    d = S.layer_desc(8, 128, 64, 512, 100, 8, num_kv_heads=16)         # more KV than query heads
    assert S.starkv_decode_workspace_bytes(d, 4, 100) == 0
    d = S.layer_desc(32, 128, 64, 512, 100, 8, num_kv_heads=8)
    assert S.starkv_decode_workspace_bytes(d, 4, 100) > 0


@pytest.mark.parametrize("kv_heads", [0, 8])
def test_decode_and_append_batch_over_256(kv_heads):
    """300 short sequences: several 256-row batch tiles in the append GEMM and the up-projection.

    With 8 KV heads, most K-pass segments are one page long, so the query tiles
    change slot at almost every tile.
    """
    sh = W.LayerShape(32, 128, 64, 2048 if not kv_heads else 512, num_kv_heads=kv_heads)
    rng = np.random.default_rng(5)
    wl = W.custom("wide", 5150, sh, rng.integers(1, 48, size=300), append=True)
    Ld, appended, _ = append_check(wl)
    got, *_ = run_decode(Ld)
    sample = [0, 1, 255, 256, 257, 299]
    ref = oracle_rows(wl, 0, W.activation(wl, 0, W.ACT_Q), Ld["A_np"], sample, wl.seq_lens, appended)
    assert_close({b: got[b] for b in sample}, ref)
