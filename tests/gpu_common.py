"""Helpers shared by the GPU parity tests (the test_gpu_* files).

Tolerances (stated for the fp16-output path with fp32 accumulation): for
decode outputs, max |gpu - oracle| <= 2e-3 and relative L2 error <= 1e-3 over
the compared rows.  Appended codes: placement and every untouched byte
bit-exact; code values within one fp16 ulp of the fp64 code plus the fp32
dot-product rounding bound (which only matters for codes near zero), and
within the same max-abs / rel-L2 bounds.
"""
import numpy as np
import torch

import rank_compressed_kv_star_b200 as S
from oracle import starkv_oracle as O
from starkv_inputs import device as D, workloads as W

MAX_ABS, REL_L2 = 2e-3, 1e-3
POISON = 0xFF   # workspaces start filled with NaN bytes: no result may depend on them


def rel_l2(got, ref):
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))


def desc_of(L):
    return S.layer_desc(L["H"], L["d"], L["r"], L["R"], L["nb"], L["tables"].shape[1],
                        num_kv_heads=L.get("Hkv", 0))


def run_decode(L, seq_lens=None, max_seq_len=None, q=None):
    """Decode through the C ABI over a poisoned workspace; the status word must come back clean."""
    seq_lens = L["seq_lens"] if seq_lens is None else seq_lens
    B = seq_lens.shape[0]
    if max_seq_len is None:
        max_seq_len = int(seq_lens.max().item()) if B else 0
    desc = desc_of(L)
    wsb = S.starkv_decode_workspace_bytes(desc, B, max_seq_len)
    ws = torch.full((max(wsb, 256),), POISON, dtype=torch.uint8, device="cuda")
    out = torch.full((B, L["H"], L["d"]), float("nan"), dtype=torch.float16, device="cuda")
    S.starkv_paged_decode(desc, B, max_seq_len, L["q"] if q is None else q, L["B_K"], L["B_V"],
                          L["k_cache"], L["v_cache"], L["tables"], seq_lens, L["scale"], ws, wsb, out)
    st, flags = S.starkv_decode_check(ws)
    assert st == 0, (S.STATUS[st], flags)
    return out.float().cpu().numpy().astype(np.float64), ws, desc


def oracle_rows(wl, layer, L_host_q, A_np, bs, seq_lens, appended=None, q=None):
    """fp64 oracle for sequences `bs` (codes regenerated on the host)."""
    A_K, A_V, B_K, B_V = A_np
    qn = L_host_q if q is None else q
    out = {}
    for b in bs:
        T = int(seq_lens[b])
        if T == 0:
            out[b] = np.zeros(qn.shape[1:])
            continue
        ctx = int(wl.ctx_lens[b])
        cK, cV = W.seq_codes(wl, layer, b, min(ctx, T))
        cK, cV = cK.astype(np.float64), cV.astype(np.float64)
        if T > ctx:  # the step's appended token (oracle's own fp16 codes)
            aK, aV = appended
            cK = np.concatenate([cK, aK[b][None].astype(np.float64)])
            cV = np.concatenate([cV, aV[b][None].astype(np.float64)])
        out[b] = O.attend_codes_reordered(qn[b], B_K, B_V, cK, cV, 1.0 / np.sqrt(qn.shape[2]))
    return out


def assert_close(got_rows, ref_rows):
    g = np.stack([got_rows[b] for b in sorted(ref_rows)])
    r = np.stack([ref_rows[b] for b in sorted(ref_rows)])
    err = np.abs(g - r).max()
    rl = rel_l2(g, r)
    assert np.isfinite(g).all()
    assert err <= MAX_ABS, err
    assert rl <= REL_L2, rl
    return err, rl


def full_check(wl, layer=0):
    """Whole-output decode parity against the explicit-decompression oracle (host pools)."""
    Lh = W.host_layer(wl, layer)
    Ld = D.device_layer(wl, layer, tables=Lh["tables"], nb=Lh["nb"])
    got, ws, desc = run_decode(Ld)
    ref = O.decode_explicit(Lh["q"], Lh["B_K"], Lh["B_V"], Lh["k_cache"], Lh["v_cache"],
                            Lh["tables"], Lh["seq_lens"], Lh["scale"])
    err, rl = assert_close({b: got[b] for b in range(wl.batch)}, {b: ref[b] for b in range(wl.batch)})
    return Lh, Ld, got, ws, desc, err, rl


def append_only(Ld, desc, status, B):
    S.starkv_compress_append(desc, B, Ld["k"], Ld["v"], Ld["A_K"], Ld["A_V"], Ld["tables"], Ld["ctx_lens"],
                             Ld["k_cache"], Ld["v_cache"], status=status)


def append_then_decode(Ld, desc, status, B):
    """The step as one call (starkv_append_decode): returns the decode output and its workspace."""
    T = int(Ld["seq_lens"].max().item())
    wsb = S.starkv_decode_workspace_bytes(desc, B, T)
    ws = torch.full((max(wsb, 256),), POISON, dtype=torch.uint8, device="cuda")
    out = torch.full((B, Ld["H"], Ld["d"]), float("nan"), dtype=torch.float16, device="cuda")
    S.starkv_append_decode(desc, B, T, Ld["k"], Ld["v"], Ld["A_K"], Ld["A_V"], Ld["ctx_lens"], Ld["q"], Ld["B_K"],
                           Ld["B_V"], Ld["k_cache"], Ld["v_cache"], Ld["tables"], Ld["seq_lens"], Ld["scale"],
                           ws, wsb, out, append_status=status)
    st, flags = S.starkv_decode_check(ws)
    assert st == 0, (S.STATUS[st], flags)
    return out.float().cpu().numpy().astype(np.float64), ws


def append_check(wl, layer=0, Ld=None, run=append_only):
    """Compress-and-append of one token per sequence through the C ABI, whole batch.

    ``run(Ld, desc, status, batch)`` makes the call that appends (by default
    starkv_compress_append alone).  Bit-exact: every byte of both pools
    outside the batch's target slots is unchanged (compared on the device),
    and the status word reports no skipped target.  Values: each target
    slot's codes against the oracle's fp64 codes of the same fp16 inputs,
    within one fp16 ulp plus the fp32 dot-product bound.  Returns the device
    layer, the oracle's fp16 codes and what ``run`` returned.
    """
    if Ld is None:
        Ld = D.device_layer(wl, layer)
    desc = desc_of(Ld)
    Hkv, r, R, d = Ld["Hkv"], Ld["r"], Ld["R"], Ld["d"]
    kf = Ld["k_cache"].view(-1, Hkv * r)
    vf = Ld["v_cache"].view(-1, R)
    before_k, before_v = kf.clone(), vf.clone()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ran = run(Ld, desc, status, wl.batch)
    st, flags = S.starkv_decode_check(status)
    assert st == 0 and flags == 0, (S.STATUS[st], flags)
    pos = wl.ctx_lens
    tab = Ld["tables_np"]
    rows = np.array([int(tab[b][pos[b] // 16]) * 16 + int(pos[b] % 16) for b in range(wl.batch)])
    assert len(set(rows.tolist())) == wl.batch
    keep = torch.ones(kf.shape[0], dtype=torch.bool, device="cuda")
    keep[torch.from_numpy(rows).cuda()] = False
    assert torch.equal(kf.view(torch.int16)[keep], before_k.view(torch.int16)[keep])
    assert torch.equal(vf.view(torch.int16)[keep], before_v.view(torch.int16)[keep])
    del before_k, before_v, keep
    rows_t = torch.from_numpy(rows).cuda()
    k_got = kf[rows_t].cpu().numpy().astype(np.float64)
    v_got = vf[rows_t].cpu().numpy().astype(np.float64)
    # the oracle's inputs come from the host generator, not from device tensors
    k_in = W.activation(wl, layer, W.ACT_K)
    v_in = W.activation(wl, layer, W.ACT_V)
    A_K, A_V, _, _ = Ld["A_np"]
    cK, cV = O.compress(k_in, v_in, A_K, A_V)
    # bound: one fp16 ulp of the exact code plus the fp32 dot-product error bound
    # gamma(K) * sum|terms| (K = length of the contraction), doubled for the
    # order-free accumulation
    kk, vv = k_in.astype(np.float64), v_in.astype(np.float64)
    absK = np.stack([np.abs(kk[:, h, :]) @ np.abs(A_K[h].astype(np.float64))
                     for h in range(Hkv)], axis=1).reshape(wl.batch, -1)
    absV = np.abs(vv.reshape(wl.batch, -1)) @ np.abs(A_V.astype(np.float64))
    for want, got, absum, K in ((cK.reshape(wl.batch, -1), k_got, absK, d),
                                (cV, v_got, absV, Hkv * d)):
        ulp = np.spacing(np.abs(want).astype(np.float16)).astype(np.float64)
        gamma = K * 2.0 ** -24 / (1 - K * 2.0 ** -24)
        bound = ulp + 2 * gamma * absum
        assert np.all(np.abs(got - want) <= bound), np.max(np.abs(got - want) / bound)
        assert np.abs(got - want).max() <= MAX_ABS
        assert rel_l2(got, want) <= REL_L2
    return Ld, (cK.astype(np.float16), cV.astype(np.float16)), ran


def load():
    from rank_compressed_kv_star_b200 import build
    build.build()
    build.build_inputs()
    S.load_library()
