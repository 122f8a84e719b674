#!/usr/bin/env python
"""Benchmark of the STAR-KV paged low-rank decode step on B200.

One step = the whole hot path over one batch: compress-and-append of one new
token per sequence into the paged K/V code pools, then single-token paged
decode over the updated cache, for every layer of the workload.  Inputs are
seeded and synthetic with the shapes of the pages' kernel benchmark (32-head
MHA, head_size 128, rank 64, fp16, block size 16).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 3] [--impl ours|reference]

Multi-GPU runs are independent replicas (the path has no exchange step): each
rank owns its own cache and batch, timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "compressed-KV paged decode tokens/s at 1 B200; HBM GB/s as % of ~8 TB/s peak"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
FALLBACK_F16_TFLOPS = 1590.0   # dense fp16/bf16 tensor throughput (burst) of the profiling recipe
WORKLOAD_NAMES = {
    2: "single-layer decode: 32 heads, head_size 128, K rank 64/head, V joint rank 2048, fp16, "
       "block_size 16, batch 16, seq_len 2048",
    3: "single-layer decode: 32 heads, head_size 128, K rank 64/head, V joint rank 2048, fp16, "
       "block_size 16, batch 64, seq_len 8192",
    4: "continuous batching: 32 heads, head_size 128, batch 48, seq_len ~U[512,16384], 3 layers "
       "K rank {32,64,96}, V rank 32r, fp16, block_size 16",
    5: "Llama-2-7B attention path: 32 layers, 32 heads, head_size 128, batch 8, context 32768, "
       "K rank 64/head, V rank 2048, fp16, block_size 16",
    6: "grouped-query layer: 32 query heads over 8 KV heads, head_size 128, K rank 64/KV head, "
       "V joint rank 512, fp16, block_size 16, batch 64, seq_len 8192",
}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", type=int, default=3, choices=[2, 3, 4, 5, 6])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--profile-steps", type=int, default=300,
                    help="steps of the event-instrumented region giving per-kernel times")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="budget of the oracle CPU-baseline sample")
    ap.add_argument("--batch", type=int, default=0,
                    help="profiling only: override the batch with uniform lengths --seq")
    ap.add_argument("--seq", type=int, default=0)
    ap.add_argument("--graph", action="store_true",
                    help="time the step (every layer's append + decode) as one captured CUDA graph")
    ap.add_argument("--prefill-chunk", type=int, default=0,
                    help="instead of decode: a chunked-prefill step, each sequence compressing its last N "
                         "tokens into the cache and attending causally over its whole context")
    return ap.parse_args()


def max_over_ranks(x: float, device=None) -> float:
    """Max of a per-rank float across the process group (identity when not distributed)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tokens_per_s(world: int, batch_per_rank: int, ms_per_step_max: float) -> float:
    """Replicas: every rank decodes its own batch; the job's rate uses the slowest rank's time."""
    return world * batch_per_rank / (ms_per_step_max * 1e-3)


# DRAM bytes (read + write) per processed token of the two streaming kernels,
# from ncu captures (dram__bytes_read.sum + dram__bytes_write.sum of one
# launch at batch 32, context 8192, divided by its 262,144 tokens); traffic
# grows in proportion to the tokens processed.  Keyed by layer geometry
# (query heads, KV heads, K rank, V rank).  A figure is only valid for the
# kernels as they were captured: profiles/streaming_traffic_b32_t8192.md and
# profiles/gqa_streaming_b32_t8192_full.md give the commands; an entry is
# emptied when its kernel changes.
NCU_TRAFFIC_PER_TOKEN: dict = {
    (32, 32, 64, 2048): {"kpass": 4124.2, "vpass": 4252.5},
    (32, 8, 64, 512): {"kpass": 1049.3, "vpass": 1163.9},
}


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def measured_tensor_peak():
    """Dense fp16 tensor TFLOP/s: the measured bf16 burst figure (same rate for fp16), else the fallback."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_F16_TFLOPS, "fallback"


# --------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""
    FIELDS = ("index,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str | None):
        self.uuid = uuid
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-f", self.path], stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        try:
            with open(self.path) as f:
                for line in f:
                    parts = [x.strip() for x in line.split(",")]
                    if len(parts) < 10:
                        continue
                    if self.uuid and self.uuid not in parts[1]:
                        continue
                    rows.append(parts)
            os.unlink(self.path)
        except Exception:
            return None
        if not rows:
            return None
        sm = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        mx = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[6 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------ our arm

def run_ours(args):
    import torch
    import torch.distributed as dist
    import rank_compressed_kv_star_b200 as S
    from rank_compressed_kv_star_b200 import build
    from starkv_inputs import device as D, workloads as W

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=torch.device("cuda", local))
    if rank == 0:
        build.build()
        build.build_inputs()
    if world > 1:
        dist.barrier()
    S.load_library()

    wl = W.workload(args.workload)
    if args.batch:
        seq = args.seq or wl.max_seq_len      # length defaults to the workload's own
        wl = W.Workload(f"{wl.name} (override: batch {args.batch}, length {seq})", wl.seed,
                        args.batch, wl.layers[:1], np.full(args.batch, seq - 1, dtype=np.int64))
    layers = []
    for li in range(len(wl.layers)):
        Ld = D.device_layer(wl, li)
        Ld["desc"] = S.layer_desc(Ld["H"], Ld["d"], Ld["r"], Ld["R"], Ld["nb"], Ld["tables"].shape[1],
                                  num_kv_heads=Ld["Hkv"])
        layers.append(Ld)
    B = wl.batch
    max_len = wl.max_seq_len
    wsb = max(S.starkv_decode_workspace_bytes(L["desc"], B, max_len) for L in layers)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    outs = [torch.empty((B, L["H"], L["d"]), dtype=torch.float16, device="cuda") for L in layers]
    stream = torch.cuda.current_stream()
    n_ev = 5

    def step(evs=None, app_evs=None):
        """One step: every layer's append + decode as one starkv_append_decode call, or, when timing
        the kernels one by one, starkv_compress_append then starkv_paged_decode_profiled."""
        stream = torch.cuda.current_stream()       # the capture stream while a graph is recorded
        for li, L in enumerate(layers):
            if evs is None:
                S.starkv_append_decode(L["desc"], B, max_len, L["k"], L["v"], L["A_K"], L["A_V"], L["ctx_lens"],
                                       L["q"], L["B_K"], L["B_V"], L["k_cache"], L["v_cache"], L["tables"],
                                       L["seq_lens"], L["scale"], ws, wsb, outs[li], stream=stream)
                continue
            app_evs[li][0].record(stream)
            S.starkv_compress_append(L["desc"], B, L["k"], L["v"], L["A_K"], L["A_V"], L["tables"],
                                     L["ctx_lens"], L["k_cache"], L["v_cache"], stream=stream)
            app_evs[li][1].record(stream)
            S.starkv_paged_decode_profiled(L["desc"], B, max_len, L["q"], L["B_K"], L["B_V"],
                                           L["k_cache"], L["v_cache"], L["tables"], L["seq_lens"],
                                           L["scale"], ws, wsb, outs[li], evs[li], stream=stream)

    for _ in range(args.warmup):
        step()
    st, flags = S.starkv_decode_check(ws, stream)
    if st != 0:
        raise RuntimeError(f"device status {S.STATUS[st]} flags {flags}")
    graph = None
    if args.graph:
        # the whole step (every layer) as one graph; the library makes no host
        # round trips, allocations or synchronisations inside a call
        graph = torch.cuda.CUDAGraph()
        torch.cuda.synchronize()
        with torch.cuda.graph(graph):
            step()
        for _ in range(3):
            graph.replay()
        torch.cuda.synchronize()
    run_step = graph.replay if graph is not None else step

    # ---------------- device-timed region: inputs resident, codes >> L2 per step
    K = args.steps
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    uuid = None
    try:
        uuid = str(torch.cuda.get_device_properties(local).uuid)
    except Exception:
        pass
    clocks = ClockSampler(uuid)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    t0.record(stream)
    for i in range(K):
        run_step()
    t1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if world > 1:
        dist.barrier()
    ms = t0.elapsed_time(t1) / K
    st, flags = S.starkv_decode_check(ws, stream)
    if st != 0:
        raise RuntimeError(f"device status {S.STATUS[st]} flags {flags}")

    # ---------------- per-kernel durations: a second timed region of the same
    # steps with CUDA events recorded between the kernels on the launching stream
    Kp = max(1, min(K, args.profile_steps))
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in layers] for _ in range(Kp)]
    app_evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in layers] for _ in range(Kp)]
    # torch creates the underlying cudaEvent at the first record: do that now so
    # the raw handles handed to the library are valid
    for step_evs in (evs, app_evs):
        for per_step in step_evs:
            for per_layer in per_step:
                for e in per_layer:
                    e.record(stream)
    torch.cuda.synchronize()
    for i in range(Kp):
        step(evs[i], app_evs[i])
    torch.cuda.synchronize()
    names = ["absorb", "kpass", "vpass", "finish"]
    per = {n: 0.0 for n in names}
    per["append"] = 0.0
    for i in range(Kp):
        for li in range(len(layers)):
            e = evs[i][li]
            for j, n in enumerate(names):
                per[n] += e[j].elapsed_time(e[j + 1])
            per["append"] += app_evs[i][li][0].elapsed_time(app_evs[i][li][1])
    per = {n: v / Kp for n, v in per.items()}             # ms per step (all layers)

    ms = max_over_ranks(ms, device="cuda")

    # ---------------- algorithmic bytes
    T_sum = int(wl.seq_lens.sum())
    k_bytes = sum(T_sum * L["Hkv"] * L["r"] * 2 for L in layers)
    v_bytes = sum(T_sum * L["R"] * 2 for L in layers)
    proj_bytes = sum(L["B_K"].numel() * 2 + L["B_V"].numel() * 2 + L["A_K"].numel() * 2 + L["A_V"].numel() * 2
                     for L in layers)
    act_bytes = sum(B * (L["H"] + L["Hkv"]) * L["d"] * 2 * 2 for L in layers)   # q, out; k, v
    step_bytes = k_bytes + v_bytes + proj_bytes + act_bytes
    peak, peak_kind = measured_peaks()
    kp_gbs = k_bytes / (per["kpass"] * 1e-3) / 1e9
    vp_gbs = v_bytes / (per["vpass"] * 1e-3) / 1e9
    dom = "kpass" if per["kpass"] >= per["vpass"] else "vpass"
    dom_bytes, dom_gbs = (k_bytes, kp_gbs) if dom == "kpass" else (v_bytes, vp_gbs)
    traffic = None
    geom = (layers[0]["H"], layers[0]["Hkv"], layers[0]["r"], layers[0]["R"])
    if len(layers) == 1 and dom in NCU_TRAFFIC_PER_TOKEN.get(geom, {}):
        traffic = round(NCU_TRAFFIC_PER_TOKEN[geom][dom] * T_sum)

    # ---------------- end to end: every step copies its inputs (new k, v,
    # positions, queries, block tables, lengths) from pinned host memory to the
    # device, runs starkv_append_decode on them and copies the output back to
    # pinned host memory.  Two sets of device buffers let step i+1's input copies
    # (copy stream) and step i's output copy (readback stream) overlap step i's
    # kernels; every step's copies are inside the timed region, which runs from
    # the first input copy to the last output copy.
    Ke = max(1, min(args.e2e_steps, K))
    names = ("q", "k", "v", "tables", "seq_lens", "ctx_lens")
    host_in = [{n: L[n].cpu().pin_memory() for n in names} for L in layers]
    host_out = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outs]
    dev_in = [[{n: torch.empty_like(L[n]) for n in names} for L in layers] for _ in range(2)]
    dev_out = [[torch.empty_like(o) for o in outs] for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for h in host_in for t in h.values())
    d2h = sum(o.numel() * o.element_size() for o in outs)
    copy_s, back_s = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]     # inputs of the buffer set landed
    ev_run = [torch.cuda.Event() for _ in range(2)]    # the step on that set finished
    ev_out = [torch.cuda.Event() for _ in range(2)]    # its output copied back
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    e0.record(copy_s)
    for i in range(Ke):
        j = i % 2
        with torch.cuda.stream(copy_s):
            if i >= 2:
                copy_s.wait_event(ev_run[j])           # step i-2 no longer reads these inputs
            for li in range(len(layers)):
                for n in names:
                    dev_in[j][li][n].copy_(host_in[li][n], non_blocking=True)
            ev_in[j].record(copy_s)
        stream.wait_event(ev_in[j])
        if i >= 2:
            stream.wait_event(ev_out[j])               # step i-2's output has been read back
        for li, L in enumerate(layers):
            d = dev_in[j][li]
            S.starkv_append_decode(L["desc"], B, max_len, d["k"], d["v"], L["A_K"], L["A_V"], d["ctx_lens"],
                                   d["q"], L["B_K"], L["B_V"], L["k_cache"], L["v_cache"], d["tables"],
                                   d["seq_lens"], L["scale"], ws, wsb, dev_out[j][li], stream=stream)
        ev_run[j].record(stream)
        with torch.cuda.stream(back_s):
            back_s.wait_event(ev_run[j])
            for li in range(len(layers)):
                host_out[li].copy_(dev_out[j][li], non_blocking=True)
            ev_out[j].record(back_s)
    e1.record(back_s)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / Ke, device="cuda")
    assert np.isfinite(host_out[0].float().numpy()).all()
    # the host-buffer entry point (one call per layer: its own copies, then the
    # step, then the output copy, all on one stream) for comparison
    stg_bytes = max(S.starkv_host_staging_bytes(L["desc"], B) for L in layers)
    staging = torch.empty(stg_bytes, dtype=torch.uint8, device="cuda")
    torch.cuda.synchronize()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for _ in range(Ke):
        for li, L in enumerate(layers):
            h = host_in[li]
            S.starkv_append_decode_host(L["desc"], B, max_len, h["k"], h["v"], h["ctx_lens"], h["q"], h["tables"],
                                        h["seq_lens"], L["A_K"], L["A_V"], L["B_K"], L["B_V"], L["k_cache"],
                                        L["v_cache"], L["scale"], staging, stg_bytes, ws, wsb, host_out[li],
                                        stream=stream)
    f1.record(stream)
    torch.cuda.synchronize()
    host_call_ms = max_over_ranks(f0.elapsed_time(f1) / Ke, device="cuda")

    cpu = None
    if rank == 0 and world == 1 and args.cpu_seconds > 0:
        cpu = cpu_baseline(wl, args.cpu_seconds)

    value = whole_job_tokens_per_s(world, B, ms)
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(ms, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f16", "accum": "f32", "data": "synthetic",
        "config": {"workload": (f"cfg{args.workload}: {WORKLOAD_NAMES[args.workload]}" if not args.batch
                                else wl.name), "batch": B,
                   "max_seq_len": max_len, "layers": len(layers),
                   "step": "compress-append of one token per sequence + paged decode, every layer "
                           "(one starkv_append_decode call per layer)",
                   "l2": "inputs larger than L2 (code pools of %.2f GiB read per step)" % ((k_bytes + v_bytes) / 2**30),
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "launch": "one CUDA graph per step" if graph is not None else "stream launches (PDL)"},
        "hbm": {"step_algorithmic_bytes": step_bytes,
                "step_GBps": round(step_bytes / (ms * 1e-3) / 1e9, 1),
                "frac_of_8TBps": round(step_bytes / (ms * 1e-3) / 1e9 / NOMINAL_HBM_GBS, 4),
                "frac_of_peak": round(step_bytes / (ms * 1e-3) / 1e9 / peak, 4), "peak_kind": peak_kind},
        "roofline": {"kernel": dom, "bound": "hbm", "achieved": round(dom_gbs, 1), "peak": peak,
                     "unit": "GB/s", "frac": round(dom_gbs / peak, 4), "traffic": traffic,
                     "algorithmic_bytes_per_launch": dom_bytes // len(layers), "peak_kind": peak_kind},
        "kernels_ms_per_step": {n: round(v, 5) for n, v in per.items()},
        "kernels_timing": f"CUDA events between kernels over {Kp} further steps of separate append and decode "
                          f"calls (append = the prep kernel with the V and K codes; absorb = the prep kernel "
                          f"with the query absorption; vpass includes the split reduction of the maxima; "
                          f"finish = split reduction of Z / L + up-projection)",
        "kernels_GBps": {"kpass": round(kp_gbs, 1), "vpass": round(vp_gbs, 1)},
        "e2e": {"value": round(whole_job_tokens_per_s(world, B, e2e_ms), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 5),
                "call": "per step: pinned-host input copies, starkv_append_decode per layer, output copy to "
                        "pinned host memory; two buffer sets overlap a step's copies with the previous "
                        "step's kernels",
                "host_entry_point": {"call": "starkv_append_decode_host per layer (copies and step in order on "
                                             "one stream)",
                                     "value": round(whole_job_tokens_per_s(world, B, host_call_ms), 1),
                                     "ms_per_step": round(host_call_ms, 5)}},
        "gpu_launches": K * len(layers) * 4,   # per layer: prep (append + absorb), K pass, V pass, finish
        "clocks": clk,
    }
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


# -------------------------------------------------------- CPU baseline

def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def prepare_seq(wl, b, layer, proj_cache):
    """Host inputs of one sequence of one layer: a private paged pool holding its pages
    under a shuffled block-table row (generation is not part of any timing)."""
    from starkv_inputs import workloads as W
    sh = wl.layers[layer]
    ctx = int(wl.ctx_lens[b])
    T = ctx + (1 if wl.append else 0)
    cK, cV = W.seq_codes(wl, layer, b, ctx)
    n_pages = -(-T // 16)
    row = np.random.default_rng(b).permutation(n_pages).astype(np.int32)
    kc = np.full((n_pages, 16, sh.kv_heads, sh.k_rank), np.nan, np.float16)
    vc = np.full((n_pages, 16, sh.v_rank), np.nan, np.float16)
    W.place_host(kc, row, cK)
    W.place_host(vc, row, cV)
    if layer not in proj_cache:
        proj_cache[layer] = W.projections(wl, layer)
    q, k, v = (W.activation(wl, layer, a)[b:b + 1] for a in (W.ACT_Q, W.ACT_K, W.ACT_V))
    return dict(kc=kc, vc=vc, row=row, q=q, k=k, v=v, ctx=ctx, T=T, proj=proj_cache[layer],
                append=wl.append, H=sh.num_heads)


def oracle_eval(st, heads=None):
    """Timed oracle work for one prepared sequence: append, block-table walk, decode of `heads`."""
    from oracle import starkv_oracle as O
    A_K, A_V, B_K, B_V = st["proj"]
    t0 = time.perf_counter()
    kc, vc = st["kc"], st["vc"]
    if st["append"]:
        _, _, kc, vc = O.compress_append(st["k"], st["v"], A_K, A_V, st["row"][None],
                                         np.array([st["ctx"]]), kc, vc)
    cK = O.gather(kc, st["row"], st["T"])
    cV = O.gather(vc, st["row"], st["T"])
    O.attend_codes_reordered(st["q"][0], B_K, B_V, cK, cV, 1.0 / np.sqrt(st["q"].shape[2]), heads=heads)
    return time.perf_counter() - t0


def _prepared(wl, n_seq=4):
    proj = {}
    n_layers = len(wl.layers)
    out = []
    for i in range(n_seq):
        layer = i % n_layers
        b = (i * 7919) % wl.batch
        out.append(prepare_seq(wl, b, layer, proj))
    return out


def cpu_baseline(wl, budget_s):
    seqs = _prepared(wl)
    done, spent = 0, 0.0
    while spent < budget_s:
        spent += oracle_eval(seqs[done % len(seqs)])
        done += 1
    n_layers = len(wl.layers)
    tok_per_s = done / spent / n_layers          # one decode token = one sequence through every layer
    return {"value": round(tok_per_s, 4), "unit": "tokens/s", "cores": _blas_threads(), "kind": "oracle",
            "sample": f"{done} (sequence, layer) append+decode evaluations of this workload in fp64 "
                      f"(explicit K, reordered V), cycling over {len(seqs)} prepared sequences; "
                      f"{spent:.1f} s of oracle time, code generation excluded"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    from starkv_inputs import workloads as W
    wl = W.workload(args.workload)
    seqs = _prepared(wl)
    n_layers = len(wl.layers)
    H = seqs[0]["H"]
    per_step_budget = min(2.0, 120.0 / (args.steps + args.warmup))
    # heads per step sized from one calibration evaluation
    t_full = oracle_eval(seqs[0])
    n_heads = int(max(1, min(H, round(H * per_step_budget / max(t_full, 1e-6)))))
    times, frac = [], []
    for i in range(args.warmup + args.steps):
        h0 = (i * n_heads) % H
        heads = [(h0 + j) % H for j in range(n_heads)]
        sec = oracle_eval(seqs[i % len(seqs)], heads=heads)
        if i >= args.warmup:
            times.append(sec)
            frac.append(n_heads / H)
    tokens = sum(frac) / n_layers
    value = tokens / sum(times)
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * sum(times) / len(times), 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"cfg{args.workload}: {WORKLOAD_NAMES[args.workload]}", "batch": wl.batch,
                   "max_seq_len": wl.max_seq_len, "layers": n_layers},
        "cpu_baseline": {"value": round(value, 4), "unit": "tokens/s", "cores": _blas_threads(),
                         "kind": "oracle",
                         "sample": f"each step: one sequence's append, block-table walk and decode of "
                                   f"{n_heads}/{H} heads for one layer, fp64 oracle"},
        "e2e": {"value": round(value, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


PREFILL_METRIC = "compressed-KV chunked-prefill tokens/s at 1 B200 (compress + causal attention over the codes)"


def run_prefill(args):
    """One step = compress-store of the last N tokens of every sequence + causal attention of those
    N queries over the sequence's whole context (the cache holds every token)."""
    import torch
    import rank_compressed_kv_star_b200 as S
    from rank_compressed_kv_star_b200 import build
    from starkv_inputs import device as D, gen, workloads as W
    from oracle import starkv_oracle as O

    build.build()
    build.build_inputs()
    S.load_library()
    N = args.prefill_chunk
    wl = W.workload(args.workload)
    if args.batch:   # profiling only: fewer sequences of a uniform length
        seq = args.seq or wl.max_seq_len
        wl = W.Workload(f"{wl.name} (override: batch {args.batch}, length {seq})", wl.seed, args.batch, wl.layers[:1],
                        np.full(args.batch, seq, dtype=np.int64), append=False)
    wl = W.Workload(wl.name + f" (chunked prefill: last {N} tokens)", wl.seed, wl.batch, wl.layers[:1],
                    wl.seq_lens.copy(), append=False)
    L = D.device_layer(wl, 0)
    H, Hkv, d, r, R = L["H"], L["Hkv"], L["d"], L["r"], L["R"]
    desc = S.layer_desc(H, d, r, R, L["nb"], L["tables"].shape[1], num_kv_heads=Hkv)
    B = wl.batch
    T = wl.seq_lens.astype(np.int64)
    starts = T - N
    n_rows = B * N
    rows_b = np.repeat(np.arange(B), N)
    rows_t = (starts[:, None] + np.arange(N)[None, :]).reshape(-1)
    slots = (L["tables_np"][rows_b, rows_t // 16].astype(np.int64) * 16 + rows_t % 16).astype(np.int32)
    key = gen.stream_key(wl.seed, 991)
    q = gen.codes_f16(key, n_rows, H * d, None).reshape(n_rows, H, d)
    kx = gen.codes_f16(key + 1, n_rows, Hkv * d, None).reshape(n_rows, Hkv, d)
    vx = gen.codes_f16(key + 2, n_rows, Hkv * d, None).reshape(n_rows, Hkv, d)
    offs = (np.arange(B + 1) * N).astype(np.int32)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    qd, kd, vd, sd = dev(q), dev(kx), dev(vx), dev(slots)
    st_d, of_d = dev(starts.astype(np.int32)), dev(offs)
    max_len = int(T.max())
    wsb = S.starkv_prefill_workspace_bytes(desc, B, n_rows, max_len)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    out = torch.empty((n_rows, H, d), dtype=torch.float16, device="cuda")
    stream = torch.cuda.current_stream()

    def step(qq=qd, kk=kd, vv=vd, ss=sd, sts=st_d, ofs=of_d, o=out):
        S.starkv_compress_store(desc, n_rows, kk, vv, L["A_K"], L["A_V"], ss, L["k_cache"], L["v_cache"],
                                stream=stream)
        S.starkv_paged_prefill(desc, B, n_rows, max_len, qq, L["B_K"], L["B_V"], L["k_cache"], L["v_cache"],
                               L["tables"], sts, ofs, L["scale"], ws, wsb, o, stream=stream)

    for _ in range(max(3, args.warmup)):
        step()
    stt, flags = S.starkv_decode_check(ws, stream)
    if stt != 0:
        raise RuntimeError(f"device status {S.STATUS[stt]} flags {flags}")
    K = args.steps
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    uuid = None
    try:
        uuid = str(torch.cuda.get_device_properties(0).uuid)
    except Exception:
        pass
    clocks = ClockSampler(uuid)
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    t0.record(stream)
    for _ in range(K):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = t0.elapsed_time(t1) / K

    # end to end: every step copies the chunk's inputs from pinned host memory,
    # runs the step and copies its output back to pinned host memory; two sets
    # of device buffers let a step's copies overlap the previous step's kernels
    hin = [x.cpu().pin_memory() for x in (qd, kd, vd, sd, st_d, of_d)]
    hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    dbuf = [[torch.empty_like(x) for x in (qd, kd, vd, sd, st_d, of_d)] for _ in range(2)]
    dout = [torch.empty_like(out) for _ in range(2)]
    copy_s, back_s = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in, ev_run, ev_out = ([torch.cuda.Event() for _ in range(2)] for _ in range(3))
    Ke = max(1, min(args.e2e_steps, K))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(copy_s)
    for i in range(Ke):
        j = i % 2
        with torch.cuda.stream(copy_s):
            if i >= 2:
                copy_s.wait_event(ev_run[j])
            for h, dd in zip(hin, dbuf[j]):
                dd.copy_(h, non_blocking=True)
            ev_in[j].record(copy_s)
        stream.wait_event(ev_in[j])
        if i >= 2:
            stream.wait_event(ev_out[j])
        step(*dbuf[j], o=dout[j])
        ev_run[j].record(stream)
        with torch.cuda.stream(back_s):
            back_s.wait_event(ev_run[j])
            hout.copy_(dout[j], non_blocking=True)
            ev_out[j].record(back_s)
    e1.record(back_s)
    torch.cuda.synchronize()
    ms_e2e = e0.elapsed_time(e1) / Ke
    h2d = sum(x.numel() * x.element_size() for x in hin)
    d2h = hout.numel() * hout.element_size()

    # algorithmic bytes: every sequence's codes read once, the chunk's codes written, q/k/v in, out
    code_bytes = int(T.sum()) * (Hkv * r + R) * 2
    step_bytes = (code_bytes + n_rows * (Hkv * r + R) * 2 + n_rows * (H + 2 * Hkv) * d * 2 + n_rows * H * d * 2
                  + (L["A_K"].numel() + L["A_V"].numel() + L["B_K"].numel() + L["B_V"].numel()) * 2)
    peak, peak_kind = measured_peaks()
    achieved = step_bytes / (ms * 1e-3) / 1e9
    # useful tensor work of the read-once path per context token: the K logits of
    # the chunk's rows (2 * N * H * r) and the weighted sum of the V codes
    # (2 * N * H * R); the larger of the two roof times sets the bound
    step_flops = int(T.sum()) * 2 * N * H * (r + R)
    tpeak, tpeak_kind = measured_tensor_peak()
    t_flops = step_flops / (tpeak * 1e12)
    t_bytes = step_bytes / (peak * 1e9)
    tensor_bound = t_flops > t_bytes
    achieved_tf = step_flops / (ms * 1e-3) / 1e12
    G = H // Hkv
    read_note = ("every page of a sequence is read once per step: a chunk's 16 rows are one virtual sequence "
                 "whose rows x heads are the extra N columns of the tensor-core K and V passes" if G <= 4 else
                 f"{G} query heads per KV head: a chunk's 16 rows form {G // 4} virtual sequences of {64 // G} rows "
                 f"(64 virtual heads per KV head), each reading the sequence's pages")

    # the oracle on one sequence's chunk
    b0 = 0
    Lh_tab = L["tables_np"][b0:b0 + 1]
    kc_h = L["k_cache"].cpu().numpy()
    vc_h = L["v_cache"].cpu().numpy()
    Ah = [x.cpu().numpy() for x in (L["B_K"], L["B_V"])]
    t_c = time.perf_counter()
    O.prefill_attention(q[:N], Ah[0], Ah[1], kc_h, vc_h, Lh_tab, starts[:1], [N], L["scale"])
    cpu_s = time.perf_counter() - t_c
    line = {
        "metric": PREFILL_METRIC, "value": round(n_rows / (ms * 1e-3), 1), "unit": "tokens/s", "n_gpus": 1,
        "steps": K, "warmup": max(3, args.warmup), "ms_per_step": round(ms, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f16", "accum": "f32", "data": "synthetic",
        "config": {"workload": wl.name, "batch": B, "chunk": N, "context": max_len, "layers": 1,
                   "step": "compress-store of the chunk + causal attention of its queries over the context",
                   "l2": f"code pools of {code_bytes / 2**30:.2f} GiB read per step"},
        "roofline": ({"kernel": "prefill step", "bound": "tensor", "achieved": round(achieved_tf, 1),
                      "peak": tpeak, "unit": "TFLOP/s", "frac": round(achieved_tf / tpeak, 4), "traffic": None,
                      "algorithmic_flops_per_step": step_flops, "peak_kind": tpeak_kind,
                      "hbm": {"achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                              "frac": round(achieved / peak, 4), "algorithmic_bytes_per_step": step_bytes,
                              "peak_kind": peak_kind},
                      "note": read_note}
                     if tensor_bound else
                     {"kernel": "prefill step", "bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                      "unit": "GB/s", "frac": round(achieved / peak, 4), "traffic": None,
                      "algorithmic_bytes_per_launch": step_bytes, "peak_kind": peak_kind,
                      "tensor": {"achieved": round(achieved_tf, 1), "peak": tpeak, "unit": "TFLOP/s",
                                 "frac": round(achieved_tf / tpeak, 4), "algorithmic_flops_per_step": step_flops,
                                 "peak_kind": tpeak_kind},
                      "note": read_note}),
        "e2e": {"value": round(n_rows / (ms_e2e * 1e-3), 1), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": round(ms_e2e, 5)},
        "gpu_launches": K * 7,   # compress-store + chunk table, absorb, K pass, weights, V pass, finish
        "clocks": clk,
        "cpu_baseline": {"value": round(N / cpu_s, 4), "unit": "tokens/s", "cores": _blas_threads(),
                         "kind": "oracle",
                         "sample": f"one sequence's {N}-token chunk over its {int(T[b0])}-token context, "
                                   f"fp64 oracle (explicit decompression), {cpu_s:.1f} s"},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    if args.impl == "reference" and args.prefill_chunk:
        raise SystemExit("the reference arm times the decode step; run --prefill-chunk with --impl ours")
    if args.impl == "reference":
        run_reference(args)
    elif args.prefill_chunk:
        run_prefill(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
