#!/usr/bin/env python
"""Benchmark of the SAS gated block-sparse attention hot path on B200.

One step = one pass of the whole path over one batch of synthetic input:
  training layer (Qwen3-4B-like: B1 T8192 Hq32/Hkv8 d128 block 64, K=15):
      sas_block_topk -> sas_gated_attn_fwd -> sas_gated_attn_bwd
  decode (131072-token cache, Hq32/Hkv8 d128 block 64, budget 2048 = K31):
      sas_block_topk (one row per KV head) -> sas_sparse_decode
Inputs are resident in HBM before timing; L2 is flushed (256 MiB memset)
before every step, outside the timed events.

metric value = kept fwd+bwd FLOPs of the training layer (4d + 10d per kept
(query head, key) pair) / device time of the whole step, over all ranks.
The decode part is reported as HBM GB/s over the selected-KV bytes.

--impl reference times the oracle (fp64, CPU) on a bounded sample of the
same workload instead.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
       under torchrun for N > 1 (one process per GPU, weak scaling: every rank
       runs the full workload).
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "gated sparse attn fwd+bwd TFLOP/s and sparse-decode HBM GB/s vs roofline (1 B200)"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# kernels timed per launch inside the timed loop (sas_kernel_timing): the
# candidates for the dominant kernel only -- each timed launch adds a pair of
# event records between kernels
TIMED_KERNELS = ("bwd_tc", "fwd_rows")


# ----------------------------------------------------------------- workload ---

def kept_pairs_per_row(T, bs, K):
    """Kept (query, key) pairs of each query position t (per query head)."""
    import numpy as np
    t = np.arange(T)
    C = t // bs
    return np.minimum(C, K) * bs + (t - C * bs + 1)


def train_flops(w):
    pairs = int(kept_pairs_per_row(w.seq, w.block_size, w.top_k).sum())
    per_head = pairs * w.batch * w.n_q_heads
    return 4 * w.head_dim * per_head, 10 * w.head_dim * per_head, per_head


def selection_stats(idx, n_sel, T, bs, G, tile=64, rows_per_chunk=128):
    """Selection overlap and executed tensor work of one training selection.

    idx [B, Hkv, T, K] (ascending kept blocks, padded), n_sel [B, Hkv, T] as
    numpy arrays. Per (b, kv head, query tile of `tile` tokens): the number of
    distinct kept blocks (the union a query-tile kernel would visit) and the
    kept selections per visited block. Per (b, kv head, key block j): the
    gathered-row kernels walk 64 own tokens plus every later token that kept
    j, in chunks of 128 / G tokens, each chunk an M = 128 row MMA over the 64
    keys of j; `executed_pairs` counts those row-key products (masked diagonal
    keys and padding rows included), to set beside the kept pairs.
    """
    import numpy as np
    B, Hkv, _, K = idx.shape
    NB = (T + bs - 1) // bs
    tpc = rows_per_chunk // G
    slot = np.arange(K)
    unions, visits, executed = [], [], 0
    for b in range(B):
        for g in range(Hkv):
            ib = idx[b, g]
            valid = slot[None, :] < n_sel[b, g][:, None]
            t_of = np.broadcast_to(np.arange(T)[:, None], ib.shape)
            hit = np.zeros((T // tile, NB), dtype=bool)
            hit[t_of[valid] // tile, ib[valid]] = True
            u = hit.sum(axis=1)
            sels = np.bincount(t_of[valid] // tile, minlength=T // tile)
            keep = u > 0
            unions.append(u[keep])
            visits.append(sels[keep] / u[keep])
            count = bs + np.bincount(ib[valid], minlength=NB)[: T // bs]
            executed += int(((count + tpc - 1) // tpc).sum()) * rows_per_chunk * bs
    u = np.concatenate(unions) if unions else np.zeros(0)
    v = np.concatenate(visits) if visits else np.zeros(0)
    return {"tile_tokens": tile,
            "union_blocks_per_tile": float(u.mean()) if u.size else 0.0,
            "selections_per_visited_block": float(v.mean()) if v.size else 0.0,
            "executed_pairs": executed}


def decode_selected_bytes(w, K):
    N = w.seq
    C = (N - 1) // w.block_size
    cur = N - C * w.block_size
    n = min(K, C)
    esize = 2 if w.dtype == "bf16" else 4
    return w.batch * w.n_kv_heads * (n * w.block_size + cur) * w.head_dim * esize * 2


def decode_graph(B, api, dd, dw, s1c, q1, dc, vc, ws_d, flush, dev, calls=32, reps=5):
    """Per-call time of `calls` sparse decodes replayed from one CUDA graph, each
    on its own index set over the resident cache (selections of seeded score
    perturbations; together larger than L2), L2 flushed before every replay
    outside the timed events. A failure is reported in the result, not raised."""
    import torch
    try:
        gen = torch.Generator().manual_seed(4242)
        sels, outs = [], []
        for _ in range(calls):
            s_r = (s1c + torch.randn(s1c.shape, generator=gen)).to(dev)
            sels.append(api.block_topk(dd, s_r))
            outs.append(torch.empty_like(q1))

        def run_all():
            for r in range(calls):
                B.sas_sparse_decode(dd, q1, dc, vc, dw.seq, sels[r].idx, sels[r].gate_logit, sels[r].n_sel,
                                    outs[r], ws_d)

        run_all()                       # once eagerly: every launch path is set up before capture
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, capture_error_mode="relaxed"):
            run_all()
        stream = torch.cuda.current_stream()
        times = []
        for i in range(reps + 1):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            graph.replay()
            e1.record(stream)
            torch.cuda.synchronize()
            if i > 0:
                times.append(e0.elapsed_time(e1))
        del graph
        per_call_us = statistics.median(times) * 1e3 / calls
        return {"calls": calls, "per_call_us": per_call_us,
                "gbs": decode_selected_bytes(dw, dw.top_k) / (per_call_us * 1e-6) / 1e9,
                "inputs": "distinct index sets over one resident cache; L2 flushed before each replay"}
    except Exception as exc:   # reported beside the other numbers, never fatal
        return {"error": f"{type(exc).__name__}: {exc}"[:200]}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def traffic_record(kernel_file):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current source of the kernel (else None)."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        recs = json.load(f)
    src = os.path.join(ROOT, "trainable_block_sparse_topk_b200", "csrc", kernel_file)
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    for r in recs:
        if r.get("file") == kernel_file and r.get("source_sha") == sha:
            return r
    return None


def max_over_ranks(x, world, device):
    """Max of a per-rank float (a device-timed duration) over all ranks of the
    process group; the value itself at N = 1."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------- clocks ---

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        self.proc.wait()
        rows = [l.strip().split(", ") for l in open(self.path) if l.strip()]
        os.unlink(self.path)
        sm = [float(r[1]) for r in rows if len(r) >= 9 and r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if len(r) >= 9 and r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in rows:
            if len(r) < 9:
                continue
            for n, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------ oracle timing ---

_INPUT_CACHE: dict = {}

def oracle_rate(w, rows_target=None, seconds=10.0, seed=5):
    """Time the oracle (as it stands) on a seeded sample of the training
    workload's rows: forward + backward. Returns (TFLOP/s, rows, seconds, threads)."""
    import numpy as np
    import oracle
    from trainable_block_sparse_topk_b200 import synth

    oracle.build()
    if _INPUT_CACHE.get("name") != w:
        _INPUT_CACHE.clear()
        _INPUT_CACHE.update(name=w, x=synth.train_inputs(w))
    x = _INPUT_CACHE["x"]
    G, bs, K, d = w.group, w.block_size, w.top_k, w.head_dim
    pairs = kept_pairs_per_row(w.seq, bs, K)
    threads = len(os.sched_getaffinity(0))
    rng = np.random.default_rng(seed)
    gd = oracle.Desc(batch=1, seq_len=w.seq, n_q_heads=G, n_kv_heads=1, head_dim=d, block_size=bs, top_k=K)
    arrays = {}

    def group(b, g):
        if (b, g) not in arrays:
            sl = slice(g * G, (g + 1) * G)
            arrays[(b, g)] = {"q": x["q"][b:b + 1, sl].numpy(), "k": x["k"][b:b + 1, g:g + 1].numpy(),
                              "v": x["v"][b:b + 1, g:g + 1].numpy(), "dO": x["dO"][b:b + 1, sl].numpy(),
                              "s": x["scores"][b:b + 1, g:g + 1].numpy()}
        return arrays[(b, g)]

    def run(nrows):
        picks = {}
        for _ in range(nrows):
            b, g, t = int(rng.integers(w.batch)), int(rng.integers(w.n_kv_heads)), int(rng.integers(w.seq))
            picks.setdefault((b, g), []).append(t)
        jobs = []
        for (b, g), ts in picks.items():
            ts = np.array(ts, dtype=np.int64)
            for part in np.array_split(ts, max(1, threads * len(ts) // nrows + 1)):
                if part.size:
                    jobs.append((group(b, g), part))
        flops = sum(int(pairs[ts].sum()) * G * 14 * d for _, ts in jobs)
        t0 = time.perf_counter()
        for a, ts in jobs:                      # forward: OpenMP over rows inside one call
            oracle.fwd(gd, a["q"], a["k"], a["v"], a["s"], ts)
        with cf.ThreadPoolExecutor(threads) as ex:   # backward: one group's rows per call, calls in parallel
            list(ex.map(lambda j: oracle.bwd(gd, j[0]["q"], j[0]["k"], j[0]["v"], j[0]["s"], j[0]["dO"], j[1]),
                        jobs))
        return flops, time.perf_counter() - t0

    if rows_target is None:
        f, s = run(256)
        rows_target = max(256, min(w.batch * w.n_kv_heads * w.seq, int(256 * seconds / max(s, 1e-3))))
    f, s = run(rows_target)
    return f / s / 1e12, rows_target, s, threads


# -------------------------------------------------------------------- ours ---

def run_ours(args, rank, world, local_rank):
    import numpy as np
    import torch
    import torch.distributed as dist

    from trainable_block_sparse_topk_b200 import api, binding as B, synth

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    tw = synth.workload(args.workload)
    dw = synth.workload("decode", top_k=args.decode_k)
    dt = torch.bfloat16 if tw.dtype == "bf16" else torch.float32

    # ---- inputs resident in HBM ----
    x = synth.train_inputs(tw)
    g = {n: x[n].to(dt).to(dev) for n in ("q", "k", "v", "dO")}
    s = x["scores"].to(dev)
    td = B.make_desc(batch=tw.batch, seq_len=tw.seq, n_q_heads=tw.n_q_heads, n_kv_heads=tw.n_kv_heads,
                     head_dim=tw.head_dim, block_size=tw.block_size, top_k=tw.top_k, dtype=tw.dtype)
    sel = api.block_topk(td, s)
    torch.cuda.synchronize()
    sel_stats = selection_stats(sel.idx.cpu().numpy(), sel.n_sel.cpu().numpy(), tw.seq, tw.block_size,
                                tw.n_q_heads // tw.n_kv_heads)
    o = torch.empty_like(g["q"])
    lse = torch.empty(g["q"].shape[:-1], dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(g["q"]), torch.empty_like(g["k"]), torch.empty_like(g["v"])
    ds = torch.empty_like(s)
    ws_f = api.workspace(B.SAS_OP_FWD, td, dev)
    ws_b = api.workspace(B.SAS_OP_BWD, td, dev)

    dc = torch.empty(dw.batch, dw.n_kv_heads, dw.seq, dw.head_dim, dtype=dt, device=dev)
    vc = torch.empty_like(dc)
    for b in range(dw.batch):
        for h in range(dw.n_kv_heads):
            dc[b, h].copy_(synth.decode_cache_slice(dw, "k", b, h).to(dt))
            vc[b, h].copy_(synth.decode_cache_slice(dw, "v", b, h).to(dt))
    q1c = synth.decode_q(dw)
    s1c = synth.decode_scores(dw, q1c)
    q1, s1 = q1c.to(dt).to(dev), s1c.to(dev)
    dd = B.make_desc(batch=dw.batch, seq_len=1, q_offset=dw.seq - 1, n_q_heads=dw.n_q_heads,
                     n_kv_heads=dw.n_kv_heads, head_dim=dw.head_dim, block_size=dw.block_size,
                     top_k=dw.top_k, dtype=dw.dtype)
    sel1 = api.block_topk(dd, s1)
    o1 = torch.empty_like(q1)
    ws_d = api.workspace(B.SAS_OP_DECODE, dd, dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    parts = ["topk", "fwd", "bwd", "decode_topk", "decode"]

    def step(ev):
        ev[0].record(stream)
        B.sas_block_topk(td, s, sel.idx, sel.gate_logit, sel.score_lse, sel.n_sel)
        ev[1].record(stream)
        B.sas_gated_attn_fwd(td, g["q"], g["k"], g["v"], sel.idx, sel.gate_logit, sel.n_sel, o, lse, ws_f)
        ev[2].record(stream)
        B.sas_gated_attn_bwd(td, g["q"], g["k"], g["v"], o, g["dO"], lse, s, sel.score_lse, sel.idx,
                             sel.gate_logit, sel.n_sel, dq, dk, dv, ds, ws_b)
        ev[3].record(stream)
        B.sas_block_topk(dd, s1, sel1.idx, sel1.gate_logit, sel1.score_lse, sel1.n_sel)
        ev[4].record(stream)
        B.sas_sparse_decode(dd, q1, dc, vc, dw.seq, sel1.idx, sel1.gate_logit, sel1.n_sel, o1, ws_d)
        ev[5].record(stream)

    def new_events():
        return [torch.cuda.Event(enable_timing=True) for _ in range(6)]

    def feed():
        # L2 flush, then a short device-side sleep so that the host has enqueued
        # the whole step before the first timed event: the events then measure
        # kernel time, not Python/ctypes submission gaps (both are outside them).
        flush.zero_()
        torch.cuda._sleep(args.feed_cycles)

    for _ in range(args.warmup):
        feed()
        step(new_events())
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()

    sampler = ClockSampler(local_rank)
    sampler.start()
    launches0 = B.sas_kernel_launches()
    B.sas_kernel_timing(",".join(TIMED_KERNELS))   # CUDA events on the launching stream
    evs = []
    for _ in range(args.steps):
        feed()
        ev = new_events()
        step(ev)
        evs.append(ev)
    torch.cuda.synchronize()
    B.sas_kernel_timing(None)
    launches = B.sas_kernel_launches() - launches0
    kern = {}
    for name in TIMED_KERNELS:
        ms, n = B.sas_kernel_time(name)
        if n:
            kern[name] = (ms, n)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = sampler.stop()

    part_ms = {p: [ev[i].elapsed_time(ev[i + 1]) for ev in evs] for i, p in enumerate(parts)}
    step_ms = [ev[0].elapsed_time(ev[5]) for ev in evs]
    total_ms = max_over_ranks(sum(step_ms), world, dev)

    f_fwd, f_bwd, per_head_pairs = train_flops(tw)
    flops = f_fwd + f_bwd
    value = flops * world * args.steps / (total_ms * 1e-3) / 1e12
    mean = {p: statistics.mean(v) for p, v in part_ms.items()}
    peaks, peak_src = load_peaks()

    # roofline of the dominant kernel: its algorithmic work per launch over its
    # mean launch duration (CUDA events around each launch, timed loop above)
    kernels_us = {k: 1e3 * ms / n for k, (ms, n) in kern.items()}
    dom_k = max(kern, key=lambda k: kern[k][0]) if kern else None
    kwork = {"bwd_tc": ("tensor", f_bwd), "fwd_rows": ("tensor", f_fwd)}
    dom = max(("fwd", "bwd", "topk", "decode"), key=lambda p: mean[p])
    kernel_file = {"fwd": "attn_fwd_rows.cu", "bwd": "attn_bwd_tc.cu", "topk": "topk.cu", "decode": "decode.cu"}[dom]
    if dom_k in kwork:
        bound, work = kwork[dom_k]
        sec = kern[dom_k][0] / kern[dom_k][1] * 1e-3
        if bound == "tensor":
            ach = work / sec / 1e12
            roof = {"bound": "tensor", "achieved": ach, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                    "frac": ach / peaks["bf16_tflops"], "peak_source": peak_src + " (bf16 burst)"}
        else:
            ach = work / sec / 1e9
            roof = {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": ach / peaks["hbm_gbs"], "peak_source": peak_src}
        roof.update(kernel=dom_k, launches=kern[dom_k][1], kernel_us=kernels_us[dom_k])
        tr = traffic_record({"bwd_tc": "attn_bwd_tc.cu", "fwd_rows": "attn_fwd_rows.cu"}[dom_k])
        roof["traffic"] = tr["dram_bytes_per_launch"] if tr and tr.get("kernel") == dom_k else None
    elif dom in ("fwd", "bwd"):
        fl = f_fwd if dom == "fwd" else f_bwd
        ach = fl / (mean[dom] * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": ach, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": ach / peaks["bf16_tflops"], "peak_source": peak_src + " (bf16 burst)"}
    elif dom == "decode":
        by = decode_selected_bytes(dw, dw.top_k)
        ach = by / (mean[dom] * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": ach / peaks["hbm_gbs"], "peak_source": peak_src}
    else:
        by = 4 * int(sum(min(t // tw.block_size, 10 ** 9) for t in range(tw.seq))) * tw.batch * tw.n_kv_heads
        ach = by / (mean[dom] * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": ach / peaks["hbm_gbs"], "peak_source": peak_src}
    if "kernel" not in roof:
        roof["call"] = {"fwd": "sas_gated_attn_fwd", "bwd": "sas_gated_attn_bwd", "topk": "sas_block_topk",
                        "decode": "sas_sparse_decode"}[dom]
        tr = traffic_record(kernel_file)
        roof["traffic"] = tr["dram_bytes_per_launch"] if tr and tr.get("call") == roof["call"] else None

    sel_bytes = decode_selected_bytes(dw, dw.top_k)
    dec_gbs = sel_bytes / (mean["decode"] * 1e-3) / 1e9
    decode_info = {"workload": f"decode N{dw.seq} B{dw.batch} Hq{dw.n_q_heads}/Hkv{dw.n_kv_heads} d{dw.head_dim} "
                               f"b{dw.block_size} K{dw.top_k} (budget {(dw.top_k + 1) * dw.block_size})",
                   "selected_bytes": sel_bytes, "decode_us": mean["decode"] * 1e3,
                   "topk_us": mean["decode_topk"] * 1e3, "gbs": dec_gbs, "frac_of_hbm": dec_gbs / peaks["hbm_gbs"],
                   "topk_share": mean["decode_topk"] / (mean["decode_topk"] + mean["decode"])}

    # ---- dense decode comparator (same cache, every token, no gate) ----
    dense_ms = []
    for i in range(args.warmup + args.steps):
        feed()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        B.sas_sparse_decode(dd, q1, dc, vc, dw.seq, None, None, None, o1, ws_d)
        e1.record(stream)
        torch.cuda.synchronize()
        if i >= args.warmup:
            dense_ms.append(e0.elapsed_time(e1))
    dense_bytes = dw.batch * dw.n_kv_heads * dw.seq * dw.head_dim * 2 * 2
    decode_info["dense_us"] = statistics.mean(dense_ms) * 1e3
    decode_info["dense_gbs"] = dense_bytes / (statistics.mean(dense_ms) * 1e-3) / 1e9
    decode_info["sparse_vs_dense_speedup"] = statistics.mean(dense_ms) / (mean["decode"] + mean["decode_topk"])

    # ---- end to end through the public API with host buffers ----
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, tw, dw, x, q1c, s1c, dc, vc, dev, dt, flops, world)

    # ---- decode pipelined: a CUDA graph of 32 calls (run last: it can only add a key) ----
    decode_info["graph"] = decode_graph(B, api, dd, dw, s1c, q1, dc, vc, ws_d, flush, dev)

    result = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": tw.dtype, "data": "synthetic (seeded)",
        "config": {"workload": f"{tw.name}: training fwd+bwd B{tw.batch} T{tw.seq} Hq{tw.n_q_heads}/Hkv{tw.n_kv_heads} "
                               f"d{tw.head_dim} b{tw.block_size} K{tw.top_k} (budget {(tw.top_k + 1) * tw.block_size})"
                               f" + decode N{dw.seq} K{dw.top_k}",
                   "global_batch": tw.batch * world, "seq_len": tw.seq, "parallelism": f"replicas x{world}",
                   "l2": "flushed before every step (256 MiB memset outside the timed events)",
                   "kept_fwd_bwd_tflop_per_step": flops / 1e12, "kept_pairs_per_head": per_head_pairs // (tw.batch * tw.n_q_heads),
                   # tensor work the gathered-row kernels execute (masked diagonal keys and
                   # chunk padding included) and the query-tile union they avoid
                   "executed_fwd_bwd_tflop_per_step": 14 * tw.head_dim * sel_stats["executed_pairs"] / 1e12,
                   "executed_over_kept": sel_stats["executed_pairs"] / per_head_pairs,
                   "selection_overlap": {k: sel_stats[k] for k in ("tile_tokens", "union_blocks_per_tile",
                                                                   "selections_per_visited_block")}},
        "parts_us": {p: mean[p] * 1e3 for p in parts},
        "kernels_us": kernels_us,
        "roofline": roof,
        "decode": decode_info,
        "gpu_launches": launches,
        "clocks": clocks,
    }
    if e2e is not None:
        result["e2e"] = e2e
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, nrows, secs, threads = oracle_rate(tw, seconds=args.cpu_seconds)
        result["cpu_baseline"] = {"value": rate, "unit": UNIT, "cores": threads, "kind": "oracle",
                                  "sample": f"{nrows} seeded query rows of {tw.name} (all G heads each), "
                                            f"fwd+bwd in {secs:.1f} s, kept FLOPs of those rows"}
    return result


def run_e2e(args, tw, dw, x, q1c, s1c, dc, vc, dev, dt, flops, world):
    """Same step through the public API, inputs from pinned host memory and
    results read back to pinned host memory inside the timed region."""
    import torch

    from trainable_block_sparse_topk_b200 import api, binding as B

    host = {n: x[n].to(dt).pin_memory() for n in ("q", "k", "v", "dO")}
    host["scores"] = x["scores"].pin_memory()
    hq1, hs1 = q1c.to(dt).pin_memory(), s1c.pin_memory()
    outs = {"o": torch.empty(x["q"].shape, dtype=dt).pin_memory(),
            "dq": torch.empty(x["q"].shape, dtype=dt).pin_memory(),
            "dk": torch.empty(x["k"].shape, dtype=dt).pin_memory(),
            "dv": torch.empty(x["v"].shape, dtype=dt).pin_memory(),
            "ds": torch.empty(x["scores"].shape, dtype=torch.float32).pin_memory(),
            "o1": torch.empty(q1c.shape, dtype=dt).pin_memory()}
    td = B.make_desc(batch=tw.batch, seq_len=tw.seq, n_q_heads=tw.n_q_heads, n_kv_heads=tw.n_kv_heads,
                     head_dim=tw.head_dim, block_size=tw.block_size, top_k=tw.top_k, dtype=tw.dtype)
    dd = B.make_desc(batch=dw.batch, seq_len=1, q_offset=dw.seq - 1, n_q_heads=dw.n_q_heads,
                     n_kv_heads=dw.n_kv_heads, head_dim=dw.head_dim, block_size=dw.block_size,
                     top_k=dw.top_k, dtype=dw.dtype)
    h2d = sum(t.numel() * t.element_size() for t in host.values()) + hq1.numel() * hq1.element_size() + \
        hs1.numel() * hs1.element_size()
    d2h = sum(t.numel() * t.element_size() for t in outs.values())
    stream = torch.cuda.current_stream()

    def step():
        g = {n: t.to(dev, non_blocking=True) for n, t in host.items()}
        sel = api.block_topk(td, g["scores"])
        o, lse = api.gated_attn_fwd(td, g["q"], g["k"], g["v"], sel)
        dq, dk, dv, ds = api.gated_attn_bwd(td, g["q"], g["k"], g["v"], o, lse, g["dO"], g["scores"], sel)
        q1, s1 = hq1.to(dev, non_blocking=True), hs1.to(dev, non_blocking=True)
        sel1 = api.block_topk(dd, s1)
        o1 = api.sparse_decode(dd, q1, dc, vc, sel1)
        for n, t in (("o", o), ("dq", dq), ("dk", dk), ("dv", dv), ("ds", ds), ("o1", o1)):
            outs[n].copy_(t, non_blocking=True)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    return {"value": flops * world * args.steps / (ms * 1e-3) / 1e12, "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms / args.steps}


# --------------------------------------------------------------- reference ---

def run_reference(args, rank, world):
    """The oracle as the reference arm: each step is the oracle's fwd+bwd on a
    bounded seeded sample of the training workload's rows, on the host cores."""
    if rank != 0:
        return None
    from trainable_block_sparse_topk_b200 import synth
    tw = synth.workload(args.workload)
    rows = args.ref_rows
    for i in range(args.warmup):
        oracle_rate(tw, rows_target=rows, seed=100 + i)
    rates, secs = [], 0.0
    threads = len(os.sched_getaffinity(0))
    for i in range(args.steps):
        r, _, s, threads = oracle_rate(tw, rows_target=rows, seed=200 + i)
        rates.append(r)
        secs += s
    value = statistics.mean(rates)
    return {"metric": METRIC, "value": value, "unit": UNIT, "impl": "reference", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs * 1e3 / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded)",
            "config": {"workload": f"{tw.name}: training fwd+bwd B{tw.batch} T{tw.seq} Hq{tw.n_q_heads}/"
                                   f"Hkv{tw.n_kv_heads} d{tw.head_dim} b{tw.block_size} K{tw.top_k}",
                       "global_batch": tw.batch, "seq_len": tw.seq, "parallelism": "host cores"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": f"{rows} seeded query rows per step (all G heads each), fwd+bwd"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="qwen4b")
    ap.add_argument("--decode-k", type=int, default=31)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--ref-rows", type=int, default=2048)
    ap.add_argument("--feed-cycles", type=int, default=4_000_000,
                    help="device sleep (clock cycles) enqueued before each timed step, outside the events")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}; using {world}", file=sys.stderr)

    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return

    from trainable_block_sparse_topk_b200.build import build
    if rank == 0:
        build()
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
        dist.barrier()
    try:
        res = run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
