#!/usr/bin/env python
"""Benchmark of the SAS gated block-sparse attention hot path on B200.

One step = one pass of the whole path over one batch of synthetic input:
  training layer (Qwen3-14B-like: B2 T32768 Hq40/Hkv8 d128 block 64, K=31):
      sas_block_topk -> sas_gated_attn_fwd -> sas_gated_attn_bwd
  decode (524288-token cache, batch 8, Hq32/Hkv8 d128 block 64, budget 2048 = K31):
      sas_block_topk (one row per batch and KV head) -> sas_sparse_decode
Inputs are resident in HBM before timing; L2 is flushed (256 MiB memset)
before every step, outside the timed events.

metric value = kept fwd+bwd FLOPs of the training layer (4d + 10d per kept
(query head, key) pair) / device time of the whole step, over all ranks.
`decode` reports every decode workload (131072-token cache at budgets
1024/2048/4096, 524288-token cache at batch 1 and 8) as HBM GB/s over the
selected-KV bytes, each timed on its own.

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
# decode part of a step, and the decode workloads reported one by one:
# (workload, batch, K)
DECODE_STEP = ("long", 8, 31)
DECODE_RECORDS = (("decode", 1, 15), ("decode", 1, 31), ("decode", 1, 63), ("long", 1, 31), ("long", 8, 31))


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


def decode_cache(w, dev, dt, threads=16):
    """Device K/V caches [B, Hkv, N, d] of a decode workload, filled slice by
    slice from the seeded generator (the host never holds the whole cache)."""
    import torch
    from trainable_block_sparse_topk_b200 import synth
    kc = torch.empty(w.batch, w.n_kv_heads, w.seq, w.head_dim, dtype=dt, device=dev)
    vc = torch.empty_like(kc)
    jobs = [(which, b, g) for b in range(w.batch) for g in range(w.n_kv_heads) for which in ("k", "v")]

    def make(job):
        which, b, g = job
        return job, synth.decode_cache_slice(w, which, b, g).to(dt).pin_memory()

    with cf.ThreadPoolExecutor(threads) as ex:
        for i in range(0, len(jobs), threads):
            for (which, b, g), sl in ex.map(make, jobs[i:i + threads]):
                (kc if which == "k" else vc)[b, g].copy_(sl, non_blocking=True)
            torch.cuda.synchronize()
    return kc, vc


def decode_graph(B, api, dd, dw, s1c, q1, dc, vc, ws_d, flush, dev, calls=32, caches=8, reps=5):
    """Per-call time of `calls` sparse decodes replayed from one CUDA graph:
    `caches` distinct caches in device memory (the base cache and copies with
    its blocks rotated, together larger than L2), each read by calls/caches
    distinct index sets (selections of seeded score perturbations); L2 flushed
    before every replay, outside the timed events. A failure is reported in
    the result, not raised."""
    import torch
    try:
        gen = torch.Generator().manual_seed(4242)
        ks, vs = [dc], [vc]
        for i in range(1, caches):
            sh = i * 37 * dw.block_size
            ks.append(torch.roll(dc, shifts=sh, dims=2))
            vs.append(torch.roll(vc, shifts=sh, dims=2))
        sels, outs = [], []
        for _ in range(calls):
            s_r = (s1c + torch.randn(s1c.shape, generator=gen)).to(dev)
            sels.append(api.block_topk(dd, s_r))
            outs.append(torch.empty_like(q1))

        def run_all():
            for r in range(calls):
                c = r % caches
                B.sas_sparse_decode(dd, q1, ks[c], vs[c], dw.seq, sels[r].idx, sels[r].gate_logit,
                                    sels[r].n_sel, outs[r], ws_d)

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
        del graph, ks, vs
        per_call_us = statistics.median(times) * 1e3 / calls
        gbs = decode_selected_bytes(dw, dw.top_k) / (per_call_us * 1e-6) / 1e9
        return {"calls": calls, "per_call_us": per_call_us, "gbs": gbs, "frac_of_hbm": gbs / load_peaks()[0]["hbm_gbs"],
                "inputs": f"{caches} distinct caches x {calls // caches} distinct index sets; "
                          "L2 flushed before each replay"}
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

_GROUP_CACHE: dict = {}


def group_inputs(w, b, g, x=None):
    """numpy float32 inputs of one (batch, KV group) sub-problem of training
    workload w: from the full inputs x when given, else drawn for this group
    alone from the seeded generator (the same values)."""
    import torch
    from trainable_block_sparse_topk_b200 import synth
    G = w.group
    if x is not None:
        sl = slice(g * G, (g + 1) * G)
        return {"q": x["q"][b:b + 1, sl].numpy(), "k": x["k"][b:b + 1, g:g + 1].numpy(),
                "v": x["v"][b:b + 1, g:g + 1].numpy(), "dO": x["dO"][b:b + 1, sl].numpy(),
                "s": x["scores"][b:b + 1, g:g + 1].numpy()}
    q = torch.stack([synth.head_slice(w, "q", b, g * G + r, w.seq, w.qkv_std) for r in range(G)])
    dO = torch.stack([synth.head_slice(w, "dO", b, g * G + r, w.seq, 1.0) for r in range(G)])
    k = synth.head_slice(w, "k", b, g, w.seq, w.qkv_std)
    v = synth.head_slice(w, "v", b, g, w.seq, w.qkv_std)
    if w.score_kind == "gauss":
        sc = torch.randn(w.seq, w.n_blocks, generator=synth._gen(w.seed, "s", b, g))
    else:
        kbar = k.reshape(w.n_blocks, w.block_size, w.head_dim).mean(1)
        sc = synth.pooled_scores(w, q.mean(0), kbar, b, g)
    return {"q": q[None].numpy(), "k": k[None, None].numpy(), "v": v[None, None].numpy(),
            "dO": dO[None].numpy(), "s": sc[None, None].numpy()}


def oracle_rate(w, x=None, rows_target=None, seconds=10.0, seed=5, max_groups=None):
    """Time the oracle (as it stands) on a seeded sample of the training
    workload's rows: forward + backward of every sampled (b, kv head, t) row
    with its G heads. The rows are drawn uniformly from all (b, kv head)
    groups, or from `max_groups` seeded groups when given (bounds the input
    drawing). Returns (TFLOP/s, rows, seconds, threads)."""
    import numpy as np
    import oracle

    oracle.build()
    G, bs, K, d = w.group, w.block_size, w.top_k, w.head_dim
    pairs = kept_pairs_per_row(w.seq, bs, K)
    threads = len(os.sched_getaffinity(0))
    rng = np.random.default_rng(seed)
    groups = [(b, g) for b in range(w.batch) for g in range(w.n_kv_heads)]
    if max_groups is not None and max_groups < len(groups):
        groups = [groups[i] for i in rng.choice(len(groups), max_groups, replace=False)]
    gd = oracle.Desc(batch=1, seq_len=w.seq, n_q_heads=G, n_kv_heads=1, head_dim=d, block_size=bs, top_k=K)
    arrays = {}

    def group(bg):
        if x is not None:
            if bg not in arrays:
                arrays[bg] = group_inputs(w, bg[0], bg[1], x)
            return arrays[bg]
        key = (w, bg)
        if key not in _GROUP_CACHE:      # drawn once per process
            _GROUP_CACHE[key] = group_inputs(w, bg[0], bg[1])
        return _GROUP_CACHE[key]

    def run(nrows):
        picks = {}
        for _ in range(nrows):
            bg = groups[int(rng.integers(len(groups)))]
            picks.setdefault(bg, []).append(int(rng.integers(w.seq)))
        jobs = []
        for bg, ts in picks.items():
            ts = np.array(ts, dtype=np.int64)
            for part in np.array_split(ts, max(1, threads * len(ts) // nrows + 1)):
                if part.size:
                    jobs.append((group(bg), part))
        flops = sum(int(pairs[ts].sum()) * G * 14 * d for _, ts in jobs)
        t0 = time.perf_counter()
        for a, ts in jobs:                      # forward: OpenMP over rows inside one call
            oracle.fwd(gd, a["q"], a["k"], a["v"], a["s"], ts)
        with cf.ThreadPoolExecutor(threads) as ex:   # backward: one group's rows per call, calls in parallel
            list(ex.map(lambda j: oracle.bwd(gd, j[0]["q"], j[0]["k"], j[0]["v"], j[0]["s"], j[0]["dO"], j[1]),
                        jobs))
        return flops, time.perf_counter() - t0

    if rows_target is None:
        f, s = run(64)
        rows_target = max(64, min(w.batch * w.n_kv_heads * w.seq, int(64 * seconds / max(s, 1e-3))))
    f, s = run(rows_target)
    return f / s / 1e12, rows_target, s, threads


# -------------------------------------------------------------------- ours ---

def decode_inputs(name, batch, K, dev, dt, caches):
    """Seeded decode inputs of workload `name` at `batch` and budget K: the
    cache (shared between batch sizes of one workload: batch b of the smaller
    one is batch b of the larger), the new token's queries and the block
    scores, on the device; plus the host copies of q and the scores."""
    from trainable_block_sparse_topk_b200 import synth
    w = synth.workload(name, batch=batch, top_k=K)
    if name not in caches or caches[name][0].shape[0] < batch:
        caches[name] = decode_cache(w, dev, dt)
    kc, vc = caches[name]
    kc, vc = kc[:batch], vc[:batch]
    qh = synth.decode_q(w)
    sh = synth.decode_scores(w, qh)
    return w, kc, vc, qh, sh


def paginate(kc, vc, bs, gen):
    """Page pools [P, Hkv, bs, d] holding the blocks of contiguous caches
    [B, Hkv, N, d] in shuffled pages, and the block table [B, N / bs]."""
    import torch
    Bn, H, N, d = kc.shape
    nb = N // bs
    table = torch.randperm(Bn * nb, generator=gen).to(torch.int32).view(Bn, nb).contiguous()
    kp = torch.empty(Bn * nb, H, bs, d, dtype=kc.dtype, device=kc.device)
    vp = torch.empty_like(kp)
    for b in range(Bn):
        idx = table[b].long().to(kc.device)
        kp[idx] = kc[b].view(H, nb, bs, d).transpose(0, 1)
        vp[idx] = vc[b].view(H, nb, bs, d).transpose(0, 1)
    return kp, vp, table.to(kc.device)


def decode_desc(B, w):
    return B.make_desc(batch=w.batch, seq_len=1, q_offset=w.seq - 1, n_q_heads=w.n_q_heads,
                       n_kv_heads=w.n_kv_heads, head_dim=w.head_dim, block_size=w.block_size, top_k=w.top_k,
                       dtype=w.dtype)


def run_ours(args, rank, world, local_rank):
    import torch

    from trainable_block_sparse_topk_b200 import api, binding as B, synth

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    tw = synth.workload(args.workload)
    dt = torch.bfloat16 if tw.dtype == "bf16" else torch.float32
    peaks, peak_src = load_peaks()

    # ---- training inputs resident in HBM ----
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

    # ---- decode inputs: the step's workload, then the others ----
    caches = {}
    dw, dc, vc, q1c, s1c = decode_inputs(*DECODE_STEP, dev, dt, caches)
    q1, s1 = q1c.to(dt).to(dev), s1c.to(dev)
    dd = decode_desc(B, dw)
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

    def new_events(n=6):
        return [torch.cuda.Event(enable_timing=True) for _ in range(n)]

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
        import torch.distributed as dist
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
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    clocks = sampler.stop()

    # every kernel of the step on its own (three more steps, outside the timed
    # loop, CUDA events around each launch): per-launch mean microseconds
    side_names = ("block_topk", "sel_bitmap_T", "sel_stream_index", "sel_stream_fill", "fwd_rows_shift", "fwd_rows",
                  "fwd_rows_finalize", "fwd_rows_fixup", "rowdot", "bwd_tc", "cast_dq", "dscore")
    B.sas_kernel_timing(",".join(side_names))
    for _ in range(3):
        feed()
        step(new_events())
    torch.cuda.synchronize()
    B.sas_kernel_timing(None)
    step_kernels_us = {}
    for name in side_names:
        ms, n = B.sas_kernel_time(name)
        if n:
            step_kernels_us[name] = {"us_per_launch": 1e3 * ms / n, "launches_per_step": n / 3}

    part_ms = {p: [ev[i].elapsed_time(ev[i + 1]) for ev in evs] for i, p in enumerate(parts)}
    step_ms = [ev[0].elapsed_time(ev[5]) for ev in evs]
    total_ms = max_over_ranks(sum(step_ms), world, dev)

    f_fwd, f_bwd, per_head_pairs = train_flops(tw)
    flops = f_fwd + f_bwd
    value = flops * world * args.steps / (total_ms * 1e-3) / 1e12
    mean = {p: statistics.mean(v) for p, v in part_ms.items()}

    # roofline of the dominant kernel: its algorithmic work per launch over its
    # mean launch duration (CUDA events around each launch, timed loop above)
    kernels_us = {k: 1e3 * ms / n for k, (ms, n) in kern.items()}
    train_k = {k: v for k, v in kern.items() if k in ("bwd_tc", "fwd_rows")}
    dom_k = max(train_k, key=lambda k: train_k[k][0]) if train_k else None
    if dom_k is not None:
        work = {"bwd_tc": f_bwd, "fwd_rows": f_fwd}[dom_k]
        sec = kern[dom_k][0] / kern[dom_k][1] * 1e-3
        ach = work / sec / 1e12
        roof = {"bound": "tensor", "achieved": ach, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": ach / peaks["bf16_tflops"], "peak_source": peak_src + " (bf16 burst)",
                "kernel": dom_k, "launches": kern[dom_k][1], "kernel_us": kernels_us[dom_k]}
        tr = traffic_record({"bwd_tc": "attn_bwd_tc.cu", "fwd_rows": "attn_fwd_rows.cu"}[dom_k])
        roof["traffic"] = tr["dram_bytes_per_launch_scaled"].get(tw.name) if tr and tr.get("kernel") == dom_k \
            and isinstance(tr.get("dram_bytes_per_launch_scaled"), dict) else None
    else:   # no tensor-core kernel on this shape: the costlier training call
        dom = max(("fwd", "bwd"), key=lambda p: mean[p])
        fl = f_fwd if dom == "fwd" else f_bwd
        ach = fl / (mean[dom] * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": ach, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": ach / peaks["bf16_tflops"], "peak_source": peak_src + " (bf16 burst)",
                "call": {"fwd": "sas_gated_attn_fwd", "bwd": "sas_gated_attn_bwd"}[dom], "traffic": None}
    # the other timed kernels, each against its own roofline
    kernel_frac = {}
    if "fwd_rows" in kern:
        kernel_frac["fwd_rows"] = f_fwd / (kernels_us["fwd_rows"] * 1e-6) / 1e12 / peaks["bf16_tflops"]
    if "bwd_tc" in kern:
        kernel_frac["bwd_tc"] = f_bwd / (kernels_us["bwd_tc"] * 1e-6) / 1e12 / peaks["bf16_tflops"]
    causal_score_bytes = 4 * sum(min(t // tw.block_size, tw.n_blocks) for t in range(tw.seq)) * tw.batch * tw.n_kv_heads
    topk_gbs = causal_score_bytes / (mean["topk"] * 1e-3) / 1e9

    # ---- every decode workload on its own: top-K, then sparse decode ----
    def time_decode(w, kc, vc, q, sc, dense=False):
        d = decode_desc(B, w)
        sl = api.block_topk(d, sc)
        out = torch.empty_like(q)
        ws = api.workspace(B.SAS_OP_DECODE, d, dev)
        tk, dec = [], []
        for i in range(args.warmup + args.steps):
            feed()
            ev = new_events(3)
            ev[0].record(stream)
            if not dense:
                B.sas_block_topk(d, sc, sl.idx, sl.gate_logit, sl.score_lse, sl.n_sel)
            ev[1].record(stream)
            if dense:
                B.sas_sparse_decode(d, q, kc, vc, w.seq, None, None, None, out, ws)
            else:
                B.sas_sparse_decode(d, q, kc, vc, w.seq, sl.idx, sl.gate_logit, sl.n_sel, out, ws)
            ev[2].record(stream)
            torch.cuda.synchronize()
            if i >= args.warmup:
                tk.append(ev[0].elapsed_time(ev[1]) * 1e3)
                dec.append(ev[1].elapsed_time(ev[2]) * 1e3)
        # means, not medians: single event intervals of a few microseconds come
        # in coarse steps, and only the mean over the steps resolves below one
        return statistics.mean(tk), statistics.mean(dec)

    decode_recs = []
    if not args.no_records:
        for name, batch, K in DECODE_RECORDS:
            w, kc, vc, qh, sh = decode_inputs(name, batch, K, dev, dt, caches)
            q, sc = qh.to(dt).to(dev), sh.to(dev)
            tk_us, dec_us = time_decode(w, kc, vc, q, sc)
            by = decode_selected_bytes(w, K)
            rec = {"workload": f"{name} N{w.seq} B{batch} Hq{w.n_q_heads}/Hkv{w.n_kv_heads} d{w.head_dim} "
                               f"b{w.block_size} K{K} (budget {(K + 1) * w.block_size})",
                   "selected_bytes": by, "topk_us": tk_us, "decode_us": dec_us,
                   "gbs": by / (dec_us * 1e-6) / 1e9, "frac_of_hbm": by / (dec_us * 1e-6) / 1e9 / peaks["hbm_gbs"],
                   "topk_share": tk_us / (tk_us + dec_us)}
            if (name, K) in (("decode", 31), ("long", 31)) and batch == 1:
                _, dense_us = time_decode(w, kc, vc, q, sc, dense=True)
                dense_bytes = w.batch * w.n_kv_heads * w.seq * w.head_dim * 2 * 2
                rec.update(dense_us=dense_us, dense_gbs=dense_bytes / (dense_us * 1e-6) / 1e9,
                           sparse_vs_dense_speedup=dense_us / (dec_us + tk_us))
            decode_recs.append(rec)
        # paged pools with a cache length per sequence: the batch-8 workload's
        # blocks in shuffled pages, sequence b of length N - 4097 b
        pw, pkc, pvc, pqh, psh = decode_inputs("long", 8, 31, dev, dt, caches)
        kp, vp, table = paginate(pkc, pvc, pw.block_size, torch.Generator().manual_seed(43))
        lens = torch.tensor([pw.seq - 4097 * b for b in range(pw.batch)], dtype=torch.int32, device=dev)
        pd = decode_desc(B, pw)
        pq, ps = pqh.to(dt).to(dev), psh.to(dev)
        psel = api.block_topk_varlen(pd, ps, lens)
        pws = api.workspace(B.SAS_OP_DECODE, pd, dev)
        po = torch.empty_like(pq)
        ptk, pdec = [], []
        for i in range(args.warmup + args.steps):
            feed()
            ev = new_events(3)
            ev[0].record(stream)
            B.sas_block_topk_varlen(pd, ps, lens, psel.idx, psel.gate_logit, psel.score_lse, psel.n_sel)
            ev[1].record(stream)
            B.sas_sparse_decode_paged(pd, pq, kp, vp, table, lens, psel.idx, psel.gate_logit, psel.n_sel, po, pws)
            ev[2].record(stream)
            torch.cuda.synchronize()
            if i >= args.warmup:
                ptk.append(ev[0].elapsed_time(ev[1]) * 1e3)
                pdec.append(ev[1].elapsed_time(ev[2]) * 1e3)
        pby = sum(pw.n_kv_heads * (min(31, (int(n) - 1) // 64) * 64 + int(n) - (int(n) - 1) // 64 * 64) * 128 * 4
                  for n in lens.tolist())
        tk_us, dec_us = statistics.mean(ptk), statistics.mean(pdec)
        decode_recs.append({"workload": f"paged long N<={pw.seq} (N_b = N - 4097 b) B{pw.batch} Hq{pw.n_q_heads}/"
                                        f"Hkv{pw.n_kv_heads} d128 b64 K31, shuffled pages",
                            "selected_bytes": pby, "topk_us": tk_us, "decode_us": dec_us,
                            "gbs": pby / (dec_us * 1e-6) / 1e9, "frac_of_hbm": pby / (dec_us * 1e-6) / 1e9 / peaks["hbm_gbs"],
                            "topk_share": tk_us / (tk_us + dec_us)})
        del kp, vp
        torch.cuda.empty_cache()

        # the serving step in one call: pooled-key scan of every cached block,
        # top-K, sparse decode (batch-8 long cache; kbar = each block's mean key)
        kbar = torch.stack([pkc[b].float().view(pw.n_kv_heads, -1, pw.block_size, pw.head_dim).mean(2).to(dt)
                            for b in range(pw.batch)])
        pdd = decode_desc(B, pw)
        sc_buf = torch.empty(pw.batch, pw.n_kv_heads, 1, pw.n_blocks, dtype=torch.float32, device=dev)
        psel2 = api.block_topk(pdd, sc_buf.zero_())
        po2 = torch.empty_like(pq)
        pws2 = api.workspace(B.SAS_OP_DECODE, pdd, dev)
        scan_us, call_us = [], []
        for i in range(args.warmup + args.steps):
            feed()
            ev = new_events(3)
            ev[0].record(stream)
            B.sas_block_scores_pooled(pdd, pq, kbar, sc_buf)
            ev[1].record(stream)
            B.sas_sparse_decode_pooled(pdd, pq, pkc, pvc, pw.seq, kbar, sc_buf, psel2.idx, psel2.gate_logit,
                                       psel2.score_lse, psel2.n_sel, po2, pws2)
            ev[2].record(stream)
            torch.cuda.synchronize()
            if i >= args.warmup:
                scan_us.append(ev[0].elapsed_time(ev[1]) * 1e3)
                call_us.append(ev[1].elapsed_time(ev[2]) * 1e3)
        C5 = (pw.seq - 1) // pw.block_size
        scan_bytes = pw.batch * pw.n_kv_heads * C5 * pw.head_dim * 2
        sby = decode_selected_bytes(pw, 31)
        su, cu = statistics.mean(scan_us), statistics.mean(call_us)
        decode_recs.append({"workload": f"pooled-key scan + top-K + decode in one call, long N{pw.seq} B{pw.batch} K31",
                            "scan_bytes": scan_bytes, "scan_us": su, "scan_gbs": scan_bytes / (su * 1e-6) / 1e9,
                            "scan_frac_of_hbm": scan_bytes / (su * 1e-6) / 1e9 / peaks["hbm_gbs"],
                            "selected_bytes": sby, "call_us": cu, "scan_share": su / cu,
                            "call_gbs_scan_plus_selected": (scan_bytes + sby) / (cu * 1e-6) / 1e9})
        del kbar
        torch.cuda.empty_cache()
        # per-query-head selection: decode on the batch-1 long cache, each of the
        # 32 query heads with its own 31 blocks (selected bytes summed per head)
        hw, hkc, hvc, hq, _ = decode_inputs("long", 1, 31, dev, dt, caches)
        hd = B.make_desc(batch=1, seq_len=1, q_offset=hw.seq - 1, n_q_heads=hw.n_q_heads, n_kv_heads=hw.n_kv_heads,
                         head_dim=hw.head_dim, block_size=hw.block_size, top_k=31, dtype=hw.dtype, select_heads=True)
        hs = torch.randn(1, hw.n_q_heads, 1, hw.n_blocks, generator=torch.Generator().manual_seed(77)).to(dev)
        hsel = api.block_topk(hd, hs)
        hqd = hq.to(dt).to(dev)
        ho = torch.empty_like(hqd)
        hws = api.workspace(B.SAS_OP_DECODE, hd, dev)
        htk, hdec = [], []
        for i in range(args.warmup + args.steps):
            feed()
            ev = new_events(3)
            ev[0].record(stream)
            B.sas_block_topk(hd, hs, hsel.idx, hsel.gate_logit, hsel.score_lse, hsel.n_sel)
            ev[1].record(stream)
            B.sas_sparse_decode(hd, hqd, hkc, hvc, hw.seq, hsel.idx, hsel.gate_logit, hsel.n_sel, ho, hws)
            ev[2].record(stream)
            torch.cuda.synchronize()
            if i >= args.warmup:
                htk.append(ev[0].elapsed_time(ev[1]) * 1e3)
                hdec.append(ev[1].elapsed_time(ev[2]) * 1e3)
        hby = hw.n_q_heads * decode_selected_bytes(hw, 31) // hw.n_kv_heads
        tk_us, dec_us = statistics.mean(htk), statistics.mean(hdec)
        decode_recs.append({"workload": f"per-query-head selection, long N{hw.seq} B1 Hq{hw.n_q_heads}/Hkv"
                                        f"{hw.n_kv_heads} K31 (one selection per query head)",
                            "selected_bytes": hby, "topk_us": tk_us, "decode_us": dec_us,
                            "gbs": hby / (dec_us * 1e-6) / 1e9, "frac_of_hbm": hby / (dec_us * 1e-6) / 1e9 / peaks["hbm_gbs"],
                            "topk_share": tk_us / (tk_us + dec_us)})
        torch.cuda.empty_cache()
    # per-query-head selection, training: the Qwen3-4B-like layer with one score
    # row per query head (the group's scores plus seeded per-head noise)
    per_head_train = None
    if not args.no_records:
        pw4 = synth.workload("qwen4b")
        x4 = synth.train_inputs(pw4)
        g4 = {n: x4[n].to(dt).to(dev) for n in ("q", "k", "v", "dO")}
        s4 = (x4["scores"].repeat_interleave(pw4.n_q_heads // pw4.n_kv_heads, 1) +
              0.5 * torch.randn(pw4.batch, pw4.n_q_heads, pw4.seq, pw4.n_blocks,
                                generator=torch.Generator().manual_seed(78))).to(dev)
        del x4
        d4 = B.make_desc(batch=pw4.batch, seq_len=pw4.seq, n_q_heads=pw4.n_q_heads, n_kv_heads=pw4.n_kv_heads,
                         head_dim=pw4.head_dim, block_size=pw4.block_size, top_k=pw4.top_k, dtype=pw4.dtype,
                         select_heads=True)
        sel4 = api.block_topk(d4, s4)
        wf4, wb4 = api.workspace(B.SAS_OP_FWD, d4, dev), api.workspace(B.SAS_OP_BWD, d4, dev)
        o4, lse4 = torch.empty_like(g4["q"]), torch.empty(g4["q"].shape[:-1], dtype=torch.float32, device=dev)
        dq4, dk4, dv4 = torch.empty_like(g4["q"]), torch.empty_like(g4["k"]), torch.empty_like(g4["v"])
        ds4 = torch.empty_like(s4)
        t4 = []
        for i in range(args.warmup + args.steps):
            feed()
            ev = new_events(2)
            ev[0].record(stream)
            B.sas_block_topk(d4, s4, sel4.idx, sel4.gate_logit, sel4.score_lse, sel4.n_sel)
            B.sas_gated_attn_fwd(d4, g4["q"], g4["k"], g4["v"], sel4.idx, sel4.gate_logit, sel4.n_sel, o4, lse4, wf4)
            B.sas_gated_attn_bwd(d4, g4["q"], g4["k"], g4["v"], o4, g4["dO"], lse4, s4, sel4.score_lse, sel4.idx,
                                 sel4.gate_logit, sel4.n_sel, dq4, dk4, dv4, ds4, wb4)
            ev[1].record(stream)
            torch.cuda.synchronize()
            if i >= args.warmup:
                t4.append(ev[0].elapsed_time(ev[1]))
        f4f, f4b, _ = train_flops(pw4)
        ms4 = statistics.mean(t4)
        per_head_train = {"workload": f"qwen4b layer B{pw4.batch} T{pw4.seq} Hq{pw4.n_q_heads}/Hkv{pw4.n_kv_heads} "
                                      f"K{pw4.top_k}, one selection per query head",
                          "step_ms": ms4, "kept_fwd_bwd_tflop": (f4f + f4b) / 1e12,
                          "tflops": (f4f + f4b) / (ms4 * 1e-3) / 1e12}
        del g4, s4, wf4, wb4, o4, dq4, dk4, dv4, ds4, sel4
        torch.cuda.empty_cache()
    step_by = decode_selected_bytes(dw, DECODE_STEP[2])
    # the same event pair around one trivial kernel: the floor under every
    # isolated microsecond-scale time above (launch and event overhead)
    tiny = torch.zeros(1, device=dev)
    floor = []
    for i in range(args.warmup + args.steps):
        feed()
        ev = new_events(2)
        ev[0].record(stream)
        tiny.add_(1.0)
        ev[1].record(stream)
        torch.cuda.synchronize()
        if i >= args.warmup:
            floor.append(ev[0].elapsed_time(ev[1]) * 1e3)
    decode_info = {"peak_hbm_gbs": peaks["hbm_gbs"], "peak_source": peak_src,
                   "one_trivial_kernel_us": statistics.mean(floor), "records": decode_recs,
                   "step_part": {"workload": f"{dw.name} N{dw.seq} B{dw.batch} K{DECODE_STEP[2]}",
                                 "topk_us": mean["decode_topk"] * 1e3, "decode_us": mean["decode"] * 1e3,
                                 "gbs": step_by / (mean["decode"] * 1e-3) / 1e9}}

    # ---- end to end through the public API with host buffers ----
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, tw, x, dw, dc, vc, q1c, s1c, dev, dt, flops, world)

    # ---- decode pipelined: a CUDA graph of 32 calls over distinct caches (run last) ----
    if not args.no_records:
        gw, gkc, gvc, gq, gs = decode_inputs("decode", 1, 31, dev, dt, caches)
        decode_info["graph"] = decode_graph(B, api, decode_desc(B, gw), gw, gs, gq.to(dt).to(dev), gkc, gvc,
                                            api.workspace(B.SAS_OP_DECODE, decode_desc(B, gw), dev), flush, dev)
        decode_info["graph"]["workload"] = f"decode N{gw.seq} B1 K31"
        # the batch-8 long-cache decode the same way: 3 caches (the base one and
        # two rotated copies, 17 GB each) x 8 index sets, 67 MB selected per call
        lw, lkc, lvc, lq, ls = decode_inputs("long", 8, 31, dev, dt, caches)
        decode_info["graph_long_b8"] = decode_graph(B, api, decode_desc(B, lw), lw, ls, lq.to(dt).to(dev), lkc, lvc,
                                                    api.workspace(B.SAS_OP_DECODE, decode_desc(B, lw), dev), flush,
                                                    dev, calls=24, caches=3)
        decode_info["graph_long_b8"]["workload"] = f"long N{lw.seq} B8 K31"

    result = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": tw.dtype, "data": "synthetic (seeded)",
        "config": {"workload": f"{tw.name}: training fwd+bwd B{tw.batch} T{tw.seq} Hq{tw.n_q_heads}/Hkv{tw.n_kv_heads} "
                               f"d{tw.head_dim} b{tw.block_size} K{tw.top_k} (budget {(tw.top_k + 1) * tw.block_size})"
                               f" + sparse decode N{dw.seq} B{dw.batch} K{dw.top_k}",
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
        "step_kernels_us": step_kernels_us,
        "kernel_frac_of_bf16_peak": kernel_frac,
        "topk": {"causal_score_bytes": causal_score_bytes, "gbs": topk_gbs, "frac_of_hbm": topk_gbs / peaks["hbm_gbs"]},
        "roofline": roof,
        "decode": decode_info,
        "per_head_training": per_head_train,
        "gpu_launches": launches,
        "clocks": clocks,
    }
    if e2e is not None:
        result["e2e"] = e2e
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, nrows, secs, threads = oracle_rate(tw, x=x, seconds=args.cpu_seconds)
        result["cpu_baseline"] = {"value": rate, "unit": UNIT, "cores": threads, "kind": "oracle",
                                  "sample": f"{nrows} seeded query rows of {tw.name} drawn uniformly over all "
                                            f"(batch, KV head) groups (all G heads each), fwd+bwd in {secs:.1f} s; "
                                            f"rate = kept FLOPs of those rows / time"}
    return result


def run_e2e(args, tw, x, dw, dc, vc, q1c, s1c, dev, dt, flops, world):
    """Same step through the public API, inputs from pinned host memory and
    every output read back to pinned host memory inside the timed region.
    Copies run on their own streams, as a training loop would run them: the
    inputs of step i + 1 go up while step i computes, and the results of step
    i come down while step i + 1 computes; the timed region starts before the
    first upload and ends after the last read-back."""
    import torch

    from trainable_block_sparse_topk_b200 import api, binding as B

    host = {n: x[n].to(dt).pin_memory() for n in ("q", "k", "v", "dO")}
    host["scores"] = x["scores"].pin_memory()
    host["q1"], host["s1"] = q1c.to(dt).pin_memory(), s1c.pin_memory()
    outs = {"o": torch.empty(x["q"].shape, dtype=dt).pin_memory(),
            "dq": torch.empty(x["q"].shape, dtype=dt).pin_memory(),
            "dk": torch.empty(x["k"].shape, dtype=dt).pin_memory(),
            "dv": torch.empty(x["v"].shape, dtype=dt).pin_memory(),
            "ds": torch.empty(x["scores"].shape, dtype=torch.float32).pin_memory(),
            "o1": torch.empty(q1c.shape, dtype=dt).pin_memory()}
    td = B.make_desc(batch=tw.batch, seq_len=tw.seq, n_q_heads=tw.n_q_heads, n_kv_heads=tw.n_kv_heads,
                     head_dim=tw.head_dim, block_size=tw.block_size, top_k=tw.top_k, dtype=tw.dtype)
    dd = decode_desc(B, dw)
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = sum(t.numel() * t.element_size() for t in outs.values())
    comp = torch.cuda.current_stream()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()

    def upload():
        with torch.cuda.stream(up):
            g = {n: t.to(dev, non_blocking=True) for n, t in host.items()}
        ev = torch.cuda.Event()
        ev.record(up)
        return g, ev

    def compute(g):
        for t in g.values():
            t.record_stream(comp)
        sel = api.block_topk(td, g["scores"])
        o, lse = api.gated_attn_fwd(td, g["q"], g["k"], g["v"], sel)
        dq, dk, dv, ds = api.gated_attn_bwd(td, g["q"], g["k"], g["v"], o, lse, g["dO"], g["scores"], sel)
        sel1 = api.block_topk(dd, g["s1"])
        o1 = api.sparse_decode(dd, g["q1"], dc, vc, sel1)
        return {"o": o, "dq": dq, "dk": dk, "dv": dv, "ds": ds, "o1": o1}

    def download(res):
        ev = torch.cuda.Event()
        ev.record(comp)
        down.wait_event(ev)
        with torch.cuda.stream(down):
            for n, t in res.items():
                t.record_stream(down)
                outs[n].copy_(t, non_blocking=True)

    def run(n):
        nxt = upload()
        for i in range(n):
            g, ev = nxt
            comp.wait_event(ev)
            if i + 1 < n:
                nxt = upload()      # the next step's inputs go up while this one computes
            download(compute(g))
        comp.wait_stream(down)

    run(args.warmup)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    up.wait_event(e0)
    run(args.steps)
    e1.record(comp)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    return {"value": flops * world * args.steps / (ms * 1e-3) / 1e12, "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms / args.steps,
            "copies": "pinned host buffers; uploads and read-backs on their own streams, overlapping the "
                      "neighbouring steps' compute; timed from before the first upload to after the last read-back"}


# --------------------------------------------------------------- reference ---

def run_reference(args, rank, world):
    """The oracle as the reference arm: each step is the oracle's fwd+bwd on a
    bounded seeded sample of the training workload's rows, on the host cores
    (rows drawn from a few seeded (batch, KV head) groups, whose inputs are
    drawn alone)."""
    if rank != 0:
        return None
    from trainable_block_sparse_topk_b200 import synth
    tw = synth.workload(args.workload)
    rows = args.ref_rows
    for i in range(args.warmup):
        oracle_rate(tw, rows_target=rows, seed=100 + i, max_groups=2)
    rates, secs = [], 0.0
    threads = len(os.sched_getaffinity(0))
    for i in range(args.steps):
        r, _, s, threads = oracle_rate(tw, rows_target=rows, seed=200 + i, max_groups=2)
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
                             "sample": f"{rows} seeded query rows per step from 2 seeded (batch, KV head) groups "
                                       "(all G heads each), fwd+bwd"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    global DECODE_STEP
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="qwen14b")
    ap.add_argument("--decode", default=":".join(map(str, DECODE_STEP)),
                    help="decode part of the step, workload:batch:K")
    ap.add_argument("--no-records", action="store_true",
                    help="skip the per-workload decode records and the decode graph (smaller runs for profiling)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--ref-rows", type=int, default=512)
    ap.add_argument("--feed-cycles", type=int, default=4_000_000,
                    help="device sleep (clock cycles) enqueued before each timed step, outside the events")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    dn, db, dk = args.decode.split(":")
    DECODE_STEP = (dn, int(db), int(dk))

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
