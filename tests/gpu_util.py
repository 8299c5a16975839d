"""Helpers for the GPU parity tests: run the libsas path on a workload and
compute the oracle's values for chosen rows, one (batch, KV group) at a time.

The oracle always receives the CPU float32 copies of the very inputs the GPU
received (bf16 values are exact in float32); nothing computed on the GPU is
ever given to it.
"""
from __future__ import annotations

import concurrent.futures as cf

import numpy as np
import torch

import oracle
from trainable_block_sparse_topk_b200 import api, binding as B, synth


def dev_dtype(w):
    return torch.float32 if w.dtype == "fp32" else torch.bfloat16


def train_desc(w, **over):
    kw = dict(batch=w.batch, seq_len=w.seq, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads,
              head_dim=w.head_dim, block_size=w.block_size, top_k=w.top_k, dtype=w.dtype)
    kw.update(over)
    return B.make_desc(**kw)


def run_train(w, inputs=None, gate="softmax", with_bwd=True, **over):
    """Top-K + forward (+ backward) through the C ABI. Returns (inputs, out)."""
    x = synth.train_inputs(w) if inputs is None else inputs
    d = train_desc(w, gate=gate, **over)
    dt = dev_dtype(w)
    g = {n: x[n].to(dt).cuda() for n in ("q", "k", "v", "dO")}
    s = x["scores"].cuda()
    sel = api.block_topk(d, s)
    o, lse = api.gated_attn_fwd(d, g["q"], g["k"], g["v"], sel)
    out = {"idx": sel.idx, "gl": sel.gate_logit, "slse": sel.score_lse, "nsel": sel.n_sel, "o": o, "lse": lse}
    if with_bwd:
        dq, dk, dv, ds = api.gated_attn_bwd(d, g["q"], g["k"], g["v"], o, lse, g["dO"], s, sel)
        out.update(dq=dq, dk=dk, dv=dv, ds=ds)
    torch.cuda.synchronize()
    return x, {k: v.cpu() for k, v in out.items()}


def group_desc(w, gate=oracle.GATE_SOFTMAX, top_k=None):
    """Oracle descriptor of one (batch, KV group) sub-problem."""
    return oracle.Desc(batch=1, seq_len=w.seq, n_q_heads=w.group, n_kv_heads=1, head_dim=w.head_dim,
                       block_size=w.block_size, top_k=w.top_k if top_k is None else top_k, gate=gate)


def group_arrays(x, w, b, g):
    G = w.group
    sl = slice(g * G, (g + 1) * G)
    return {"q": x["q"][b:b + 1, sl].numpy(), "k": x["k"][b:b + 1, g:g + 1].numpy(),
            "v": x["v"][b:b + 1, g:g + 1].numpy(), "dO": x["dO"][b:b + 1, sl].numpy(),
            "s": x["scores"][b:b + 1, g:g + 1].numpy()}


def sample_rows(w, n, seed):
    """Seeded sample of (b, g, t): the first rows (fewer candidates than K),
    tile edges, the last row and uniform picks."""
    rng = np.random.default_rng(seed)
    T, bs = w.seq, w.block_size
    fixed = [0, 1, bs - 1, bs, 2 * bs - 1, (w.top_k + 1) * bs, T // 2, T - bs, T - 1]
    ts = sorted(set([t for t in fixed if 0 <= t < T] + list(rng.integers(0, T, size=n))))
    out = []
    for t in ts:
        out.append((int(rng.integers(0, w.batch)), int(rng.integers(0, w.n_kv_heads)), int(t)))
    return out


def by_group(rows):
    grp = {}
    for b, g, t in rows:
        grp.setdefault((b, g), []).append(t)
    return grp


def rows_touching_block(w, x, b, g, j, gate):
    """Rows of group (b, g) whose attention includes key block j, per the
    oracle's own selection: the block's own queries (it is their current
    block) and every later query whose top-K keeps j."""
    a = group_arrays(x, w, b, g)
    d = group_desc(w, gate)
    bs = w.block_size
    cand = np.arange((j + 1) * bs, w.seq, dtype=np.int64)
    rows = list(range(j * bs, (j + 1) * bs))
    if cand.size:
        idx, _, _, nsel = oracle.topk(d, a["s"], cand)
        keep = (idx == j).any(1)
        rows += cand[keep].tolist()
    return np.array(sorted(rows), dtype=np.int64)


def parallel_oracle_bwd(d, a, rows, chunks=8):
    """oracle.bwd over row chunks in threads (the C call releases the GIL);
    row-local outputs are concatenated and dk/dv summed."""
    parts = [c for c in np.array_split(rows, min(chunks, max(1, rows.size))) if c.size]
    with cf.ThreadPoolExecutor(len(parts)) as ex:
        res = list(ex.map(lambda r: oracle.bwd(d, a["q"], a["k"], a["v"], a["s"], a["dO"], r), parts))
    out = {k: np.concatenate([r[k] for r in res]) for k in ("dq", "gsum", "gsum_cur", "ds")}
    out["dk"] = sum(r["dk"] for r in res)
    out["dv"] = sum(r["dv"] for r in res)
    return out


def normwise(got, ref):
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    den = max(np.abs(ref).max(), 1e-30)
    return float(np.abs(got - ref).max() / den)


# ------------------------------------------------------------------- decode ---

def decode_desc(w, N, top_k=None, gate="softmax", batch=None):
    return B.make_desc(batch=w.batch if batch is None else batch, seq_len=1, q_offset=N - 1,
                       n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads, head_dim=w.head_dim,
                       block_size=w.block_size, top_k=w.top_k if top_k is None else top_k, dtype=w.dtype,
                       gate=gate)


def build_decode_cache(w, threads=16):
    """Device K/V caches [B, Hkv, N, d] filled slice by slice from the seeded
    generator (the CPU never holds the whole cache)."""
    dt = dev_dtype(w)
    kc = torch.empty(w.batch, w.n_kv_heads, w.seq, w.head_dim, dtype=dt, device="cuda")
    vc = torch.empty_like(kc)
    jobs = [(which, b, g) for b in range(w.batch) for g in range(w.n_kv_heads) for which in ("k", "v")]

    def make(job):
        which, b, g = job
        return job, synth.decode_cache_slice(w, which, b, g).to(dt).pin_memory()

    with cf.ThreadPoolExecutor(threads) as ex:
        for i in range(0, len(jobs), threads):
            chunk = list(ex.map(make, jobs[i:i + threads]))
            for (which, b, g), sl in chunk:
                (kc if which == "k" else vc)[b, g].copy_(sl, non_blocking=True)
            torch.cuda.synchronize()     # the pinned slices of this chunk may now be freed
    return kc, vc

