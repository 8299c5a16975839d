"""The oracle for SAS gated block-sparse causal attention (fp64, CPU).

TEST INFRASTRUCTURE. Only the test suite, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline / reference arm may import this package. The
product library never imports it, and this package imports nothing from the
product.

The arithmetic lives in ``sas_oracle.c`` (plain loops, double precision); this
module compiles it with gcc on first use and marshals numpy arrays to it.
Every function takes float32 inputs (bf16 data is exact in float32) and
returns float64 results, except indices (int32).

Row ids: a training row is r = (b * Hkv + g) * T + t, one (batch, KV group,
query position) whose G query heads share one block selection.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sas_oracle.c")
_LIB = os.path.join(_HERE, "libsas_oracle.so")

GATE_SOFTMAX = 0
GATE_NONE = 1
GATE_SIGMOID = 2            # independent gates sigmoid(s_i)
GATE_RAW = 3                # the raw score as the log-gate
GATE_SOFTMAX_SELECTED = 4   # softmax over the kept blocks only
GATE_STE = 5                # hard gate 1 on kept blocks, softmax-gate gradient (straight-through)


def build(force: bool = False) -> str:
    """Compile sas_oracle.c into libsas_oracle.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               "-Wall", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Desc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("seq_len", ctypes.c_int32),
                ("q_offset", ctypes.c_int32), ("n_q_heads", ctypes.c_int32),
                ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("block_size", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("scale", ctypes.c_double), ("gate", ctypes.c_int32)]


@dataclass
class Desc:
    """Problem shape, in the notation of the method: B, T, Hq, Hkv, d, block size, K."""
    batch: int
    seq_len: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    block_size: int
    top_k: int
    q_offset: int = 0
    scale: float = 0.0          # <= 0 -> 1/sqrt(head_dim)
    gate: int = GATE_SOFTMAX

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def n_blocks(self) -> int:
        return -(-(self.q_offset + self.seq_len) // self.block_size)

    @property
    def n_rows(self) -> int:
        return self.batch * self.n_kv_heads * self.seq_len

    def c(self) -> _Desc:
        return _Desc(self.batch, self.seq_len, self.q_offset, self.n_q_heads, self.n_kv_heads,
                     self.head_dim, self.block_size, self.top_k, float(self.scale), self.gate)


_lib = None


def _setup(lib):
    """Declare the C signatures on a loaded oracle library."""
    P = ctypes.c_void_p
    I64 = ctypes.c_int64
    D = ctypes.POINTER(_Desc)
    lib.sas_oracle_topk.argtypes = [D, P, I64, P, P, P, P, P]
    lib.sas_oracle_fwd.argtypes = [D, P, P, P, P, I64, P, P, P]
    lib.sas_oracle_bwd.argtypes = [D, P, P, P, P, P, I64, P, P, P, P, P, P, P]
    lib.sas_oracle_decode.argtypes = [D, P, P, P, I64, P, P]
    for f in (lib.sas_oracle_topk, lib.sas_oracle_fwd, lib.sas_oracle_bwd, lib.sas_oracle_decode):
        f.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = _setup(ctypes.CDLL(build()))
    return _lib


def _f32(a) -> np.ndarray:
    a = np.asarray(a)
    if a.dtype != np.float32 or not a.flags.c_contiguous:
        a = np.ascontiguousarray(a, dtype=np.float32)
    return a


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


def _rows(desc: Desc, rows) -> np.ndarray:
    if rows is None:
        return np.arange(desc.n_rows, dtype=np.int64)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    if rows.size and (rows.min() < 0 or rows.max() >= desc.n_rows):
        raise ValueError("row id out of range")
    return rows


def topk(desc: Desc, scores, rows=None):
    """Gate normaliser and hard top-K for the listed rows.

    scores: [B, Hkv, T, NB] float32. Returns (idx [n,K] int32 ascending, -1
    padded; gate_logit [n,K] f64, 0 in padding; score_lse [n] f64; n_sel [n])."""
    s = _f32(scores)
    assert s.size == desc.n_rows * desc.n_blocks, "scores shape"
    rows = _rows(desc, rows)
    n, K = rows.size, desc.top_k
    idx = np.empty((n, K), np.int32)
    gl = np.empty((n, K), np.float64)
    lse = np.empty(n, np.float64)
    nsel = np.empty(n, np.int32)
    d = desc.c()
    rc = _load().sas_oracle_topk(ctypes.byref(d), _ptr(s), n, _ptr(rows), _ptr(idx), _ptr(gl),
                                 _ptr(lse), _ptr(nsel))
    assert rc == 0
    return idx, gl, lse, nsel


def fwd(desc: Desc, q, k, v, scores, rows=None):
    """Gated sparse forward of the listed rows.

    q [B,Hq,T,d], k/v [B,Hkv,T,d], scores [B,Hkv,T,NB] (float32).
    Returns (o [n,G,d] f64, attn_lse [n,G] f64)."""
    q, k, v, s = _f32(q), _f32(k), _f32(v), _f32(scores)
    rows = _rows(desc, rows)
    n, G = rows.size, desc.group
    o = np.empty((n, G, desc.head_dim), np.float64)
    lse = np.empty((n, G), np.float64)
    d = desc.c()
    rc = _load().sas_oracle_fwd(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(s), n, _ptr(rows),
                                _ptr(o), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle fwd: training rows need q_offset == 0")
    return o, lse


def bwd(desc: Desc, q, k, v, scores, dO, rows=None):
    """Backward of the listed rows with upstream gradient dO [B,Hq,T,d].

    Returns dict with dq [n,G,d], dk/dv [B,Hkv,T,d] (contributions of the
    listed rows only), gsum [n,K], gsum_cur [n], ds [n,NB] (all float64)."""
    q, k, v, s, dO = _f32(q), _f32(k), _f32(v), _f32(scores), _f32(dO)
    rows = _rows(desc, rows)
    n, G, K, dh = rows.size, desc.group, desc.top_k, desc.head_dim
    dq = np.empty((n, G, dh), np.float64)
    kv_shape = (desc.batch, desc.n_kv_heads, desc.seq_len, dh)
    dk = np.zeros(kv_shape, np.float64)
    dv = np.zeros(kv_shape, np.float64)
    gsum = np.empty((n, K), np.float64)
    gcur = np.empty(n, np.float64)
    ds = np.empty((n, desc.n_blocks), np.float64)
    d = desc.c()
    rc = _load().sas_oracle_bwd(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(s), _ptr(dO), n,
                                _ptr(rows), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(gsum), _ptr(gcur),
                                _ptr(ds))
    if rc != 0:
        raise ValueError("oracle bwd: training rows need q_offset == 0")
    return {"dq": dq, "dk": dk, "dv": dv, "gsum": gsum, "gsum_cur": gcur, "ds": ds}


def decode(desc: Desc, q, k_cache, v_cache, scores=None):
    """One decode step at position N-1 = desc.q_offset (desc.seq_len == 1).

    q [B,Hq,d]; k_cache/v_cache [B,Hkv,S,d] with S >= N; scores [B,Hkv,1,NB]
    or None for dense attention over all N tokens. Returns o [B,Hq,d] f64."""
    q, kc, vc = _f32(q), _f32(k_cache), _f32(v_cache)
    stride = kc.shape[2]
    sp = None
    if scores is not None:
        s = _f32(scores)
        assert s.size == desc.batch * desc.n_kv_heads * desc.n_blocks
        sp = _ptr(s)
    o = np.empty((desc.batch, desc.n_q_heads, desc.head_dim), np.float64)
    d = desc.c()
    rc = _load().sas_oracle_decode(ctypes.byref(d), _ptr(q), _ptr(kc), _ptr(vc), stride, sp, _ptr(o))
    if rc != 0:
        raise ValueError("oracle decode needs seq_len == 1")
    return o


def gather_pages(pages, block_table, seq_len: int, block_size: int):
    """Contiguous cache [Hkv, N, d] of one sequence from page pools
    [P, Hkv, block, d]: block j of the sequence is page block_table[j]
    (study note 3-7 inference path, step 3: blocks read from a paged cache)."""
    nb = -(-seq_len // block_size)
    blocks = [pages[int(block_table[j])] for j in range(nb)]        # each [Hkv, block, d]
    return np.concatenate(blocks, axis=1)[:, :seq_len]


def topk_varlen(desc: Desc, scores, seq_lens):
    """Decode-row top-K (desc.seq_len == 1) with a cache length per sequence:
    row (i, g) is the row of position seq_lens[i] - 1, with its own candidates.
    scores [B, Hkv, 1, NB]. Returns (idx [B*Hkv, K], gate_logit, score_lse, n_sel)."""
    s = _f32(scores)
    out = []
    for i, n in enumerate(seq_lens):
        d = Desc(batch=1, seq_len=1, q_offset=int(n) - 1, n_q_heads=desc.group, n_kv_heads=1,
                 head_dim=desc.head_dim, block_size=desc.block_size, top_k=desc.top_k, gate=desc.gate)
        for g in range(desc.n_kv_heads):
            row = s[i, g, 0, :d.n_blocks].reshape(1, 1, 1, -1)
            out.append(topk(d, row))
    return tuple(np.concatenate([o[k] for o in out]) for k in range(4))


def decode_paged(desc: Desc, q, k_pages, v_pages, block_table, seq_lens, scores=None):
    """Decode over paged K/V with a cache length per sequence: for each
    sequence i, the pages of its blocks are gathered into a contiguous cache of
    N_i = seq_lens[i] tokens and the plain decode runs at position N_i - 1 (its
    own current block and candidates). k_pages/v_pages [P, Hkv, block, d],
    block_table [B, max_blocks], scores [B, Hkv, 1, NB] or None (dense).
    Returns o [B, Hq, d] f64."""
    q = _f32(q)
    o = np.empty((desc.batch, desc.n_q_heads, desc.head_dim), np.float64)
    for i, n in enumerate(seq_lens):
        n = int(n)
        kc = gather_pages(k_pages, block_table[i], n, desc.block_size)[None]
        vc = gather_pages(v_pages, block_table[i], n, desc.block_size)[None]
        d = Desc(batch=1, seq_len=1, q_offset=n - 1, n_q_heads=desc.n_q_heads, n_kv_heads=desc.n_kv_heads,
                 head_dim=desc.head_dim, block_size=desc.block_size, top_k=desc.top_k, gate=desc.gate)
        sc = None if scores is None else _f32(scores)[i:i + 1, :, :, :d.n_blocks]
        o[i] = decode(d, q[i:i + 1], kc, vc, sc)[0]
    return o


def pooled_scores(desc: Desc, q, kbar):
    """Block scores of the decode rows from pooled keys, the fixed scorer that
    stands in for the trained selector (study note 3-7 inference path, step 1:
    score every cached block; 5-6: this scan dominates decode at long context):
    s[b, g, 0, j] = qbar . kbar[b, g, j] for the C = floor(q_offset / block)
    historical blocks, with qbar the mean of the group's G query heads; 0 for
    j >= C. q [B, Hq, d], kbar [B, Hkv, >= C, d]. Returns [B, Hkv, 1, NB] f64."""
    q, kb = _f32(q).astype(np.float64), _f32(kbar).astype(np.float64)
    G, C = desc.group, desc.q_offset // desc.block_size
    out = np.zeros((desc.batch, desc.n_kv_heads, 1, desc.n_blocks), np.float64)
    for b in range(desc.batch):
        for g in range(desc.n_kv_heads):
            qbar = q[b, g * G:(g + 1) * G].sum(0) / G
            for j in range(C):
                out[b, g, 0, j] = float(np.dot(qbar, kb[b, g, j]))
    return out


# ------------------------------------------------- per-query-head selection ---
#
# A generalisation of the selection granularity (study note 3-1 selects per
# query group, 3-7 scores per group): every query head h keeps
# its own top-K blocks from its own score row s[b, h, t, :], and still reads
# the K/V of its KV head h // G. By definition this is the per-group problem
# with one query head per group over K/V heads repeated G times; the gradient
# of a repeated K/V head is the sum over its copies.

def per_head_desc(desc: Desc) -> Desc:
    """The per-group problem in which each query head is its own group."""
    return Desc(batch=desc.batch, seq_len=desc.seq_len, n_q_heads=desc.n_q_heads, n_kv_heads=desc.n_q_heads,
                head_dim=desc.head_dim, block_size=desc.block_size, top_k=desc.top_k, q_offset=desc.q_offset,
                scale=desc.scale, gate=desc.gate)


def _repeat_heads(x, G: int):
    return np.repeat(_f32(x), G, axis=1)


def topk_per_head(desc: Desc, scores, rows=None):
    """Top-K of every (b, query head, t) row; scores [B, Hq, T, NB]."""
    return topk(per_head_desc(desc), scores, rows)


def fwd_per_head(desc: Desc, q, k, v, scores, rows=None):
    """Forward with a selection per query head; scores [B, Hq, T, NB], rows
    over (b, query head, t). Returns (o [n,1,d], attn_lse [n,1])."""
    G = desc.group
    return fwd(per_head_desc(desc), q, _repeat_heads(k, G), _repeat_heads(v, G), scores, rows)


def bwd_per_head(desc: Desc, q, k, v, scores, dO, rows=None):
    """Backward with a selection per query head. dk/dv [B,Hkv,T,d] sum the
    contributions of the G query heads of each KV head; gsum/ds per
    (b, query head, t) row."""
    G = desc.group
    r = bwd(per_head_desc(desc), q, _repeat_heads(k, G), _repeat_heads(v, G), scores, dO, rows)
    B, T, dh = desc.batch, desc.seq_len, desc.head_dim
    r["dk"] = r["dk"].reshape(B, desc.n_kv_heads, G, T, dh).sum(2)
    r["dv"] = r["dv"].reshape(B, desc.n_kv_heads, G, T, dh).sum(2)
    return r


def decode_per_head(desc: Desc, q, k_cache, v_cache, scores=None):
    """Decode with a selection per query head; scores [B, Hq, 1, NB]."""
    G = desc.group
    return decode(per_head_desc(desc), q, _repeat_heads(k_cache, G), _repeat_heads(v_cache, G), scores)
