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
