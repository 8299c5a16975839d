"""Seeded synthetic inputs for the SAS hot path.

This module is shared by the test suite, the benchmark and the oracle-side
checks. It only draws random tensors and the selector-score stand-in; it holds
none of the attention method's arithmetic and imports nothing else from this
package.

Every tensor is drawn on the CPU in float32 from a torch.Generator seeded by
(config seed, tensor name, batch, head), rounded to the config's dtype, and
returned as float32 (bf16 values are exact in float32) so that the device copy
and the oracle see identical values. Drawing per (batch, head) slice lets a
test regenerate one slice of a large cache without drawing the rest.

Workloads (shapes of the paper's Qwen3 layers, block 64; a tiny fp32 case):
  tiny    B1 T512 b32 Hq2/Hkv1 d64 K4, fp32; q,k,v,dO,s ~ N(0,1)
  qwen4b  B1 T8192 b64 Hq32/Hkv8 d128 K15, bf16; q,k,v ~ 0.5 N(0,1), dO ~ N(0,1),
          s[t,j] = mean_G(q)[t] . mean_block(k)[j] + 0.1 N(0,1)
  qwen14b B2 T32768 b64 Hq40/Hkv8 d128 K31, bf16; as qwen4b plus 0.01 * j
  decode  B1 N131072 b64 Hq32/Hkv8 d128 K in {15,31,63}, bf16; cache, q ~ 0.5 N(0,1),
          s[j] = mean_G(q) . mean_block(k)[j]
  long    B in {1,8} N524288 b64 Hq32/Hkv8 d128 K31, bf16; cache, q ~ 0.5 N(0,1),
          s ~ N(0,1), +3 on a seeded 5% of the historical blocks of each row
"""
from __future__ import annotations

import hashlib
from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str            # "train" or "decode"
    batch: int
    seq: int             # T (train) or cache length N (decode)
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    block_size: int
    top_k: int
    dtype: str           # "fp32" or "bf16"
    seed: int
    qkv_std: float
    score_noise: float = 0.0      # std of the noise added to pooled-key scores
    recency: float = 0.0          # + recency * block index
    boost_frac: float = 0.0       # "long" decode: fraction of boosted blocks
    boost: float = 0.0
    score_kind: str = "pooled"    # "pooled" (q-bar . k-bar) or "gauss"

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def n_blocks(self) -> int:
        return -(-self.seq // self.block_size)

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "fp32" else torch.bfloat16


WORKLOADS = {
    "tiny": Workload("tiny", "train", 1, 512, 2, 1, 64, 32, 4, "fp32", 0, 1.0,
                     score_kind="gauss"),
    "qwen4b": Workload("qwen4b", "train", 1, 8192, 32, 8, 128, 64, 15, "bf16", 1, 0.5,
                       score_noise=0.1),
    "qwen14b": Workload("qwen14b", "train", 2, 32768, 40, 8, 128, 64, 31, "bf16", 2, 0.5,
                        score_noise=0.1, recency=0.01),
    "decode": Workload("decode", "decode", 1, 131072, 32, 8, 128, 64, 31, "bf16", 3, 0.5),
    "long": Workload("long", "decode", 1, 524288, 32, 8, 128, 64, 31, "bf16", 4, 0.5,
                     score_kind="gauss", boost_frac=0.05, boost=3.0),
}


def workload(name: str, **over) -> Workload:
    w = WORKLOADS[name]
    return replace(w, **over) if over else w


def _gen(seed: int, *tag) -> torch.Generator:
    h = hashlib.sha256(repr((seed,) + tag).encode()).digest()
    g = torch.Generator(device="cpu")
    g.manual_seed(int.from_bytes(h[:8], "little") & ((1 << 63) - 1))
    return g


def _round(x: torch.Tensor, w: Workload) -> torch.Tensor:
    """Round to the workload dtype and return float32 holding the exact values."""
    if w.dtype == "bf16":
        return x.to(torch.bfloat16).to(torch.float32)
    return x


def head_slice(w: Workload, name: str, b: int, h: int, rows: int, std: float) -> torch.Tensor:
    """One [rows, d] slice of tensor `name` for batch b, head h (float32)."""
    g = _gen(w.seed, name, b, h)
    x = torch.randn(rows, w.head_dim, generator=g, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return _round(x, w)


# ------------------------------------------------------------------ training ---

def train_qkv(w: Workload, which: str) -> torch.Tensor:
    """q [B,Hq,T,d], k or v [B,Hkv,T,d], dO [B,Hq,T,d] (float32 holding dtype values)."""
    heads = w.n_kv_heads if which in ("k", "v") else w.n_q_heads
    std = 1.0 if which == "dO" else w.qkv_std
    out = torch.empty(w.batch, heads, w.seq, w.head_dim, dtype=torch.float32)
    for b in range(w.batch):
        for h in range(heads):
            out[b, h] = head_slice(w, which, b, h, w.seq, std)
    return out


def pooled_scores(w: Workload, qbar: torch.Tensor, kbar: torch.Tensor, b: int, g: int) -> torch.Tensor:
    """Selector stand-in: s[t, j] = qbar[t] . kbar[j] (+ noise, + recency * j)."""
    s = qbar @ kbar.T
    if w.score_noise:
        s.add_(torch.randn(s.shape, generator=_gen(w.seed, "s_noise", b, g)) * w.score_noise)
    if w.recency:
        s.add_(w.recency * torch.arange(s.shape[1], dtype=torch.float32))
    return s


def train_scores(w: Workload, q: torch.Tensor | None = None, k: torch.Tensor | None = None) -> torch.Tensor:
    """Per-query block scores [B, Hkv, T, NB] float32."""
    NB = w.n_blocks
    out = torch.empty(w.batch, w.n_kv_heads, w.seq, NB, dtype=torch.float32)
    G = w.group
    for b in range(w.batch):
        for g in range(w.n_kv_heads):
            if w.score_kind == "gauss":
                out[b, g] = torch.randn(w.seq, NB, generator=_gen(w.seed, "s", b, g))
                continue
            qg = q[b, g * G:(g + 1) * G] if q is not None else torch.stack(
                [head_slice(w, "q", b, g * G + r, w.seq, w.qkv_std) for r in range(G)])
            kg = k[b, g] if k is not None else head_slice(w, "k", b, g, w.seq, w.qkv_std)
            qbar = qg.mean(0)
            kbar = kg.reshape(NB, w.block_size, w.head_dim).mean(1)
            out[b, g] = pooled_scores(w, qbar, kbar, b, g)
    return out


def train_inputs(w: Workload) -> dict:
    """All inputs of one training step (CPU float32 tensors)."""
    q = train_qkv(w, "q")
    k = train_qkv(w, "k")
    v = train_qkv(w, "v")
    dO = train_qkv(w, "dO")
    s = train_scores(w, q, k)
    return {"q": q, "k": k, "v": v, "dO": dO, "scores": s}


# -------------------------------------------------------------------- decode ---

def decode_q(w: Workload) -> torch.Tensor:
    """The new token's queries [B, Hq, d]."""
    out = torch.empty(w.batch, w.n_q_heads, w.head_dim)
    for b in range(w.batch):
        for h in range(w.n_q_heads):
            out[b, h] = head_slice(w, "dq_q", b, h, 1, w.qkv_std)[0]
    return out


def decode_cache_slice(w: Workload, which: str, b: int, g: int) -> torch.Tensor:
    """One [N, d] slice of the K or V cache (float32 holding dtype values)."""
    return head_slice(w, "cache_" + which, b, g, w.seq, w.qkv_std)


def decode_scores(w: Workload, q: torch.Tensor) -> torch.Tensor:
    """Block scores [B, Hkv, 1, NB] of the new token at position N-1."""
    NB = w.n_blocks
    C = (w.seq - 1) // w.block_size
    G = w.group
    out = torch.zeros(w.batch, w.n_kv_heads, 1, NB)
    for b in range(w.batch):
        for g in range(w.n_kv_heads):
            if w.score_kind == "gauss":
                s = torch.randn(NB, generator=_gen(w.seed, "ds", b, g))
                if w.boost_frac:
                    gb = _gen(w.seed, "boost", b, g)
                    nb = int(round(w.boost_frac * C))
                    sel = torch.randperm(C, generator=gb)[:nb]
                    s[sel] += w.boost
                out[b, g, 0] = s
            else:
                kc = decode_cache_slice(w, "k", b, g)
                kbar = kc[: NB * w.block_size].reshape(NB, w.block_size, w.head_dim).mean(1)
                qbar = q[b, g * G:(g + 1) * G].mean(0)
                out[b, g, 0] = kbar @ qbar
    return out
