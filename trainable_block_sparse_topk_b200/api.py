"""Convenience layer over the C ABI: allocates outputs and workspaces with torch
and calls the binding. Every computation is a libsas kernel.

    desc = make_desc(B, T, Hq, Hkv, d, block, K, dtype="bf16")
    sel = block_topk(desc, scores)                   # idx, gate_logit, score_lse, n_sel
    o, lse = gated_attn_fwd(desc, q, k, v, sel)
    dq, dk, dv, ds = gated_attn_bwd(desc, q, k, v, o, lse, dO, scores, sel)
    o = sparse_decode(ddesc, q1, k_cache, v_cache, sel1)   # sel1=None: dense

`SASAttention` wraps top-K + forward + backward as a torch.autograd.Function
whose gradients flow to q, k, v and to the block scores.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import binding as B


@dataclass
class Selection:
    idx: torch.Tensor         # [B, Hkv, T, K] int32
    gate_logit: torch.Tensor  # [B, Hkv, T, K] float32
    score_lse: torch.Tensor   # [B, Hkv, T] float32
    n_sel: torch.Tensor       # [B, Hkv, T] int32


def workspace(op: int, desc, device=None) -> torch.Tensor | None:
    n = B.sas_workspace_size(op, desc)
    if n == 0:
        return None
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def block_topk(desc, scores: torch.Tensor, out: Selection | None = None, stream=None) -> Selection:
    Bn, H, T, K = desc.batch, desc.n_sel_groups, desc.seq_len, desc.top_k
    dev = scores.device
    if out is None:
        out = Selection(torch.empty(Bn, H, T, K, dtype=torch.int32, device=dev),
                        torch.empty(Bn, H, T, K, dtype=torch.float32, device=dev),
                        torch.empty(Bn, H, T, dtype=torch.float32, device=dev),
                        torch.empty(Bn, H, T, dtype=torch.int32, device=dev))
    B.sas_block_topk(desc, scores, out.idx, out.gate_logit, out.score_lse, out.n_sel, stream)
    return out


def gated_attn_fwd(desc, q, k, v, sel: Selection, ws=None, stream=None):
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:-1], dtype=torch.float32, device=q.device)
    if ws is None:
        ws = workspace(B.SAS_OP_FWD, desc, q.device)
    B.sas_gated_attn_fwd(desc, q, k, v, sel.idx, sel.gate_logit, sel.n_sel, o, lse, ws, stream)
    return o, lse


def gated_attn_bwd(desc, q, k, v, o, lse, dO, scores, sel: Selection, ws=None, stream=None):
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ds = torch.empty_like(scores)
    if ws is None:
        ws = workspace(B.SAS_OP_BWD, desc, q.device)
    B.sas_gated_attn_bwd(desc, q, k, v, o, dO, lse, scores, sel.score_lse, sel.idx, sel.gate_logit, sel.n_sel,
                         dq, dk, dv, ds, ws, stream)
    return dq, dk, dv, ds


def sparse_decode(desc, q, k_cache, v_cache, sel: Selection | None, ws=None, stream=None):
    o = torch.empty_like(q)
    if ws is None:
        ws = workspace(B.SAS_OP_DECODE, desc, q.device)
    if sel is None:
        B.sas_sparse_decode(desc, q, k_cache, v_cache, k_cache.shape[2], None, None, None, o, ws, stream)
    else:
        B.sas_sparse_decode(desc, q, k_cache, v_cache, k_cache.shape[2], sel.idx, sel.gate_logit, sel.n_sel,
                            o, ws, stream)
    return o


def block_topk_varlen(desc, scores: torch.Tensor, seq_lens: torch.Tensor, stream=None) -> Selection:
    """Decode-row top-K with a cache length per sequence (seq_lens int32 [B])."""
    Bn, H, K = desc.batch, desc.n_sel_groups, desc.top_k
    dev = scores.device
    out = Selection(torch.empty(Bn, H, 1, K, dtype=torch.int32, device=dev),
                    torch.empty(Bn, H, 1, K, dtype=torch.float32, device=dev),
                    torch.empty(Bn, H, 1, dtype=torch.float32, device=dev),
                    torch.empty(Bn, H, 1, dtype=torch.int32, device=dev))
    B.sas_block_topk_varlen(desc, scores, seq_lens, out.idx, out.gate_logit, out.score_lse, out.n_sel, stream)
    return out


def sparse_decode_paged(desc, q, k_pages, v_pages, block_table, seq_lens, sel: Selection | None, ws=None,
                        stream=None):
    """Decode over page pools [num_pages, Hkv, block, d]; sel=None: dense."""
    o = torch.empty_like(q)
    if ws is None:
        ws = workspace(B.SAS_OP_DECODE, desc, q.device)
    if sel is None:
        B.sas_sparse_decode_paged(desc, q, k_pages, v_pages, block_table, seq_lens, None, None, None, o, ws, stream)
    else:
        B.sas_sparse_decode_paged(desc, q, k_pages, v_pages, block_table, seq_lens, sel.idx, sel.gate_logit,
                                  sel.n_sel, o, ws, stream)
    return o


def sparse_decode_pooled(desc, q, k_cache, v_cache, kbar, ws=None, stream=None):
    """Pooled-key block scores, top-K and sparse decode in one call; returns
    (o, scores, Selection)."""
    Bn, H, K = desc.batch, desc.n_sel_groups, desc.top_k
    dev = q.device
    scores = torch.empty(Bn, H, 1, desc.n_blocks, dtype=torch.float32, device=dev)
    sel = Selection(torch.empty(Bn, H, 1, K, dtype=torch.int32, device=dev),
                    torch.empty(Bn, H, 1, K, dtype=torch.float32, device=dev),
                    torch.empty(Bn, H, 1, dtype=torch.float32, device=dev),
                    torch.empty(Bn, H, 1, dtype=torch.int32, device=dev))
    o = torch.empty_like(q)
    if ws is None:
        ws = workspace(B.SAS_OP_DECODE, desc, dev)
    B.sas_sparse_decode_pooled(desc, q, k_cache, v_cache, k_cache.shape[2], kbar, scores, sel.idx, sel.gate_logit,
                               sel.score_lse, sel.n_sel, o, ws, stream)
    return o, scores, sel


class SASAttention(torch.autograd.Function):
    """o = SAS gated block-sparse attention(q, k, v; scores). Differentiable in
    q, k, v and scores (the score gradient flows through the softmax gate)."""

    @staticmethod
    def forward(ctx, q, k, v, scores, desc):
        sel = block_topk(desc, scores)
        o, lse = gated_attn_fwd(desc, q, k, v, sel)
        ctx.desc = desc
        ctx.save_for_backward(q, k, v, scores, o, lse, sel.idx, sel.gate_logit, sel.score_lse, sel.n_sel)
        return o

    @staticmethod
    def backward(ctx, dO):
        q, k, v, scores, o, lse, idx, gl, slse, nsel = ctx.saved_tensors
        sel = Selection(idx, gl, slse, nsel)
        dq, dk, dv, ds = gated_attn_bwd(ctx.desc, q, k, v, o, lse, dO.contiguous(), scores, sel)
        return dq, dk, dv, ds, None
