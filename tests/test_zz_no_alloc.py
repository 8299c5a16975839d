"""The allocation-free decode entry point against the regular one.

sas_sparse_decode_noalloc serves callers that cannot call cudaMalloc (a fixed
device-memory budget set aside at start-up, a host framework that owns every
device allocation, a path where allocating is not allowed). It keeps the split
partials in a static device array inside libsas instead of a caller workspace.
This file runs last (pytest collects it after the others), passes alone in a
fresh process as well as after the rest of the suite, and checks, through the
C ABI, two calls in a row against sas_sparse_decode and against the oracle,
within the bf16 output tolerance of the other parity tests.
"""
import numpy as np
import pytest
import torch

import oracle
from trainable_block_sparse_topk_b200 import api, binding as B, synth
from trainable_block_sparse_topk_b200.build import build

pytestmark = pytest.mark.gpu

TOL_BF16_O = 1e-2


def _cache(w):
    """The K and V caches on the host (float32 holding bf16 values)."""
    kc = torch.empty(w.batch, w.n_kv_heads, w.seq, w.head_dim)
    vc = torch.empty_like(kc)
    for b in range(w.batch):
        for g in range(w.n_kv_heads):
            kc[b, g] = synth.decode_cache_slice(w, "k", b, g)
            vc[b, g] = synth.decode_cache_slice(w, "v", b, g)
    return kc, vc


def _desc(w, K):
    return B.make_desc(batch=w.batch, seq_len=1, q_offset=w.seq - 1, n_q_heads=w.n_q_heads,
                       n_kv_heads=w.n_kv_heads, head_dim=w.head_dim, block_size=w.block_size, top_k=K)


def test_noalloc_matches_workspace_decode_twice():
    build()
    oracle.build()
    w = synth.workload("decode", seq=16384 + 37)
    hk, hv = _cache(w)
    kc, vc = hk.to(torch.bfloat16).cuda(), hv.to(torch.bfloat16).cuda()
    gen = torch.Generator().manual_seed(123)
    calls = [(31, False), (15, True)]          # sparse K=31, then dense decode with another query
    for K, dense in calls:
        d = _desc(w, K)
        q = (0.5 * torch.randn(w.batch, w.n_q_heads, w.head_dim, generator=gen)).to(torch.bfloat16).cuda()
        s = torch.randn(w.batch, w.n_kv_heads, 1, d.n_blocks, generator=gen).cuda()
        sel = None if dense else api.block_topk(d, s)
        ref = api.sparse_decode(d, q, kc, vc, sel)
        out = torch.full_like(q, float("nan"))
        if dense:
            B.sas_sparse_decode_noalloc(d, q, kc, vc, w.seq, None, None, None, out)
        else:
            B.sas_sparse_decode_noalloc(d, q, kc, vc, w.seq, sel.idx, sel.gate_logit, sel.n_sel, out)
        torch.cuda.synchronize()
        err = (out.float() - ref.float()).abs().max().item()
        assert err <= TOL_BF16_O, (K, dense, err)
        od = oracle.Desc(batch=w.batch, seq_len=1, q_offset=w.seq - 1, n_q_heads=w.n_q_heads,
                         n_kv_heads=w.n_kv_heads, head_dim=w.head_dim, block_size=w.block_size, top_k=K)
        oref = oracle.decode(od, q.float().cpu().numpy(), hk.numpy(), hv.numpy(),
                             None if dense else s.cpu().numpy())
        err_o = float(np.abs(out.float().cpu().numpy() - oref).max())
        assert err_o <= TOL_BF16_O, (K, dense, err_o)


def test_noalloc_rejects_oversize():
    """A shape whose decode workspace (sas_workspace_size) exceeds the static
    array is refused before any launch, with the workspace status."""
    build()
    w = synth.workload("decode", batch=16, seq=64 * 66)
    d = _desc(w, 64)
    assert B.sas_workspace_size(B.SAS_OP_DECODE, d) > 8 << 20
    kc = torch.zeros(w.batch, w.n_kv_heads, w.seq, w.head_dim, dtype=torch.bfloat16, device="cuda")
    q = torch.zeros(w.batch, w.n_q_heads, w.head_dim, dtype=torch.bfloat16, device="cuda")
    sel = api.block_topk(d, torch.zeros(w.batch, w.n_kv_heads, 1, d.n_blocks, device="cuda"))
    with pytest.raises(B.SasError) as ei:
        B.sas_sparse_decode_noalloc(d, q, kc, kc, w.seq, sel.idx, sel.gate_logit, sel.n_sel, torch.empty_like(q))
    assert ei.value.status == B.SAS_ERR_WORKSPACE
