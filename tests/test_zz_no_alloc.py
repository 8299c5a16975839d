"""The allocation-free decode entry point against the regular one.

sas_sparse_decode_noalloc serves callers that cannot call cudaMalloc (a fixed
device-memory budget set aside at start-up, a host framework that owns every
device allocation, a path where allocating is not allowed). It keeps the split
partials in a static device array inside libsas instead of a caller workspace.
This file runs last (pytest collects it after the others), passes alone in a
fresh process as well as after the rest of the suite, and checks, through the
C ABI, two calls in a row against sas_sparse_decode within the bf16 output
tolerance of the other parity tests.
"""
import pytest
import torch

from trainable_block_sparse_topk_b200 import api, binding as B, synth
from trainable_block_sparse_topk_b200.build import build

pytestmark = pytest.mark.gpu

TOL_BF16_O = 1e-2


def _cache(w):
    dt = torch.bfloat16
    kc = torch.empty(w.batch, w.n_kv_heads, w.seq, w.head_dim, dtype=dt, device="cuda")
    vc = torch.empty_like(kc)
    for b in range(w.batch):
        for g in range(w.n_kv_heads):
            kc[b, g].copy_(synth.decode_cache_slice(w, "k", b, g).to(dt))
            vc[b, g].copy_(synth.decode_cache_slice(w, "v", b, g).to(dt))
    return kc, vc


def _desc(w, K):
    return B.make_desc(batch=w.batch, seq_len=1, q_offset=w.seq - 1, n_q_heads=w.n_q_heads,
                       n_kv_heads=w.n_kv_heads, head_dim=w.head_dim, block_size=w.block_size, top_k=K)


def test_noalloc_matches_workspace_decode_twice():
    build()
    w = synth.workload("decode", seq=16384 + 37)
    kc, vc = _cache(w)
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


def test_noalloc_rejects_oversize():
    """16 x 8 KV heads x 33 splits (two kept blocks per split) x 4 heads x 130
    floats needs more than the static array: refused before any launch, with
    the workspace status."""
    build()
    w = synth.workload("decode", batch=16, seq=64 * 66)
    d = _desc(w, 64)
    kc = torch.zeros(w.batch, w.n_kv_heads, w.seq, w.head_dim, dtype=torch.bfloat16, device="cuda")
    q = torch.zeros(w.batch, w.n_q_heads, w.head_dim, dtype=torch.bfloat16, device="cuda")
    sel = api.block_topk(d, torch.zeros(w.batch, w.n_kv_heads, 1, d.n_blocks, device="cuda"))
    with pytest.raises(B.SasError) as ei:
        B.sas_sparse_decode_noalloc(d, q, kc, kc, w.seq, sel.idx, sel.gate_logit, sel.n_sel, torch.empty_like(q))
    assert ei.value.status == B.SAS_ERR_WORKSPACE
