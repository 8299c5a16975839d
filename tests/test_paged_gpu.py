"""GPU parity of the paged decode with a cache length per sequence
(sas_block_topk_varlen + sas_sparse_decode_paged) against the oracle.

The pools hold one block of every KV head per page; the block table places a
sequence's blocks in shuffled pages (plus pages no sequence uses). Indices of
the per-sequence top-K are compared bit-exactly, outputs within the bf16
tolerance. The small case covers the edge lengths (one token, exactly one
block, a partial current block); the large one is the 524288-token workload at
batch 8 with a different length per sequence, checked on sampled groups."""
import numpy as np
import pytest
import torch

import oracle
from tests import gpu_util as U
from trainable_block_sparse_topk_b200 import api, binding as B, synth
from trainable_block_sparse_topk_b200.build import build

pytestmark = pytest.mark.gpu

TOL_BF16_O = 1e-2


def paginate(kc, vc, bs, spare, gen):
    """Scatter contiguous caches [B, Hkv, N, d] into page pools [P, Hkv, bs, d]
    through a shuffled table; `spare` pages belong to no sequence."""
    Bn, H, N, d = kc.shape
    nb = -(-N // bs)
    P = Bn * nb + spare
    perm = torch.randperm(P, generator=gen)[: Bn * nb].to(torch.int32)
    table = perm.view(Bn, nb).contiguous()
    kp = torch.zeros(P, H, bs, d, dtype=kc.dtype, device=kc.device)
    vp = torch.zeros_like(kp)
    pad = nb * bs - N
    for b in range(Bn):
        kb = torch.nn.functional.pad(kc[b], (0, 0, 0, pad)).view(H, nb, bs, d).transpose(0, 1)
        vb = torch.nn.functional.pad(vc[b], (0, 0, 0, pad)).view(H, nb, bs, d).transpose(0, 1)
        idx = table[b].long().to(kc.device)
        kp[idx] = kb
        vp[idx] = vb
    return kp, vp, table


def run_paged(d, q, kp, vp, table, lens, s, dense=False):
    tab, ln = table.cuda(), torch.tensor(lens, dtype=torch.int32).cuda()
    sel = None if dense else api.block_topk_varlen(d, s.cuda(), ln)
    o = api.sparse_decode_paged(d, q.cuda(), kp, vp, tab, ln, sel)
    torch.cuda.synchronize()
    return sel, o.float().cpu().numpy()


def test_paged_varlen_small_elementwise():
    build()
    oracle.build()
    gen = torch.Generator().manual_seed(41)
    Bn, Hq, Hkv, N, bs, K = 4, 32, 8, 20000, 64, 31
    lens = [20000, 13377, 64, 1]
    kc = (0.5 * torch.randn(Bn, Hkv, N, 128, generator=gen)).to(torch.bfloat16)
    vc = (0.5 * torch.randn(Bn, Hkv, N, 128, generator=gen)).to(torch.bfloat16)
    q = (0.5 * torch.randn(Bn, Hq, 128, generator=gen)).to(torch.bfloat16)
    s = torch.randn(Bn, Hkv, 1, -(-N // bs), generator=gen)
    kp, vp, table = paginate(kc.cuda(), vc.cuda(), bs, spare=37, gen=gen)
    d = B.make_desc(batch=Bn, seq_len=1, q_offset=N - 1, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=128,
                    block_size=bs, top_k=K)
    od = oracle.Desc(batch=Bn, seq_len=1, q_offset=N - 1, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=128,
                     block_size=bs, top_k=K)
    sel, got = run_paged(d, q, kp, vp, table, lens, s)
    ridx, _, _, rn = oracle.topk_varlen(od, s.numpy(), lens)
    np.testing.assert_array_equal(sel.idx.cpu().numpy().reshape(ridx.shape), ridx)
    np.testing.assert_array_equal(sel.n_sel.cpu().numpy().reshape(rn.shape), rn)
    kpn, vpn = kp.float().cpu().numpy(), vp.float().cpu().numpy()
    ref = oracle.decode_paged(od, q.float().numpy(), kpn, vpn, table.numpy(), lens, s.numpy())
    assert np.abs(got - ref).max() <= TOL_BF16_O
    _, gotd = run_paged(d, q, kp, vp, table, lens, s, dense=True)
    refd = oracle.decode_paged(od, q.float().numpy(), kpn, vpn, table.numpy(), lens, None)
    assert np.abs(gotd - refd).max() <= TOL_BF16_O


def test_paged_varlen_long_batch8():
    """524288-token workload, batch 8, N_b = 524288 - 4097 b, shuffled pages."""
    build()
    oracle.build()
    w = synth.workload("long", batch=8)
    kc, vc = U.build_decode_cache(w)
    gen = torch.Generator().manual_seed(43)
    kp, vp, table = paginate(kc, vc, w.block_size, spare=11, gen=gen)
    del kc, vc
    torch.cuda.empty_cache()
    lens = [w.seq - 4097 * b for b in range(w.batch)]
    q = synth.decode_q(w)
    s = synth.decode_scores(w, q)
    d = U.decode_desc(w, w.seq)
    sel, got = run_paged(d, q.to(torch.bfloat16), kp, vp, table, lens, s)
    G = w.group
    for b, g in [(0, 0), (3, 5), (7, 7), (5, 2)]:
        n = lens[b]
        odg = oracle.Desc(batch=1, seq_len=1, q_offset=n - 1, n_q_heads=G, n_kv_heads=1, head_dim=w.head_dim,
                          block_size=w.block_size, top_k=w.top_k)
        sg = s[b:b + 1, g:g + 1, :, :odg.n_blocks].numpy()
        ridx, _, _, _ = oracle.topk(odg, sg)
        np.testing.assert_array_equal(sel.idx[b, g, 0].cpu().numpy(), ridx[0])
        kk = synth.decode_cache_slice(w, "k", b, g)[:n].numpy()[None, None]
        vv = synth.decode_cache_slice(w, "v", b, g)[:n].numpy()[None, None]
        ref = oracle.decode(odg, q[b:b + 1, g * G:(g + 1) * G].numpy(), kk, vv, sg)
        assert np.abs(got[b, g * G:(g + 1) * G] - ref[0]).max() <= TOL_BF16_O, (b, g)
    del kp, vp
    torch.cuda.empty_cache()
