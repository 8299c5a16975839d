"""Per-query-head selection (desc.select_heads = 1): every query head keeps its
own top-K from its own score row and reads its KV head's K/V; the K/V
gradients sum over the heads that share them. GPU results against the
oracle's per-head composition (oracle.fwd_per_head / bwd_per_head /
decode_per_head), on the CUDA-core fp32 path (every output elementwise), the
bf16 tensor-core paths (sampled rows, whole key blocks) and decode."""
import numpy as np
import pytest
import torch

import oracle
from tests import gpu_util as U
from trainable_block_sparse_topk_b200 import api, binding as B, synth

pytestmark = pytest.mark.gpu

TOL_FP32 = 1e-4
TOL_BF16_O = 1e-2
TOL_BF16_GRAD = 2e-2


def head_scores(w, seed):
    """Seeded per-head block scores [B, Hq, T, NB]: the workload's own group
    scores plus per-head noise, so the heads of a group select differently."""
    x = synth.train_inputs(w)
    g = torch.Generator().manual_seed(seed)
    s = x["scores"].repeat_interleave(w.group, 1)
    s = s + 0.5 * torch.randn(s.shape, generator=g)
    return x, s.contiguous()


def run(w, x, s, gate="softmax"):
    d = U.train_desc(w, gate=gate, select_heads=True)
    dt = U.dev_dtype(w)
    g = {n: x[n].to(dt).cuda() for n in ("q", "k", "v", "dO")}
    sc = s.cuda()
    sel = api.block_topk(d, sc)
    o, lse = api.gated_attn_fwd(d, g["q"], g["k"], g["v"], sel)
    dq, dk, dv, ds = api.gated_attn_bwd(d, g["q"], g["k"], g["v"], o, lse, g["dO"], sc, sel)
    torch.cuda.synchronize()
    out = dict(idx=sel.idx, nsel=sel.n_sel, o=o, lse=lse, dq=dq, dk=dk, dv=dv, ds=ds)
    return {k: v.cpu() for k, v in out.items()}


def odesc(w, gate=oracle.GATE_SOFTMAX):
    return oracle.Desc(batch=w.batch, seq_len=w.seq, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads,
                       head_dim=w.head_dim, block_size=w.block_size, top_k=w.top_k, gate=gate)


@pytest.mark.parametrize("gate", ["softmax", "none"])
def test_per_head_tiny_fp32_full(gate):
    """The tiny fp32 workload (Hq2/Hkv1): every output elementwise at 1e-4."""
    w = synth.workload("tiny")
    x, s = head_scores(w, 7)
    out = run(w, x, s, gate)
    d = odesc(w, oracle.GATE_SOFTMAX if gate == "softmax" else oracle.GATE_NONE)
    B_, Hq, T, dh = w.batch, w.n_q_heads, w.seq, w.head_dim
    idx, _, _, nsel = oracle.topk_per_head(d, s.numpy())
    assert np.array_equal(out["idx"].numpy().reshape(idx.shape), idx)
    assert np.array_equal(out["nsel"].numpy().reshape(-1), nsel)
    o, lse = oracle.fwd_per_head(d, x["q"].numpy(), x["k"].numpy(), x["v"].numpy(), s.numpy())
    np.testing.assert_allclose(out["o"].numpy(), o.reshape(B_, Hq, T, dh), atol=TOL_FP32, rtol=0)
    np.testing.assert_allclose(out["lse"].numpy(), lse.reshape(B_, Hq, T), atol=TOL_FP32, rtol=0)
    r = oracle.bwd_per_head(d, x["q"].numpy(), x["k"].numpy(), x["v"].numpy(), s.numpy(), x["dO"].numpy())
    np.testing.assert_allclose(out["dq"].numpy(), r["dq"].reshape(B_, Hq, T, dh), atol=TOL_FP32, rtol=0)
    np.testing.assert_allclose(out["dk"].numpy(), r["dk"], atol=TOL_FP32, rtol=0)
    np.testing.assert_allclose(out["dv"].numpy(), r["dv"], atol=TOL_FP32, rtol=0)
    np.testing.assert_allclose(out["ds"].numpy(), r["ds"].reshape(s.shape), atol=TOL_FP32, rtol=0)


def test_per_head_bf16_tensor_core():
    """bf16 d128 b64 with G = 5 query heads per KV head (the tensor-core forward
    and backward over one head per selection group): top-K bit-exact, o at
    1e-2, dq / ds / dk / dv at 2e-2 normwise on sampled rows and key blocks."""
    w = synth.Workload("mid", "train", 1, 1024, 10, 2, 128, 64, 5, "bf16", 21, 0.5, score_noise=0.1)
    x, s = head_scores(w, 8)
    out = run(w, x, s)
    d = odesc(w)
    T, Hq = w.seq, w.n_q_heads
    idx, _, _, nsel = oracle.topk_per_head(d, s.numpy())
    assert np.array_equal(out["idx"].numpy().reshape(idx.shape), idx)
    assert np.array_equal(out["nsel"].numpy().reshape(-1), nsel)
    rng = np.random.default_rng(3)
    heads = [0, 4, 5, Hq - 1]
    ts = sorted(set([0, 63, 64, 130, T - 1] + list(rng.integers(0, T, 12))))
    rows = np.array([h * T + t for h in heads for t in ts])          # (b = 0, query head, t)
    o, _ = oracle.fwd_per_head(d, x["q"].numpy(), x["k"].numpy(), x["v"].numpy(), s.numpy(), rows)
    got_o = np.stack([out["o"][0, h, t].float().numpy() for h in heads for t in ts])
    assert np.abs(got_o - o[:, 0]).max() <= TOL_BF16_O
    r = oracle.bwd_per_head(d, x["q"].numpy(), x["k"].numpy(), x["v"].numpy(), s.numpy(), x["dO"].numpy(), rows)
    got_dq = np.stack([out["dq"][0, h, t].float().numpy() for h in heads for t in ts])
    assert U.normwise(got_dq, r["dq"][:, 0]) <= TOL_BF16_GRAD
    got_ds = np.stack([out["ds"][0, h, t].numpy() for h in heads for t in ts])
    assert U.normwise(got_ds, r["ds"]) <= TOL_BF16_GRAD
    # whole key blocks: every row of the layer contributes, so the full oracle backward
    rf = oracle.bwd_per_head(d, x["q"].numpy(), x["k"].numpy(), x["v"].numpy(), s.numpy(), x["dO"].numpy())
    bs = w.block_size
    for g, j in ((0, 1), (1, 7), (1, T // bs - 1)):
        sl = slice(j * bs, (j + 1) * bs)
        assert U.normwise(out["dk"][0, g, sl].float().numpy(), rf["dk"][0, g, sl]) <= TOL_BF16_GRAD, (g, j)
        assert U.normwise(out["dv"][0, g, sl].float().numpy(), rf["dv"][0, g, sl]) <= TOL_BF16_GRAD, (g, j)


@pytest.mark.parametrize("batch", [1, 4])
def test_per_head_decode(batch):
    """Decode with a selection per query head (Hq8/Hkv2, 8229-token cache,
    K15): top-K bit-exact and every head's output at 1e-2."""
    N, K, Hq, Hkv = 8192 + 37, 15, 8, 2
    gen = torch.Generator().manual_seed(31 + batch)
    kc = (0.5 * torch.randn(batch, Hkv, N, 128, generator=gen)).to(torch.bfloat16)
    vc = (0.5 * torch.randn(batch, Hkv, N, 128, generator=gen)).to(torch.bfloat16)
    q = (0.5 * torch.randn(batch, Hq, 128, generator=gen)).to(torch.bfloat16)
    NB = -(-N // 64)
    s = torch.randn(batch, Hq, 1, NB, generator=gen)
    d = B.make_desc(batch=batch, seq_len=1, q_offset=N - 1, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=128,
                    block_size=64, top_k=K, select_heads=True)
    sel = api.block_topk(d, s.cuda())
    o = api.sparse_decode(d, q.cuda(), kc.cuda(), vc.cuda(), sel).float().cpu().numpy()
    od = oracle.Desc(batch=batch, seq_len=1, q_offset=N - 1, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=128,
                     block_size=64, top_k=K)
    idx, _, _, _ = oracle.topk_per_head(od, s.numpy())
    assert np.array_equal(sel.idx.cpu().numpy().reshape(idx.shape), idx)
    ref = oracle.decode_per_head(od, q.float().numpy(), kc.float().numpy(), vc.float().numpy(), s.numpy())
    assert np.abs(o - ref).max() <= TOL_BF16_O


@pytest.mark.parametrize("gate", ["sigmoid", "ste"])
def test_per_head_gate_modes_fp32(gate):
    """Per-head selection under other gate activations (fp32 path, elementwise)."""
    w = synth.workload("tiny")
    x, s = head_scores(w, 9)
    out = run(w, x, s, gate)
    d = odesc(w, {"sigmoid": oracle.GATE_SIGMOID, "ste": oracle.GATE_STE}[gate])
    B_, Hq, T, dh = w.batch, w.n_q_heads, w.seq, w.head_dim
    o, _ = oracle.fwd_per_head(d, x["q"].numpy(), x["k"].numpy(), x["v"].numpy(), s.numpy())
    np.testing.assert_allclose(out["o"].numpy(), o.reshape(B_, Hq, T, dh), atol=TOL_FP32, rtol=0)
    r = oracle.bwd_per_head(d, x["q"].numpy(), x["k"].numpy(), x["v"].numpy(), s.numpy(), x["dO"].numpy())
    np.testing.assert_allclose(out["dk"].numpy(), r["dk"], atol=TOL_FP32, rtol=0)
    np.testing.assert_allclose(out["ds"].numpy(), r["ds"].reshape(s.shape), atol=TOL_FP32, rtol=0)


def test_per_head_paged_varlen():
    """Per-head selection over paged pools with a length per sequence."""
    gen = torch.Generator().manual_seed(51)
    Bn, Hq, Hkv, N, bs, K = 2, 8, 2, 9000, 64, 15
    lens = [9000, 4097]
    G = Hq // Hkv
    kc = (0.5 * torch.randn(Bn, Hkv, N, 128, generator=gen)).to(torch.bfloat16)
    vc = (0.5 * torch.randn(Bn, Hkv, N, 128, generator=gen)).to(torch.bfloat16)
    q = (0.5 * torch.randn(Bn, Hq, 128, generator=gen)).to(torch.bfloat16)
    NB = -(-N // bs)
    s = torch.randn(Bn, Hq, 1, NB, generator=gen)
    nb = NB
    table = torch.randperm(Bn * nb + 5, generator=gen)[: Bn * nb].to(torch.int32).view(Bn, nb).contiguous()
    P = Bn * nb + 5
    kp = torch.zeros(P, Hkv, bs, 128, dtype=torch.bfloat16)
    vp = torch.zeros_like(kp)
    pad = nb * bs - N
    for b in range(Bn):
        kb = torch.nn.functional.pad(kc[b], (0, 0, 0, pad)).view(Hkv, nb, bs, 128).transpose(0, 1)
        vb = torch.nn.functional.pad(vc[b], (0, 0, 0, pad)).view(Hkv, nb, bs, 128).transpose(0, 1)
        kp[table[b].long()] = kb
        vp[table[b].long()] = vb
    d = B.make_desc(batch=Bn, seq_len=1, q_offset=N - 1, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=128,
                    block_size=bs, top_k=K, select_heads=True)
    ln = torch.tensor(lens, dtype=torch.int32).cuda()
    sel = api.block_topk_varlen(d, s.cuda(), ln)
    o = api.sparse_decode_paged(d, q.cuda(), kp.cuda(), vp.cuda(), table.cuda(), ln, sel).float().cpu().numpy()
    od = oracle.Desc(batch=Bn, seq_len=1, q_offset=N - 1, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=128,
                     block_size=bs, top_k=K)
    ph = oracle.per_head_desc(od)
    ridx, _, _, _ = oracle.topk_varlen(ph, s.numpy(), lens)
    np.testing.assert_array_equal(sel.idx.cpu().numpy().reshape(ridx.shape), ridx)
    kpr = np.repeat(kp.float().numpy(), G, axis=1)
    vpr = np.repeat(vp.float().numpy(), G, axis=1)
    ref = oracle.decode_paged(ph, q.float().numpy(), kpr, vpr, table.numpy(), lens, s.numpy())
    assert np.abs(o - ref).max() <= TOL_BF16_O
