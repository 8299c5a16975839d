"""GPU parity: every CUDA output against the oracle, on the same seeded inputs.

Tolerances (stated by the method's accuracy targets): top-K indices and counts
bit-exact; gate logits and normalisers within fp32 rounding; fp32 paths within
1e-4 absolute; bf16 outputs within 1e-2 absolute; bf16 gradients within 2e-2
normwise relative (max |diff| / max |ref| per tensor).

Small workloads are compared element by element everywhere; the full-size
workloads in the benchmark's launch configuration are compared on sampled
rows, key blocks and KV groups that the oracle computes one by one.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from tests import gpu_util as U
from trainable_block_sparse_topk_b200 import api, binding as B, synth

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
TOL_FP32 = 1e-4
TOL_BF16_O = 1e-2
TOL_BF16_GRAD = 2e-2
ORACLE_GATE = {"softmax": oracle.GATE_SOFTMAX, "none": oracle.GATE_NONE, "sigmoid": oracle.GATE_SIGMOID,
               "raw": oracle.GATE_RAW, "softmax_selected": oracle.GATE_SOFTMAX_SELECTED, "ste": oracle.GATE_STE}


@pytest.fixture(scope="module", autouse=True)
def _setup():
    from trainable_block_sparse_topk_b200.build import build
    build()
    oracle.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    yield
    assert B.sas_device_timeouts() == 0


def check_topk_rows(w, x, out, rows_by_group, top_k=None, q_offset=0, T=None):
    K = w.top_k if top_k is None else top_k
    T = w.seq if T is None else T
    for (b, g), ts in rows_by_group.items():
        d = oracle.Desc(batch=1, seq_len=T, n_q_heads=w.group, n_kv_heads=1, head_dim=w.head_dim,
                        block_size=w.block_size, top_k=K, q_offset=q_offset)
        s = x[b:b + 1, g:g + 1].numpy()
        idx, gl, lse, nsel = oracle.topk(d, s, ts)
        gi = out["idx"][b, g, ts].numpy()
        np.testing.assert_array_equal(gi, idx)
        np.testing.assert_array_equal(out["nsel"][b, g, ts].numpy(), nsel)
        glg = out["gl"][b, g, ts].numpy().astype(np.float64)
        for r in range(len(ts)):
            n = nsel[r]
            np.testing.assert_allclose(glg[r, :n], gl[r, :n], atol=2e-5, rtol=1e-6)
        sl = out["slse"][b, g, ts].numpy().astype(np.float64)
        fin = np.isfinite(lse)
        np.testing.assert_allclose(sl[fin], lse[fin], atol=2e-5, rtol=1e-6)
        assert np.all(np.isneginf(sl[~fin]))


# ------------------------------------------------------------------ top-K ---

def test_topk_golden_ties():
    with open(os.path.join(GOLDEN, "topk_ties.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        svals = [float(v) for v in c["s"]]
        C, K, bs = len(svals), c["K"], 32
        N = C * bs + 1
        s = torch.zeros(1, 1, 1, -(-N // bs))
        s[0, 0, 0, :C] = torch.tensor(svals) if C else s[0, 0, 0, :0]
        d = B.make_desc(batch=1, seq_len=1, q_offset=N - 1, n_q_heads=1, n_kv_heads=1, head_dim=64,
                        block_size=bs, top_k=K)
        sel = api.block_topk(d, s.cuda())
        assert sel.idx[0, 0, 0].cpu().tolist() == c["idx"], c["name"]
        assert int(sel.n_sel[0, 0, 0]) == min(C, K)


@pytest.mark.parametrize("ncand,K", [(31, 4), (127, 15), (500, 31), (2047, 63), (8191, 31), (8191, 64)])
def test_topk_ties_random(ncand, K):
    """Rows full of exact ties (small integers, +-0.0, -inf) at every row length
    the kernel variants cover, against the oracle's brute-force sort."""
    rng = np.random.default_rng(ncand + K)
    bs, rows = 64, 8
    N = ncand * bs + 1
    NB = -(-N // bs)
    s = rng.integers(-2, 3, size=(2, rows // 2, 1, NB)).astype(np.float32)
    s[rng.random(s.shape) < 0.1] = -np.inf
    s[rng.random(s.shape) < 0.1] = -0.0
    s[0, 0, 0, :] = 1.0                       # one all-equal row
    st = torch.from_numpy(s)
    d = B.make_desc(batch=2, seq_len=1, q_offset=N - 1, n_q_heads=rows // 2, n_kv_heads=rows // 2,
                    head_dim=64, block_size=bs, top_k=K)
    sel = api.block_topk(d, st.cuda())
    out = {"idx": sel.idx.cpu(), "gl": sel.gate_logit.cpu(), "slse": sel.score_lse.cpu(), "nsel": sel.n_sel.cpu()}
    w = synth.Workload("ties", "decode", 2, N, rows // 2, rows // 2, 64, bs, K, "fp32", 0, 1.0)
    grp = {(b, g): [0] for b in range(2) for g in range(rows // 2)}
    check_topk_rows(w, st, out, grp, top_k=K, q_offset=N - 1, T=1)


@pytest.mark.parametrize("name", ["tiny", "qwen4b", "qwen14b"])
def test_topk_train_workloads(name):
    w = synth.workload(name)
    x = synth.train_scores(w)
    d = U.train_desc(w)
    sel = api.block_topk(d, x.cuda())
    out = {"idx": sel.idx.cpu(), "gl": sel.gate_logit.cpu(), "slse": sel.score_lse.cpu(), "nsel": sel.n_sel.cpu()}
    if name == "tiny":
        grp = {(0, 0): list(range(w.seq))}
    else:
        grp = U.by_group(U.sample_rows(w, 3000, seed=11))
        # plus every row of one whole group
        grp.setdefault((w.batch - 1, w.n_kv_heads - 1), [])
        grp[(w.batch - 1, w.n_kv_heads - 1)] = list(range(w.seq))
    check_topk_rows(w, x, out, {k: sorted(set(v)) for k, v in grp.items()})


# ------------------------------------------------------------ tiny (fp32) ---

@pytest.fixture(scope="module")
def tiny_run():
    w = synth.workload("tiny")
    return (w,) + U.run_train(w)


def test_tiny_fwd_bwd_fp32_full(tiny_run):
    """Every output of the fp32 path within 1e-4 of the oracle."""
    w, x, out = tiny_run
    d = U.group_desc(w)
    a = U.group_arrays(x, w, 0, 0)
    o, lse = oracle.fwd(d, a["q"], a["k"], a["v"], a["s"])
    G = w.group
    go = out["o"][0].numpy().transpose(1, 0, 2)          # [T, G, d]
    np.testing.assert_allclose(go, o, atol=TOL_FP32, rtol=0)
    np.testing.assert_allclose(out["lse"][0].numpy().T, lse, atol=TOL_FP32, rtol=0)
    r = oracle.bwd(d, a["q"], a["k"], a["v"], a["s"], a["dO"])
    np.testing.assert_allclose(out["dq"][0].numpy().transpose(1, 0, 2), r["dq"], atol=TOL_FP32, rtol=0)
    np.testing.assert_allclose(out["dk"].numpy(), r["dk"], atol=TOL_FP32, rtol=0)
    np.testing.assert_allclose(out["dv"].numpy(), r["dv"], atol=TOL_FP32, rtol=0)
    np.testing.assert_allclose(out["ds"][0, 0].numpy(), r["ds"], atol=TOL_FP32, rtol=0)
    assert G == 2


@pytest.mark.parametrize("over", [dict(gate="none"), dict(top_k=16, gate="none"), dict(top_k=1),
                                  dict(top_k=16)])
def test_tiny_variants_fp32(over):
    """Gate off, K >= C (dense), K = 1, and K >= C with the gate, all elementwise."""
    w = synth.workload("tiny")
    gate = over.get("gate", "softmax")
    K = over.get("top_k", w.top_k)
    x, out = U.run_train(w, gate=gate, top_k=K)
    d = U.group_desc(w, gate=oracle.GATE_NONE if gate == "none" else oracle.GATE_SOFTMAX, top_k=K)
    a = U.group_arrays(x, w, 0, 0)
    o, lse = oracle.fwd(d, a["q"], a["k"], a["v"], a["s"])
    np.testing.assert_allclose(out["o"][0].numpy().transpose(1, 0, 2), o, atol=TOL_FP32, rtol=0)
    r = oracle.bwd(d, a["q"], a["k"], a["v"], a["s"], a["dO"])
    np.testing.assert_allclose(out["dq"][0].numpy().transpose(1, 0, 2), r["dq"], atol=TOL_FP32, rtol=0)
    np.testing.assert_allclose(out["dk"].numpy(), r["dk"], atol=TOL_FP32, rtol=0)
    np.testing.assert_allclose(out["dv"].numpy(), r["dv"], atol=TOL_FP32, rtol=0)
    np.testing.assert_allclose(out["ds"][0, 0].numpy(), r["ds"], atol=TOL_FP32, rtol=0)


@pytest.mark.parametrize("shape", [
    dict(batch=2, seq=256, n_q_heads=8, n_kv_heads=1, head_dim=64, block_size=32, top_k=3, dtype="bf16"),
    dict(batch=1, seq=384, n_q_heads=5, n_kv_heads=1, head_dim=128, block_size=64, top_k=2, dtype="bf16"),
    dict(batch=1, seq=320, n_q_heads=3, n_kv_heads=3, head_dim=128, block_size=32, top_k=5, dtype="fp32"),
    dict(batch=2, seq=192, n_q_heads=4, n_kv_heads=2, head_dim=64, block_size=64, top_k=1, dtype="fp32"),
    dict(batch=1, seq=448, n_q_heads=2, n_kv_heads=2, head_dim=128, block_size=64, top_k=3, dtype="bf16"),
    dict(batch=1, seq=512, n_q_heads=4, n_kv_heads=2, head_dim=128, block_size=64, top_k=4, dtype="bf16"),
])
def test_small_shapes_elementwise(shape):
    """Ragged small problems over the supported ranges (G = 1..8, d 64/128,
    block 32/64, both dtypes), every element against the oracle. The last two
    run the gathered-row forward with two Q stages (G = 1) and with three at
    the largest metadata slot that fits (G = 2)."""
    w = synth.Workload("small", "train", shape["batch"], shape["seq"], shape["n_q_heads"], shape["n_kv_heads"],
                       shape["head_dim"], shape["block_size"], shape["top_k"], shape["dtype"], 99, 0.5,
                       score_kind="gauss")
    x, out = U.run_train(w)
    bf = w.dtype == "bf16"
    for b in range(w.batch):
        for g in range(w.n_kv_heads):
            d = U.group_desc(w)
            a = U.group_arrays(x, w, b, g)
            o, _ = oracle.fwd(d, a["q"], a["k"], a["v"], a["s"])
            G = w.group
            go = out["o"][b, g * G:(g + 1) * G].float().numpy().transpose(1, 0, 2)
            np.testing.assert_allclose(go, o, atol=TOL_BF16_O if bf else TOL_FP32, rtol=0)
            r = oracle.bwd(d, a["q"], a["k"], a["v"], a["s"], a["dO"])
            gdq = out["dq"][b, g * G:(g + 1) * G].float().numpy().transpose(1, 0, 2)
            gdk = out["dk"][b:b + 1, g:g + 1].float().numpy()
            gdv = out["dv"][b:b + 1, g:g + 1].float().numpy()
            gds = out["ds"][b, g].numpy()
            if bf:
                for got, ref in ((gdq, r["dq"]), (gdk, r["dk"]), (gdv, r["dv"]), (gds, r["ds"])):
                    assert U.normwise(got, ref) <= TOL_BF16_GRAD
            else:
                for got, ref in ((gdq, r["dq"]), (gdk, r["dk"]), (gdv, r["dv"]), (gds, r["ds"])):
                    np.testing.assert_allclose(got, ref, atol=TOL_FP32, rtol=0)


# ------------------------------------------------------ full-size bf16 runs ---

@pytest.fixture(scope="module", params=["qwen4b", "qwen14b"])
def big_run(request):
    w = synth.workload(request.param)
    x, out = U.run_train(w)
    return w, x, out


def test_big_rows_fwd_dq_ds(big_run):
    """Sampled rows: o within 1e-2, dq and the score gradient within 2e-2."""
    w, x, out = big_run
    G = w.group
    rows = U.sample_rows(w, 400 if w.name == "qwen4b" else 150, seed=3)
    got_o, ref_o, got_dq, ref_dq, got_ds, ref_ds = [], [], [], [], [], []
    for (b, g), ts in U.by_group(rows).items():
        ts = np.array(sorted(set(ts)), dtype=np.int64)
        d = U.group_desc(w)
        a = U.group_arrays(x, w, b, g)
        o, _ = oracle.fwd(d, a["q"], a["k"], a["v"], a["s"], ts)
        r = U.parallel_oracle_bwd(d, a, ts)
        got_o.append(out["o"][b, g * G:(g + 1) * G][:, ts].float().numpy().transpose(1, 0, 2))
        ref_o.append(o)
        got_dq.append(out["dq"][b, g * G:(g + 1) * G][:, ts].float().numpy().transpose(1, 0, 2))
        ref_dq.append(r["dq"])
        got_ds.append(out["ds"][b, g][ts].numpy())
        ref_ds.append(r["ds"])
    go, ro = np.concatenate(got_o), np.concatenate(ref_o)
    assert np.abs(go - ro).max() <= TOL_BF16_O
    assert U.normwise(np.concatenate(got_dq), np.concatenate(ref_dq)) <= TOL_BF16_GRAD
    assert U.normwise(np.concatenate(got_ds), np.concatenate(ref_ds)) <= TOL_BF16_GRAD


def test_big_key_blocks_dk_dv(big_run):
    """Sampled key blocks: dk, dv of block j from every row that attends it."""
    w, x, out = big_run
    nT = w.seq // w.block_size
    picks = [(0, 0, 1), (w.batch - 1, w.n_kv_heads - 1, nT - 2), (0, w.n_kv_heads // 2, nT // 2)]
    if w.name == "qwen14b":
        picks[2] = (w.batch - 1, 1, nT - 40)
    bs = w.block_size
    for b, g, j in picks:
        rows = U.rows_touching_block(w, x, b, g, j, oracle.GATE_SOFTMAX)
        d = U.group_desc(w)
        a = U.group_arrays(x, w, b, g)
        r = U.parallel_oracle_bwd(d, a, rows, chunks=16)
        ref_dk = r["dk"][0, 0, j * bs:(j + 1) * bs]
        ref_dv = r["dv"][0, 0, j * bs:(j + 1) * bs]
        got_dk = out["dk"][b, g, j * bs:(j + 1) * bs].float().numpy()
        got_dv = out["dv"][b, g, j * bs:(j + 1) * bs].float().numpy()
        assert U.normwise(got_dk, ref_dk) <= TOL_BF16_GRAD, (b, g, j)
        assert U.normwise(got_dv, ref_dv) <= TOL_BF16_GRAD, (b, g, j)


def test_score_gradient_rows_of_640_columns():
    """Rows of 513-1024 block columns take the 16-byte score-gradient kernel
    with eight 128-column pieces (the layers above use four): the tiny recipe
    at T 20480, block 32 (640 columns), sampled rows' ds elementwise."""
    w = synth.workload("tiny", seq=20480)
    x, out = U.run_train(w)
    ts = np.array(sorted({t for _, _, t in U.sample_rows(w, 60, seed=7)}), dtype=np.int64)
    r = U.parallel_oracle_bwd(U.group_desc(w), U.group_arrays(x, w, 0, 0), ts)
    np.testing.assert_allclose(out["ds"][0, 0][ts].numpy(), r["ds"], atol=TOL_FP32, rtol=0)
    np.testing.assert_allclose(out["dq"][0][:, ts].numpy().transpose(1, 0, 2), r["dq"], atol=TOL_FP32, rtol=0)


# ------------------------------------------------------------------ decode ---

def decode_check(w, kc, vc, q, s, N, K, groups, dense=False, gate="softmax"):
    d = U.decode_desc(w, N, top_k=K, gate=gate)
    qd = q.to(U.dev_dtype(w)).cuda()
    sel = None if dense else api.block_topk(d, s.cuda())
    o = api.sparse_decode(d, qd, kc, vc, sel).float().cpu().numpy()
    G = w.group
    worst = 0.0
    for b, g in groups:
        od = oracle.Desc(batch=1, seq_len=1, q_offset=N - 1, n_q_heads=G, n_kv_heads=1, head_dim=w.head_dim,
                         block_size=w.block_size, top_k=K,
                         gate=ORACLE_GATE[gate])
        kk = synth.decode_cache_slice(w, "k", b, g)[:N].numpy()[None, None]
        vv = synth.decode_cache_slice(w, "v", b, g)[:N].numpy()[None, None]
        ref = oracle.decode(od, q[b:b + 1, g * G:(g + 1) * G].numpy(), kk, vv,
                            None if dense else s[b:b + 1, g:g + 1].numpy())
        worst = max(worst, float(np.abs(o[b, g * G:(g + 1) * G] - ref[0]).max()))
    assert worst <= TOL_BF16_O, worst
    return worst


@pytest.fixture(scope="module")
def decode_ws():
    w = synth.workload("decode")
    kc, vc = U.build_decode_cache(w)
    q = synth.decode_q(w)
    s = synth.decode_scores(w, q)
    yield w, kc, vc, q, s
    del kc, vc
    torch.cuda.empty_cache()


def decode_topk_check(w, s, K):
    """sas_block_topk on the decode rows (T = 1, q_offset = N - 1) of every
    (batch, KV head): indices and counts bit-exact, gate logits and the
    normaliser within fp32 rounding of the oracle's brute-force sort."""
    d = U.decode_desc(w, w.seq, top_k=K)
    sel = api.block_topk(d, s.cuda())
    out = {"idx": sel.idx.cpu(), "gl": sel.gate_logit.cpu(), "slse": sel.score_lse.cpu(),
           "nsel": sel.n_sel.cpu()}
    grp = {(b, g): [0] for b in range(w.batch) for g in range(w.n_kv_heads)}
    wk = synth.Workload(w.name, "decode", w.batch, w.seq, w.n_q_heads, w.n_kv_heads, w.head_dim, w.block_size,
                        K, w.dtype, w.seed, w.qkv_std)
    check_topk_rows(wk, s, out, grp, top_k=K, q_offset=w.seq - 1, T=1)
    C = (w.seq - 1) // w.block_size
    assert (out["nsel"] == min(K, C)).all()


@pytest.mark.parametrize("K", [15, 31, 63])
def test_decode_topk_bit_exact(decode_ws, K):
    """The 131072-token decode workload's pooled-key scores at each budget."""
    w, _, _, _, s = decode_ws
    decode_topk_check(w, s, K)


@pytest.mark.parametrize("batch", [1, 8])
def test_long_decode_topk_bit_exact(batch):
    """The 524288-token workload's boosted scores (8191 candidates per row),
    every (batch, KV head) row, budget 2048 (K = 31)."""
    w = synth.workload("long", batch=batch)
    s = synth.decode_scores(w, synth.decode_q(w))
    decode_topk_check(w, s, w.top_k)


@pytest.mark.parametrize("K", [15, 31, 63])
def test_decode_budgets(decode_ws, K):
    w, kc, vc, q, s = decode_ws
    groups = [(0, g) for g in range(w.n_kv_heads)]
    decode_check(w, kc, vc, q, s, w.seq, K, groups)


@pytest.mark.parametrize("N", [1, 63, 64, 65, 100000])
def test_decode_ragged_lengths(decode_ws, N):
    """Cache lengths that leave a partial (or single-token) current block and
    rows with fewer candidates than K; the cache stride stays the full length."""
    w, kc, vc, q, _ = decode_ws
    NB = -(-N // w.block_size)
    s = torch.randn(1, w.n_kv_heads, 1, NB, generator=torch.Generator().manual_seed(N))
    groups = [(0, g) for g in (0, 3, 7)]
    decode_check(w, kc, vc, q, s, N, 31, groups)
    decode_check(w, kc, vc, q, s, N, 31, groups, gate="none")


@pytest.mark.parametrize("batch", [2, 4, 12, 24])
def test_decode_group_splits(batch):
    """Sparse decode at batch sizes that take each split of the block lists:
    clusters of 8, 4 and 1 CTAs per (batch, KV head) (16, 32, 96 groups) and
    the flat split over persistent CTAs once there are more groups than SMs
    (192 groups)."""
    w = synth.workload("decode", batch=batch, seq=8192 + 37)
    kc, vc = U.build_decode_cache(w)
    q = synth.decode_q(w)
    s = torch.randn(batch, w.n_kv_heads, 1, w.n_blocks, generator=torch.Generator().manual_seed(batch))
    groups = [(0, 0), (batch - 1, w.n_kv_heads - 1), (batch // 2, 3)]
    decode_check(w, kc, vc, q, s, w.seq, 31, groups)
    decode_check(w, kc, vc, q, s, w.seq, 15, groups[:2], gate="none")
    del kc, vc
    torch.cuda.empty_cache()


def test_decode_dense(decode_ws):
    w, kc, vc, q, s = decode_ws
    decode_check(w, kc, vc, q, s, w.seq, 31, [(0, 0), (0, 5)], dense=True)


@pytest.mark.parametrize("batch", [1, 8])
def test_long_decode(batch):
    """524288-token cache, budget 2048: sparse on sampled groups, dense too."""
    w = synth.workload("long", batch=batch)
    kc, vc = U.build_decode_cache(w)
    q = synth.decode_q(w)
    s = synth.decode_scores(w, q)
    groups = [(0, 0), (batch - 1, w.n_kv_heads - 1)] + ([(3, 2)] if batch > 3 else [])
    decode_check(w, kc, vc, q, s, w.seq, w.top_k, groups)
    decode_check(w, kc, vc, q, s, w.seq, w.top_k, groups[:1], dense=True)
    del kc, vc
    torch.cuda.empty_cache()


def test_autograd_function_matches_abi():
    """The autograd wrapper returns exactly what the direct calls return."""
    w = synth.workload("tiny")
    x, out = U.run_train(w)
    d = U.train_desc(w)
    q = x["q"].cuda().requires_grad_()
    k = x["k"].cuda().requires_grad_()
    v = x["v"].cuda().requires_grad_()
    s = x["scores"].cuda().requires_grad_()
    o = api.SASAttention.apply(q, k, v, s, d)
    o.backward(x["dO"].cuda())
    assert torch.equal(o.detach().cpu(), out["o"])
    assert torch.equal(q.grad.cpu(), out["dq"]) or torch.allclose(q.grad.cpu(), out["dq"], atol=1e-6)
    assert torch.allclose(s.grad.cpu(), out["ds"], atol=1e-6)
    assert math.isfinite(float(o.sum()))


def test_gqa_group_of_five_matches_oracle():
    """The tensor-core training path (gathered-row forward and backward)
    against the oracle, elementwise on a mid-size problem with G = 5 (128 rows
    per chunk hold 25 tokens and 3 padding rows)."""
    w = synth.Workload("mid", "train", 2, 1024, 10, 2, 128, 64, 5, "bf16", 21, 0.5, score_noise=0.1)
    x, out = U.run_train(w)
    G = w.group
    for b in range(w.batch):
        for g in range(w.n_kv_heads):
            d = U.group_desc(w)
            a = U.group_arrays(x, w, b, g)
            o, lse = oracle.fwd(d, a["q"], a["k"], a["v"], a["s"])
            go = out["o"][b, g * G:(g + 1) * G].float().numpy().transpose(1, 0, 2)
            assert np.abs(go - o).max() <= TOL_BF16_O
            np.testing.assert_allclose(out["lse"][b, g * G:(g + 1) * G].numpy().T, lse, atol=1e-4, rtol=0)
            r = oracle.bwd(d, a["q"], a["k"], a["v"], a["s"], a["dO"])
            got = {"dq": out["dq"][b, g * G:(g + 1) * G].float().numpy().transpose(1, 0, 2),
                   "dk": out["dk"][b:b + 1, g:g + 1].float().numpy(),
                   "dv": out["dv"][b:b + 1, g:g + 1].float().numpy(), "ds": out["ds"][b, g].numpy()}
            for key, val in got.items():
                assert U.normwise(val, r[key]) <= TOL_BF16_GRAD, key


def test_rows_beyond_the_softmax_shift_are_recomputed():
    """The gathered-row forward shifts each row's softmax by the row's own
    logit. Rows planted so that a neighbour key's logit exceeds the own one by
    about 650 (log2 units) overflow that shift; they must come out of the exact
    recompute, elementwise equal to the oracle, and the backward must follow."""
    w = synth.Workload("far", "train", 1, 512, 4, 1, 128, 64, 3, "bf16", 33, 0.5, score_kind="gauss")
    x = synth.train_inputs(w)
    gen = torch.Generator().manual_seed(5)
    u = torch.where(torch.rand(w.head_dim, generator=gen) < 0.5, -1.0, 1.0)
    for t in (130, 301, 302, 450):                 # the key t-1 shares t's block
        x["q"][0, :, t] = 20.0 * u
        x["k"][0, 0, t] = -u
        x["k"][0, 0, t - 1] = u
    x["scores"] = synth.train_scores(w, x["q"], x["k"])
    x, out = U.run_train(w, inputs=x)
    d = U.group_desc(w)
    a = U.group_arrays(x, w, 0, 0)
    o, lse = oracle.fwd(d, a["q"], a["k"], a["v"], a["s"])
    go = out["o"][0].float().numpy().transpose(1, 0, 2)
    assert np.isfinite(go).all()
    assert np.abs(go - o).max() <= TOL_BF16_O
    np.testing.assert_allclose(out["lse"][0].numpy().T, lse, atol=1e-4 * np.abs(lse).max(), rtol=0)
    r = oracle.bwd(d, a["q"], a["k"], a["v"], a["s"], a["dO"])
    got = {"dq": out["dq"][0].float().numpy().transpose(1, 0, 2), "dk": out["dk"].float().numpy(),
           "dv": out["dv"].float().numpy(), "ds": out["ds"][0, 0].numpy()}
    for key, val in got.items():
        assert U.normwise(val, r[key]) <= TOL_BF16_GRAD, key


def test_kernel_timing_hook_times_each_launch():
    """sas_kernel_timing / sas_kernel_time: one forward call on the tiny fp32
    workload records one CUDA-core forward launch with a positive duration;
    nothing is recorded once timing is off."""
    w = synth.workload("tiny")
    B.sas_kernel_timing("fwd_simt,block_topk")
    U.run_train(w, with_bwd=False)
    B.sas_kernel_timing(None)
    ms, n = B.sas_kernel_time("fwd_simt")
    assert n == 1 and ms > 0.0
    assert B.sas_kernel_time("block_topk")[1] == 1
    U.run_train(w, with_bwd=False)
    assert B.sas_kernel_time("fwd_simt")[1] == 1


def test_kernel_timing_filter():
    """Only the kernels named in the filter are recorded."""
    w = synth.workload("tiny")
    B.sas_kernel_timing("block_topk")
    U.run_train(w, with_bwd=False)
    B.sas_kernel_timing(None)
    assert B.sas_kernel_time("block_topk")[1] == 1
    assert B.sas_kernel_time("fwd_simt") == (0.0, 0)


# -------------------------------------------------------------- gate modes ---

GATE_MODES = {"sigmoid": oracle.GATE_SIGMOID, "raw": oracle.GATE_RAW,
              "softmax_selected": oracle.GATE_SOFTMAX_SELECTED, "ste": oracle.GATE_STE}


@pytest.mark.parametrize("gate", sorted(GATE_MODES))
def test_gate_modes_fp32_elementwise(gate):
    """Each gate activation on the tiny fp32 workload: top-K indices bit-exact,
    log-gates within fp32 rounding, every output and gradient within 1e-4."""
    w = synth.workload("tiny")
    x, out = U.run_train(w, gate=gate)
    d = U.group_desc(w, gate=GATE_MODES[gate])
    a = U.group_arrays(x, w, 0, 0)
    idx, gl, _, nsel = oracle.topk(d, a["s"])
    np.testing.assert_array_equal(out["idx"][0, 0].numpy(), idx)
    for r in range(w.seq):
        np.testing.assert_allclose(out["gl"][0, 0, r, :nsel[r]].numpy(), gl[r, :nsel[r]], atol=2e-5, rtol=1e-6)
    o, lse = oracle.fwd(d, a["q"], a["k"], a["v"], a["s"])
    np.testing.assert_allclose(out["o"][0].numpy().transpose(1, 0, 2), o, atol=TOL_FP32, rtol=0)
    r = oracle.bwd(d, a["q"], a["k"], a["v"], a["s"], a["dO"])
    np.testing.assert_allclose(out["dq"][0].numpy().transpose(1, 0, 2), r["dq"], atol=TOL_FP32, rtol=0)
    np.testing.assert_allclose(out["dk"].numpy(), r["dk"], atol=TOL_FP32, rtol=0)
    np.testing.assert_allclose(out["dv"].numpy(), r["dv"], atol=TOL_FP32, rtol=0)
    np.testing.assert_allclose(out["ds"][0, 0].numpy(), r["ds"], atol=TOL_FP32, rtol=0)


@pytest.mark.parametrize("gate", sorted(GATE_MODES))
def test_gate_modes_bf16_tensor_cores(gate):
    """Each gate activation through the tensor-core path (bf16, d 128, block
    64, G = 5): outputs within 1e-2, gradients and the score gradient within
    2e-2 normwise of the oracle."""
    w = synth.Workload("mid", "train", 1, 1024, 10, 2, 128, 64, 5, "bf16", 21, 0.5, score_noise=0.1)
    x, out = U.run_train(w, gate=gate)
    G = w.group
    for g in range(w.n_kv_heads):
        d = U.group_desc(w, gate=GATE_MODES[gate])
        a = U.group_arrays(x, w, 0, g)
        o, _ = oracle.fwd(d, a["q"], a["k"], a["v"], a["s"])
        assert np.abs(out["o"][0, g * G:(g + 1) * G].float().numpy().transpose(1, 0, 2) - o).max() <= TOL_BF16_O
        r = oracle.bwd(d, a["q"], a["k"], a["v"], a["s"], a["dO"])
        got = {"dq": out["dq"][0, g * G:(g + 1) * G].float().numpy().transpose(1, 0, 2),
               "dk": out["dk"][:, g:g + 1].float().numpy(), "dv": out["dv"][:, g:g + 1].float().numpy(),
               "ds": out["ds"][0, g].numpy()}
        for key, val in got.items():
            assert U.normwise(val, r[key]) <= TOL_BF16_GRAD, (gate, key)


@pytest.mark.parametrize("gate", sorted(GATE_MODES))
def test_gate_modes_decode(gate, decode_ws):
    """Each gate activation in the tensor-core decode (131072-token cache, K31)."""
    w, kc, vc, q, s = decode_ws
    decode_check(w, kc, vc, q, s, w.seq, 31, [(0, g) for g in (0, 4, 7)], gate=gate)


# --------------------------------------------- pooled-key scores (serving) ---

def test_pooled_scores_topk_decode(decode_ws):
    """sas_sparse_decode_pooled on the 131072-token cache: the block scores
    within float32 rounding of the oracle's fp64 pooled scores; the top-K of
    those very scores bit-exact; the output within 1e-2 of the oracle's decode
    with that selection."""
    w, kc, vc, q, _ = decode_ws
    kbar = kc.float().view(w.batch, w.n_kv_heads, -1, w.block_size, w.head_dim).mean(3).to(torch.bfloat16)
    d = U.decode_desc(w, w.seq, top_k=31)
    o, sc, sel = api.sparse_decode_pooled(d, q.to(torch.bfloat16).cuda(), kc, vc, kbar)
    torch.cuda.synchronize()
    od = oracle.Desc(batch=w.batch, seq_len=1, q_offset=w.seq - 1, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads,
                     head_dim=w.head_dim, block_size=w.block_size, top_k=31)
    ref_s = oracle.pooled_scores(od, q.numpy(), kbar.float().cpu().numpy())
    got_s = sc.cpu().numpy()
    np.testing.assert_allclose(got_s, ref_s, atol=2e-5, rtol=1e-5)
    idx, _, _, _ = oracle.topk(od, got_s)
    np.testing.assert_array_equal(sel.idx.cpu().numpy().reshape(idx.shape), idx)
    G = w.group
    got = o.float().cpu().numpy()
    for g in (0, 3, 7):
        og = oracle.Desc(batch=1, seq_len=1, q_offset=w.seq - 1, n_q_heads=G, n_kv_heads=1, head_dim=w.head_dim,
                         block_size=w.block_size, top_k=31)
        kk = synth.decode_cache_slice(w, "k", 0, g).numpy()[None, None]
        vv = synth.decode_cache_slice(w, "v", 0, g).numpy()[None, None]
        ref = oracle.decode(og, q[0:1, g * G:(g + 1) * G].numpy(), kk, vv, got_s[0:1, g:g + 1])
        assert np.abs(got[0, g * G:(g + 1) * G] - ref[0]).max() <= TOL_BF16_O


# ------------------------------------------------- sharding by (batch, KV head) ---

def test_kv_head_and_batch_shards_reproduce_the_full_call():
    """The path has no exchange step: every (batch, KV head) group is
    independent. Running it on each half of the KV heads (training) and on
    each half of the batch (decode) -- as the ranks of a multi-GPU run would --
    and concatenating gives the full call's results: top-K bit-exact, the rest
    within the bf16 tolerances (the order of floating-point additions differs)."""
    w = synth.Workload("mid", "train", 2, 1024, 10, 2, 128, 64, 5, "bf16", 21, 0.5, score_noise=0.1)
    x = synth.train_inputs(w)
    _, full = U.run_train(w, inputs=x)
    G = w.group
    for g in range(w.n_kv_heads):
        part = {"q": x["q"][:, g * G:(g + 1) * G].contiguous(), "k": x["k"][:, g:g + 1].contiguous(),
                "v": x["v"][:, g:g + 1].contiguous(), "dO": x["dO"][:, g * G:(g + 1) * G].contiguous(),
                "scores": x["scores"][:, g:g + 1].contiguous()}
        wg = synth.Workload("mid_shard", "train", w.batch, w.seq, G, 1, w.head_dim, w.block_size, w.top_k,
                            w.dtype, w.seed, w.qkv_std)
        _, sh = U.run_train(wg, inputs=part)
        assert torch.equal(sh["idx"], full["idx"][:, g:g + 1])
        assert (sh["o"].float() - full["o"][:, g * G:(g + 1) * G].float()).abs().max() <= TOL_BF16_O
        for key, sl in (("dq", np.s_[:, g * G:(g + 1) * G]), ("dk", np.s_[:, g:g + 1]), ("dv", np.s_[:, g:g + 1]),
                        ("ds", np.s_[:, g:g + 1])):
            assert U.normwise(sh[key].float().numpy(), full[key][sl].float().numpy()) <= TOL_BF16_GRAD, key
    # decode: each half of the batch against the full batch
    N, K = 8191, 31
    gen = torch.Generator().manual_seed(5)
    kc = (0.5 * torch.randn(4, 2, N, 128, generator=gen)).to(torch.bfloat16).cuda()
    vc = (0.5 * torch.randn(4, 2, N, 128, generator=gen)).to(torch.bfloat16).cuda()
    q = (0.5 * torch.randn(4, 8, 128, generator=gen)).to(torch.bfloat16).cuda()
    s = torch.randn(4, 2, 1, -(-N // 64), generator=gen).cuda()
    mk = lambda bsz: B.make_desc(batch=bsz, seq_len=1, q_offset=N - 1, n_q_heads=8, n_kv_heads=2, head_dim=128,
                                 block_size=64, top_k=K)
    of = api.sparse_decode(mk(4), q, kc, vc, api.block_topk(mk(4), s))
    for h in (0, 1):
        sl = slice(2 * h, 2 * h + 2)
        d2 = mk(2)
        oh = api.sparse_decode(d2, q[sl].contiguous(), kc[sl].contiguous(), vc[sl].contiguous(),
                               api.block_topk(d2, s[sl].contiguous()))
        assert (oh.float() - of[sl].float()).abs().max() <= 2e-3


def test_pooled_scores_many_tiles():
    """The block scan on the 524288-token shape at batch 8 (64 rows of 8191
    blocks: every scan CTA walks a run of many tiles through its ring, runs
    crossing from one (batch, KV head) row into the next), all scores against
    the oracle within float32 rounding; with a per-query-head selection too."""
    gen = torch.Generator().manual_seed(61)
    Bn, Hq, Hkv, N = 8, 32, 8, 524288
    C = (N - 1) // 64
    q = (0.5 * torch.randn(Bn, Hq, 128, generator=gen)).to(torch.bfloat16)
    kbar = (0.5 * torch.randn(Bn, Hkv, C, 128, generator=gen)).to(torch.bfloat16)
    for per_head in (False, True):
        d = B.make_desc(batch=Bn, seq_len=1, q_offset=N - 1, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=128,
                        block_size=64, top_k=31, select_heads=per_head)
        H = Hq if per_head else Hkv
        sc = torch.empty(Bn, H, 1, -(-N // 64), dtype=torch.float32, device="cuda")
        B.sas_block_scores_pooled(d, q.cuda(), kbar.cuda(), sc)
        torch.cuda.synchronize()
        od = oracle.Desc(batch=Bn, seq_len=1, q_offset=N - 1, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=128,
                         block_size=64, top_k=31)
        kb = kbar.float().numpy()
        if per_head:
            od = oracle.per_head_desc(od)
            kb = np.repeat(kb, Hq // Hkv, axis=1)
        ref = oracle.pooled_scores(od, q.float().numpy(), kb)
        np.testing.assert_allclose(sc.cpu().numpy(), ref, atol=2e-5, rtol=1e-5)
