"""Pins of the oracle to things other than itself (CPU only).

Each check is written independently of oracle/sas_oracle.c:
  * dense reduction: gate off and K >= C is textbook causal softmax attention
    (study note 1-1, dense attention eq.), here a plain torch fp64 matmul;
  * the materialised [T, T] bias formulation, i.e. the naive implementation the
    study note (3-6) describes, with the identity of 2-2, built with a stable
    torch sort for the top-K, and its fp64 autograd for every gradient;
  * shift invariance of the normalised gate (arXiv text, 4, ablation discussion);
  * central finite differences on tiny inputs;
  * the row sums that follow from softmax: sum_i ds_i = 0 and
    Gsum_current = -sum_I Gsum;
  * hand-derived worked examples and tie cases under tests/golden/;
  * brute-force top-K by numpy lexsort;
  * decode row == training row p = N-1.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand_problem(seed, B=2, T=48, Hq=4, Hkv=2, d=16, bs=8, K=2, gate=0, scale_s=1.0):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Hq, T, d, generator=g)
    k = torch.randn(B, Hkv, T, d, generator=g)
    v = torch.randn(B, Hkv, T, d, generator=g)
    dO = torch.randn(B, Hq, T, d, generator=g)
    NB = -(-T // bs)
    s = torch.randn(B, Hkv, T, NB, generator=g) * scale_s
    return dict(q=q, k=k, v=v, dO=dO, s=s, B=B, T=T, Hq=Hq, Hkv=Hkv, d=d, bs=bs, K=K, gate=gate)


def desc_of(oracle, P, **over):
    kw = dict(batch=P["B"], seq_len=P["T"], n_q_heads=P["Hq"], n_kv_heads=P["Hkv"],
              head_dim=P["d"], block_size=P["bs"], top_k=P["K"], gate=P["gate"])
    kw.update(over)
    return oracle.Desc(**kw)


# ------------------------------------------------------- independent references ---

def dense_causal_torch(q, k, v, scale):
    """Textbook causal softmax attention with GQA head sharing, fp64."""
    G = q.shape[1] // k.shape[1]
    q, k, v = q.double(), k.double().repeat_interleave(G, 1), v.double().repeat_interleave(G, 1)
    T = q.shape[2]
    logits = scale * q @ k.transpose(-1, -2)
    causal = torch.ones(T, T, dtype=torch.bool).tril()
    logits = logits.masked_fill(~causal, float("-inf"))
    return torch.softmax(logits, -1) @ v, torch.logsumexp(logits, -1)


def stable_topk(srow, C, K):
    """Top-K by a stable descending sort (equal scores keep ascending index)."""
    if C == 0:
        return []
    order = torch.sort(srow[:C], descending=True, stable=True).indices
    return sorted(order[: min(K, C)].tolist())


def bias_matrix_torch(P, s, gate_on=True):
    """The naive form: materialise the [T,T] additive bias (log-gate on kept
    historical tokens, 0 on the causal current block, -inf elsewhere) and run
    dense softmax attention. `s` may require grad."""
    B, T, Hq, Hkv, d, bs, K = (P[x] for x in ("B", "T", "Hq", "Hkv", "d", "bs", "K"))
    G = Hq // Hkv
    rows = []
    for b in range(B):
        per_g = []
        for g in range(Hkv):
            per_t = []
            for t in range(T):
                C = t // bs
                sel = stable_topk(s[b, g, t].detach(), C, K)
                row = torch.full((T,), float("-inf"), dtype=torch.float64)
                if sel:
                    lse = torch.logsumexp(s[b, g, t, :C].double(), 0)
                    for i in sel:
                        logg = (s[b, g, t, i].double() - lse) if gate_on else torch.zeros((), dtype=torch.float64)
                        row = torch.cat([row[: i * bs], logg.expand(bs), row[(i + 1) * bs:]])
                cur = torch.zeros(t - C * bs + 1, dtype=torch.float64)
                row = torch.cat([row[: C * bs], cur, row[t + 1:]])
                per_t.append(row)
            per_g.append(torch.stack(per_t))
        rows.append(torch.stack(per_g))
    bias = torch.stack(rows)                       # [B, Hkv, T, T]
    bias = bias.repeat_interleave(G, 1)            # [B, Hq, T, T]
    kk = P["k"].double().repeat_interleave(G, 1)
    vv = P["v"].double().repeat_interleave(G, 1)
    logits = P["q"].double() @ kk.transpose(-1, -2) / math.sqrt(d) + bias
    return torch.softmax(logits, -1) @ vv, torch.logsumexp(logits, -1)


def oracle_o_full(oracle, desc, P, s=None):
    """Oracle forward over every row, reshaped to [B, Hq, T, d]."""
    s = P["s"] if s is None else s
    o, lse = oracle.fwd(desc, P["q"].numpy(), P["k"].numpy(), P["v"].numpy(), s.numpy())
    B, Hkv, T, G, d = desc.batch, desc.n_kv_heads, desc.seq_len, desc.group, desc.head_dim
    o = o.reshape(B, Hkv, T, G, d).transpose(0, 1, 3, 2, 4).reshape(B, Hkv * G, T, d)
    lse = lse.reshape(B, Hkv, T, G).transpose(0, 1, 3, 2).reshape(B, Hkv * G, T)
    return o, lse


def oracle_bwd_full(oracle, desc, P, s=None):
    s = P["s"] if s is None else s
    r = oracle.bwd(desc, P["q"].numpy(), P["k"].numpy(), P["v"].numpy(), s.numpy(), P["dO"].numpy())
    B, Hkv, T, G, d = desc.batch, desc.n_kv_heads, desc.seq_len, desc.group, desc.head_dim
    r["dq"] = r["dq"].reshape(B, Hkv, T, G, d).transpose(0, 1, 3, 2, 4).reshape(B, Hkv * G, T, d)
    r["ds"] = r["ds"].reshape(B, Hkv, T, -1)
    return r


# ------------------------------------------------------------------------ tests ---

@pytest.mark.parametrize("seed", [0, 1])
def test_dense_reduction(oracle_mod, seed):
    """Gate off with K >= C equals causal softmax attention (P-1)."""
    P = rand_problem(seed, gate=1)
    NB = -(-P["T"] // P["bs"])
    desc = desc_of(oracle_mod, P, top_k=NB, gate=oracle_mod.GATE_NONE)
    o, lse = oracle_o_full(oracle_mod, desc, P)
    ro, rl = dense_causal_torch(P["q"], P["k"], P["v"], 1 / math.sqrt(P["d"]))
    np.testing.assert_allclose(o, ro.numpy(), atol=1e-12, rtol=0)
    np.testing.assert_allclose(lse, rl.numpy(), atol=1e-12, rtol=0)


def test_dense_reduction_gate_on_single_candidate(oracle_mod):
    """With K >= C and the softmax gate, rows with C <= 1 are still dense attention
    (one candidate has gate 1), and all others differ: the gate matters."""
    P = rand_problem(3, T=24, bs=8)
    desc = desc_of(oracle_mod, P, top_k=3)
    o, _ = oracle_o_full(oracle_mod, desc, P)
    ro, _ = dense_causal_torch(P["q"], P["k"], P["v"], 1 / math.sqrt(P["d"]))
    np.testing.assert_allclose(o[:, :, :16], ro.numpy()[:, :, :16], atol=1e-12, rtol=0)
    assert np.abs(o[:, :, 16:] - ro.numpy()[:, :, 16:]).max() > 1e-3


@pytest.mark.parametrize("seed,K,gate", [(0, 2, 0), (1, 3, 0), (2, 1, 0), (3, 2, 1)])
def test_bias_matrix_forward(oracle_mod, seed, K, gate):
    """Oracle forward equals the materialised-bias formulation (P-2)."""
    P = rand_problem(seed, K=K, gate=gate)
    desc = desc_of(oracle_mod, P)
    o, lse = oracle_o_full(oracle_mod, desc, P)
    ro, rl = bias_matrix_torch(P, P["s"], gate_on=(gate == 0))
    np.testing.assert_allclose(o, ro.numpy(), atol=1e-12, rtol=0)
    np.testing.assert_allclose(lse, rl.numpy(), atol=1e-12, rtol=0)


@pytest.mark.parametrize("seed,K,gate", [(0, 2, 0), (4, 3, 0), (5, 2, 1)])
def test_autograd_backward(oracle_mod, seed, K, gate):
    """Oracle gradients equal fp64 autograd of the bias formulation (P-7):
    dq, dk, dv and the score gradient (through the gate normaliser)."""
    P = rand_problem(seed, B=1, T=40, K=K, gate=gate)
    desc = desc_of(oracle_mod, P)
    q = P["q"].double().requires_grad_()
    k = P["k"].double().requires_grad_()
    v = P["v"].double().requires_grad_()
    s = P["s"].double().requires_grad_()
    Pt = dict(P, q=q, k=k, v=v)
    o, _ = bias_matrix_torch(Pt, s, gate_on=(gate == 0))
    (o * P["dO"].double()).sum().backward()
    r = oracle_bwd_full(oracle_mod, desc, P)
    np.testing.assert_allclose(r["dq"], q.grad.numpy(), atol=1e-11, rtol=0)
    np.testing.assert_allclose(r["dk"], k.grad.numpy(), atol=1e-11, rtol=0)
    np.testing.assert_allclose(r["dv"], v.grad.numpy(), atol=1e-11, rtol=0)
    sg = s.grad.numpy() if s.grad is not None else np.zeros(s.shape)   # gate off: no path to s
    np.testing.assert_allclose(r["ds"], sg, atol=1e-11, rtol=0)


@pytest.mark.parametrize("c", [1.0, 8.0, -3.5])
def test_shift_invariance(oracle_mod, c):
    """Adding c to all of a row's scores leaves the selection, the output and the
    score gradient unchanged (P-3). Scores are multiples of 2^-10 so that s + c
    is exact in float32."""
    P = rand_problem(7, K=2)
    P["s"] = torch.round(P["s"] * 1024) / 1024
    desc = desc_of(oracle_mod, P)
    s2 = P["s"] + c
    assert torch.equal(s2 - c, P["s"])
    i1 = oracle_mod.topk(desc, P["s"].numpy())
    i2 = oracle_mod.topk(desc, s2.numpy())
    np.testing.assert_array_equal(i1[0], i2[0])
    np.testing.assert_allclose(i1[1], i2[1], atol=1e-12, rtol=0)
    o1, _ = oracle_o_full(oracle_mod, desc, P)
    o2, _ = oracle_o_full(oracle_mod, desc, P, s2)
    np.testing.assert_allclose(o1, o2, atol=1e-12, rtol=0)
    r1 = oracle_bwd_full(oracle_mod, desc, P)
    r2 = oracle_bwd_full(oracle_mod, desc, P, s2)
    for key in ("dq", "dk", "dv", "ds"):
        np.testing.assert_allclose(r1[key], r2[key], atol=1e-12, rtol=0)


def test_finite_differences(oracle_mod):
    """Analytic gradients match central finite differences (P-4) on a tiny
    problem: L = sum(o * W). Score coordinates whose perturbation changes the
    top-K set are skipped (the selection is piecewise constant)."""
    P = rand_problem(11, B=1, T=16, Hq=2, Hkv=1, d=8, bs=4, K=2)
    desc = desc_of(oracle_mod, P)
    W = P["dO"].numpy()
    base = {n: P[n].numpy().astype(np.float32).copy() for n in ("q", "k", "v", "s")}

    def loss(arrs):
        o, _ = oracle_mod.fwd(desc, arrs["q"], arrs["k"], arrs["v"], arrs["s"])
        o = o.reshape(1, 1, 16, 2, 8).transpose(0, 1, 3, 2, 4).reshape(1, 2, 16, 8)
        return float((o * W).sum())

    r = oracle_bwd_full(oracle_mod, desc, P)
    grads = {"q": r["dq"], "k": r["dk"], "v": r["dv"], "s": r["ds"]}
    idx0 = oracle_mod.topk(desc, base["s"])[0]
    eps = 1e-3
    checked = 0
    for name in ("q", "k", "v", "s"):
        flat = base[name].reshape(-1)
        for j in range(flat.size):
            x = flat[j]
            xp, xm = np.float32(x + eps), np.float32(x - eps)
            hp, hm = float(xp) - float(x), float(x) - float(xm)
            arrs = {n: a.copy() for n, a in base.items()}
            arrs[name].reshape(-1)[j] = xp
            if name == "s" and not np.array_equal(oracle_mod.topk(desc, arrs["s"])[0], idx0):
                continue
            lp = loss(arrs)
            arrs[name].reshape(-1)[j] = xm
            if name == "s" and not np.array_equal(oracle_mod.topk(desc, arrs["s"])[0], idx0):
                continue
            lm = loss(arrs)
            fd = (lp - lm) / (hp + hm)
            an = grads[name].reshape(-1)[j]
            assert abs(fd - an) <= 2e-6 * max(1.0, abs(an)), (name, j, fd, an)
            checked += 1
    assert checked > 500


def test_row_sum_identities(oracle_mod):
    """sum_i ds_i = 0 per row (P-5) and the current block's dS sum balances the
    kept blocks' (P-6): both follow from sum_j dS_j = 0 for a softmax row."""
    P = rand_problem(13, K=3)
    desc = desc_of(oracle_mod, P)
    r = oracle_mod.bwd(desc, P["q"].numpy(), P["k"].numpy(), P["v"].numpy(), P["s"].numpy(),
                       P["dO"].numpy())
    assert np.abs(r["ds"].sum(1)).max() < 1e-12
    assert np.abs(r["gsum"].sum(1) + r["gsum_cur"]).max() < 1e-12
    assert np.abs(r["ds"]).max() > 1e-3


def test_golden_worked_example(oracle_mod):
    with open(os.path.join(GOLDEN, "worked_gate_example.json")) as f:
        G = json.load(f)
    dsc = oracle_mod.Desc(**{k: v for k, v in G["desc"].items()})
    T, d = dsc.seq_len, dsc.head_dim
    q = np.zeros((1, 1, T, d), np.float32)
    k = np.array(G["k"], np.float32).reshape(1, 1, T, d)
    v = np.array(G["v"], np.float32).reshape(1, 1, T, d)
    s = np.array(G["scores"], np.float32).reshape(1, 1, T, -1)
    rows = [r["t"] for r in G["rows"]]
    idx, _, _, nsel = oracle_mod.topk(dsc, s, rows)
    o, lse = oracle_mod.fwd(dsc, q, k, v, s, rows)
    for i, r in enumerate(G["rows"]):
        assert idx[i].tolist() == r["idx"] and nsel[i] == r["n_sel"]
        np.testing.assert_allclose(o[i, 0], r["o"], atol=1e-14, rtol=1e-14)
        assert abs(lse[i, 0] - r["attn_lse"]) < 1e-14
    bw = G["backward"]
    dO = np.zeros((1, 1, T, d), np.float32)
    dO[0, 0, bw["t"]] = bw["dO"]
    q2 = np.zeros_like(q)
    res = oracle_mod.bwd(dsc, q2, k, v, s, dO, [bw["t"]])
    np.testing.assert_allclose(res["dq"][0, 0], bw["dq"], atol=1e-14, rtol=1e-13)
    np.testing.assert_allclose(res["gsum"][0], bw["gsum"], atol=1e-14, rtol=1e-13)
    assert abs(res["gsum_cur"][0] - bw["gsum_cur"]) < 1e-14
    np.testing.assert_allclose(res["ds"][0], bw["ds"], atol=1e-14, rtol=1e-13)


def test_golden_topk_ties(oracle_mod):
    with open(os.path.join(GOLDEN, "topk_ties.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        svals = [float(x) for x in c["s"]]
        C, K = len(svals), c["K"]
        bs = 4
        T = C * bs + 1                      # the last row has exactly C candidates
        NB = -(-T // bs)
        s = np.zeros((1, 1, T, NB), np.float32)
        s[0, 0, T - 1, :C] = svals
        dsc = oracle_mod.Desc(batch=1, seq_len=T, n_q_heads=1, n_kv_heads=1, head_dim=4,
                              block_size=bs, top_k=K)
        idx, gl, lse, nsel = oracle_mod.topk(dsc, s, [T - 1])
        assert idx[0].tolist() == c["idx"], c["name"]
        assert nsel[0] == min(C, K)


def test_topk_bruteforce_lexsort(oracle_mod):
    """Random rows with many exact ties (small integer scores) against a numpy
    lexsort brute force; lse against a max-shifted log-sum-exp."""
    rng = np.random.default_rng(5)
    dsc = oracle_mod.Desc(batch=2, seq_len=96, n_q_heads=2, n_kv_heads=2, head_dim=4,
                          block_size=4, top_k=5)
    NB = dsc.n_blocks
    s = rng.integers(-3, 4, size=(2, 2, 96, NB)).astype(np.float32)
    s[rng.random(s.shape) < 0.05] = -np.inf
    s[rng.random(s.shape) < 0.05] = -0.0
    idx, gl, lse, nsel = oracle_mod.topk(dsc, s)
    for r in range(dsc.n_rows):
        b, g, t = r // (2 * 96), (r // 96) % 2, r % 96
        C = t // 4
        row = s[b, g, t, :C].astype(np.float64)
        order = np.lexsort((np.arange(C), -row))      # primary: -score, then index
        exp_idx = sorted(order[:min(5, C)].tolist())
        assert idx[r, :len(exp_idx)].tolist() == exp_idx
        assert (idx[r, len(exp_idx):] == -1).all()
        if C and np.isfinite(row).any():
            m = row[np.isfinite(row)].max()
            ref = m + math.log(np.exp(row - m).sum())
            assert abs(lse[r] - ref) < 1e-12
            np.testing.assert_allclose(gl[r, :nsel[r]], row[exp_idx] - ref, atol=1e-12)


def test_decode_equals_training_row(oracle_mod):
    """The decode oracle (its own loop) equals the training row p = N - 1, for
    the gated sparse case and for dense decode (gate off, every block)."""
    P = rand_problem(17, B=2, T=45, bs=8, K=2)
    T, NB = P["T"], -(-P["T"] // P["bs"])
    desc = desc_of(oracle_mod, P)
    o, _ = oracle_o_full(oracle_mod, desc, P)
    ddesc = desc_of(oracle_mod, P, seq_len=1, q_offset=T - 1)
    qd = P["q"][:, :, T - 1].numpy()
    sd = P["s"][:, :, T - 1:T].numpy()
    od = oracle_mod.decode(ddesc, qd, P["k"].numpy(), P["v"].numpy(), sd)
    np.testing.assert_allclose(od, o[:, :, T - 1], atol=1e-12, rtol=0)
    dense = oracle_mod.decode(ddesc, qd, P["k"].numpy(), P["v"].numpy(), None)
    ro, _ = dense_causal_torch(P["q"], P["k"], P["v"], 1 / math.sqrt(P["d"]))
    np.testing.assert_allclose(dense, ro[:, :, T - 1].numpy(), atol=1e-12, rtol=0)
    assert NB == 6


def test_paged_varlen_decode_pins(oracle_mod):
    """Paged decode with a cache length per sequence: for every sequence the
    oracle equals the last row of the naive [T, T] bias form (gated) and of
    textbook causal attention (dense) over that sequence's own tokens, with
    the pages placed in the pools through a shuffled block table; the
    per-sequence top-K equals a stable sort of the row's own candidates."""
    g = torch.Generator().manual_seed(23)
    B, Hkv, Hq, d, bs, K = 3, 2, 4, 16, 8, 2
    lens = [45, 17, 33]
    NB = -(-max(lens) // bs)
    k = torch.randn(B, Hkv, NB * bs, d, generator=g)
    v = torch.randn(B, Hkv, NB * bs, d, generator=g)
    q = torch.randn(B, Hq, d, generator=g)
    s = torch.randn(B, Hkv, 1, NB, generator=g)
    perm = torch.randperm(B * NB, generator=g)
    k_pages = torch.zeros(B * NB, Hkv, bs, d)
    v_pages = torch.zeros(B * NB, Hkv, bs, d)
    table = np.zeros((B, NB), np.int32)
    for i in range(B):
        for j in range(NB):
            pg = int(perm[i * NB + j])
            table[i, j] = pg
            k_pages[pg] = k[i, :, j * bs:(j + 1) * bs]
            v_pages[pg] = v[i, :, j * bs:(j + 1) * bs]
    desc = oracle_mod.Desc(batch=B, seq_len=1, q_offset=max(lens) - 1, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d,
                           block_size=bs, top_k=K)
    o = oracle_mod.decode_paged(desc, q.numpy(), k_pages.numpy(), v_pages.numpy(), table, lens, s.numpy())
    od = oracle_mod.decode_paged(desc, q.numpy(), k_pages.numpy(), v_pages.numpy(), table, lens, None)
    idx, _, _, nsel = oracle_mod.topk_varlen(desc, s.numpy(), lens)
    for i, n in enumerate(lens):
        C = (n - 1) // bs
        for gg in range(Hkv):
            assert stable_topk(s[i, gg, 0], C, K) == [int(x) for x in idx[i * Hkv + gg, :nsel[i * Hkv + gg]]]
        # sequence i as a training problem of T = n rows whose last row is the decode query
        Pi = dict(q=torch.randn(1, Hq, n, d, generator=g), k=k[i:i + 1, :, :n], v=v[i:i + 1, :, :n],
                  s=torch.randn(1, Hkv, n, -(-n // bs), generator=g), B=1, T=n, Hq=Hq, Hkv=Hkv, d=d, bs=bs, K=K)
        Pi["q"][0, :, n - 1] = q[i]
        Pi["s"][0, :, n - 1] = s[i, :, 0, :-(-n // bs)]
        ro, _ = bias_matrix_torch(Pi, Pi["s"])
        np.testing.assert_allclose(o[i], ro[0, :, n - 1].numpy(), atol=1e-12, rtol=0)
        rd, _ = dense_causal_torch(Pi["q"], Pi["k"], Pi["v"], 1 / math.sqrt(d))
        np.testing.assert_allclose(od[i], rd[0, :, n - 1].numpy(), atol=1e-12, rtol=0)


# ------------------------------------------------------------- gate modes ---

def _logg_mode(mode, srow, C, sel, i):
    """log g_i of kept block i under each gate activation the pages compare
    (arXiv text, 4, design elements), written with torch ops on the row's
    scores so that autograd differentiates it."""
    if mode == 2:                                   # independent sigmoid gates
        return torch.nn.functional.logsigmoid(srow[i].double())
    if mode == 3:                                   # raw score as the logit bias
        return srow[i].double()
    if mode == 4:                                   # softmax over the kept blocks
        return srow[i].double() - torch.logsumexp(srow[sel].double(), 0)
    if mode == 5:                                   # hard gate, straight-through softmax gradient
        g = torch.exp(srow[i].double() - torch.logsumexp(srow[:C].double(), 0))
        return torch.log(g + (1.0 - g).detach())
    raise ValueError(mode)


def bias_matrix_mode(P, s, mode):
    """The naive [T, T] bias form (as bias_matrix_torch) with the log-gate of
    gate activation `mode`."""
    B, T, Hq, Hkv, d, bs, K = (P[x] for x in ("B", "T", "Hq", "Hkv", "d", "bs", "K"))
    G = Hq // Hkv
    rows = []
    for b in range(B):
        per_g = []
        for g in range(Hkv):
            per_t = []
            for t in range(T):
                C = t // bs
                sel = stable_topk(s[b, g, t].detach(), C, K)
                row = torch.full((T,), float("-inf"), dtype=torch.float64)
                for i in sel:
                    logg = _logg_mode(mode, s[b, g, t], C, sel, i)
                    row = torch.cat([row[: i * bs], logg.expand(bs), row[(i + 1) * bs:]])
                cur = torch.zeros(t - C * bs + 1, dtype=torch.float64)
                row = torch.cat([row[: C * bs], cur, row[t + 1:]])
                per_t.append(row)
            per_g.append(torch.stack(per_t))
        rows.append(torch.stack(per_g))
    bias = torch.stack(rows).repeat_interleave(G, 1)
    kk = P["k"].double().repeat_interleave(G, 1)
    vv = P["v"].double().repeat_interleave(G, 1)
    logits = P["q"].double() @ kk.transpose(-1, -2) / math.sqrt(d) + bias
    return torch.softmax(logits, -1) @ vv, torch.logsumexp(logits, -1)


@pytest.mark.parametrize("mode", [2, 3, 4, 5])
def test_gate_modes_forward_and_autograd(oracle_mod, mode):
    """Each gate activation: the oracle's forward, log-gates and every gradient
    (dq, dk, dv and the score gradient through the activation) equal the bias
    form and its fp64 autograd."""
    P = rand_problem(30 + mode, B=1, T=40, K=2, gate=mode)
    desc = desc_of(oracle_mod, P)
    o, lse = oracle_o_full(oracle_mod, desc, P)
    ro, rl = bias_matrix_mode(P, P["s"], mode)
    np.testing.assert_allclose(o, ro.detach().numpy(), atol=1e-12, rtol=0)
    np.testing.assert_allclose(lse, rl.detach().numpy(), atol=1e-12, rtol=0)
    q = P["q"].double().requires_grad_()
    k = P["k"].double().requires_grad_()
    v = P["v"].double().requires_grad_()
    s = P["s"].double().requires_grad_()
    o2, _ = bias_matrix_mode(dict(P, q=q, k=k, v=v), s, mode)
    (o2 * P["dO"].double()).sum().backward()
    r = oracle_bwd_full(oracle_mod, desc, P)
    np.testing.assert_allclose(r["dq"], q.grad.numpy(), atol=1e-11, rtol=0)
    np.testing.assert_allclose(r["dk"], k.grad.numpy(), atol=1e-11, rtol=0)
    np.testing.assert_allclose(r["dv"], v.grad.numpy(), atol=1e-11, rtol=0)
    np.testing.assert_allclose(r["ds"], s.grad.numpy(), atol=1e-11, rtol=0)


def test_gate_mode_closed_forms(oracle_mod):
    """Log-gates of one row by hand: scores (0, 1, 2, 3), K = 2 keeps blocks 2
    and 3; sigmoid gives log(1 / (1 + e^-s)), raw gives s, the kept-block
    softmax gives s - log(e^2 + e^3), the hard gate gives 0."""
    srow = np.array([[[[0.0, 1.0, 2.0, 3.0, 0.0]]]], np.float32)
    for mode, exp in [(2, [-math.log1p(math.exp(-2.0)), -math.log1p(math.exp(-3.0))]),
                      (3, [2.0, 3.0]),
                      (4, [2.0 - math.log(math.exp(2) + math.exp(3)), 3.0 - math.log(math.exp(2) + math.exp(3))]),
                      (5, [0.0, 0.0])]:
        d = oracle_mod.Desc(batch=1, seq_len=1, q_offset=4 * 8, n_q_heads=1, n_kv_heads=1, head_dim=8,
                            block_size=8, top_k=2, gate=mode)
        idx, gl, lse, n = oracle_mod.topk(d, srow)
        assert idx[0].tolist() == [2, 3] and n[0] == 2
        np.testing.assert_allclose(gl[0], exp, atol=1e-12, rtol=0)
        assert abs(lse[0] - math.log(1 + math.e + math.e ** 2 + math.e ** 3)) < 1e-12


def test_pooled_scores_pins(oracle_mod):
    """The pooled-key block scores equal the seeded input recipe's own score
    (torch float32: mean of each block's keys dotted with the mean of the
    group's query heads) within float32 rounding, are 0 past the candidates,
    and match a hand example."""
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    from trainable_block_sparse_topk_b200 import synth
    w = synth.workload("decode", seq=64 * 9)
    q = synth.decode_q(w)
    ref = synth.decode_scores(w, q)                     # torch: kbar @ qbar per (b, g)
    kbar = torch.stack([torch.stack([synth.decode_cache_slice(w, "k", b, g).reshape(-1, 64, w.head_dim).mean(1)
                                     for g in range(w.n_kv_heads)]) for b in range(w.batch)])
    d = oracle_mod.Desc(batch=w.batch, seq_len=1, q_offset=w.seq - 1, n_q_heads=w.n_q_heads,
                        n_kv_heads=w.n_kv_heads, head_dim=w.head_dim, block_size=64, top_k=31)
    s = oracle_mod.pooled_scores(d, q.numpy(), kbar.numpy())
    C = (w.seq - 1) // 64
    np.testing.assert_allclose(s[..., :C], ref[..., :C].numpy(), atol=2e-6, rtol=1e-5)
    assert (s[..., C:] == 0).all()
    # by hand: qbar = mean of (1, 0) and (3, 2) = (2, 1); blocks (1, 1), (0, -2)
    d2 = oracle_mod.Desc(batch=1, seq_len=1, q_offset=2 * 4, n_q_heads=2, n_kv_heads=1, head_dim=2,
                         block_size=4, top_k=1)
    s2 = oracle_mod.pooled_scores(d2, np.array([[[1, 0], [3, 2]]], np.float32),
                                  np.array([[[[1, 1], [0, -2]]]], np.float32))
    np.testing.assert_array_equal(s2[0, 0, 0], [3.0, -2.0, 0.0])


# ------------------------------------------------- per-query-head selection ---

def bias_matrix_per_head_torch(P, s, gate_on=True):
    """The naive form with a selection per query head: head h builds its
    [T,T] bias from its own score row s[b, h] and attends to the K/V of head
    h // G. `s` [B, Hq, T, NB] may require grad."""
    B, T, Hq, Hkv, d, bs, K = (P[x] for x in ("B", "T", "Hq", "Hkv", "d", "bs", "K"))
    G = Hq // Hkv
    out, lses = [], []
    for b in range(B):
        ob, lb = [], []
        for h in range(Hq):
            rows = []
            for t in range(T):
                C = t // bs
                sel = stable_topk(s[b, h, t].detach(), C, K)
                row = torch.full((T,), float("-inf"), dtype=torch.float64)
                if sel:
                    lse = torch.logsumexp(s[b, h, t, :C].double(), 0)
                    for i in sel:
                        logg = (s[b, h, t, i].double() - lse) if gate_on else torch.zeros((), dtype=torch.float64)
                        row = torch.cat([row[: i * bs], logg.expand(bs), row[(i + 1) * bs:]])
                row = torch.cat([row[: C * bs], torch.zeros(t - C * bs + 1, dtype=torch.float64), row[t + 1:]])
                rows.append(row)
            bias = torch.stack(rows)
            logits = P["q"][b, h].double() @ P["k"][b, h // G].double().T / math.sqrt(d) + bias
            ob.append(torch.softmax(logits, -1) @ P["v"][b, h // G].double())
            lb.append(torch.logsumexp(logits, -1))
        out.append(torch.stack(ob))
        lses.append(torch.stack(lb))
    return torch.stack(out), torch.stack(lses)


@pytest.mark.parametrize("seed,K,gate", [(11, 2, 0), (12, 3, 1)])
def test_per_head_selection_pins(oracle_mod, seed, K, gate):
    """Per-query-head selection: the oracle's forward and every gradient
    (dq, dk/dv summed over the heads sharing a KV head, ds per head row) equal
    fp64 autograd of the per-head bias formulation, and with identical score
    rows across a group the selection -- and so the result -- equals the
    per-group oracle."""
    P = rand_problem(seed, B=1, T=40, Hq=4, Hkv=2, K=K, gate=gate)
    g = torch.Generator().manual_seed(seed + 100)
    sh = torch.randn(P["B"], P["Hq"], P["T"], P["s"].shape[-1], generator=g)
    desc = desc_of(oracle_mod, P)
    G = P["Hq"] // P["Hkv"]
    q = P["q"].double().requires_grad_()
    k = P["k"].double().requires_grad_()
    v = P["v"].double().requires_grad_()
    s = sh.double().requires_grad_()
    o, lse = bias_matrix_per_head_torch(dict(P, q=q, k=k, v=v), s, gate_on=(gate == 0))
    (o * P["dO"].double()).sum().backward()
    B, T, dh = P["B"], P["T"], P["d"]
    of, lf = oracle_mod.fwd_per_head(desc, P["q"].numpy(), P["k"].numpy(), P["v"].numpy(), sh.numpy())
    np.testing.assert_allclose(of.reshape(B, P["Hq"], T, dh), o.detach().numpy(), atol=1e-12, rtol=0)
    np.testing.assert_allclose(lf.reshape(B, P["Hq"], T), lse.detach().numpy(), atol=1e-12, rtol=0)
    r = oracle_mod.bwd_per_head(desc, P["q"].numpy(), P["k"].numpy(), P["v"].numpy(), sh.numpy(),
                                P["dO"].numpy())
    np.testing.assert_allclose(r["dq"].reshape(B, P["Hq"], T, dh), q.grad.numpy(), atol=1e-11, rtol=0)
    np.testing.assert_allclose(r["dk"], k.grad.numpy(), atol=1e-11, rtol=0)
    np.testing.assert_allclose(r["dv"], v.grad.numpy(), atol=1e-11, rtol=0)
    sg = s.grad.numpy() if s.grad is not None else np.zeros(s.shape)
    np.testing.assert_allclose(r["ds"].reshape(sh.shape), sg, atol=1e-11, rtol=0)
    # a group's heads with one shared score row reduce to the per-group selection
    s_grp = P["s"].repeat_interleave(G, 1)
    o_h, _ = oracle_mod.fwd_per_head(desc, P["q"].numpy(), P["k"].numpy(), P["v"].numpy(), s_grp.numpy())
    o_g, _ = oracle_o_full(oracle_mod, desc, P)
    np.testing.assert_allclose(o_h.reshape(B, P["Hq"], T, dh), o_g, atol=1e-12, rtol=0)


def test_per_head_decode_pin(oracle_mod):
    """Per-head decode equals the last row of the per-head training problem."""
    P = rand_problem(13, B=1, T=40, Hq=4, Hkv=2, K=2)
    g = torch.Generator().manual_seed(113)
    sh = torch.randn(P["B"], P["Hq"], P["T"], P["s"].shape[-1], generator=g)
    desc = desc_of(oracle_mod, P)
    of, _ = oracle_mod.fwd_per_head(desc, P["q"].numpy(), P["k"].numpy(), P["v"].numpy(), sh.numpy())
    N = P["T"]
    dd = desc_of(oracle_mod, P, seq_len=1, q_offset=N - 1)
    od = oracle_mod.decode_per_head(dd, P["q"][:, :, N - 1].numpy(), P["k"].numpy(), P["v"].numpy(),
                                    sh[:, :, N - 1:N].numpy())
    np.testing.assert_allclose(od, of.reshape(P["B"], P["Hq"], N, P["d"])[:, :, N - 1], atol=1e-12, rtol=0)
