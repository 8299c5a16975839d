"""Bounded device-side waits (failure detection without a GPU fault).

Every wait of a kernel for another agent's work (a copy, an MMA, another
role's warps) has a bound. With the bound set far below a copy's latency
(1 ns), the waits give up on purpose: the call must still return, count the
event in sas_device_timeouts(), and leave NaN in its outputs rather than stale
or partial numbers; with the default bound restored, the same calls on the
same CUDA context are correct again (checked against the oracle)."""
import numpy as np
import pytest
import torch

import oracle
from tests import gpu_util as U
from trainable_block_sparse_topk_b200 import api, binding as B, synth
from trainable_block_sparse_topk_b200.build import build

pytestmark = pytest.mark.gpu

TOL_BF16_O = 1e-2
TOL_BF16_GRAD = 2e-2


@pytest.fixture
def short_waits():
    build()
    oracle.build()
    B.sas_set_wait_limit(1)
    try:
        yield
    finally:
        B.sas_set_wait_limit(0)


def _decode_case():
    N, K = 4133, 7
    gen = torch.Generator().manual_seed(91)
    kc = (0.5 * torch.randn(2, 2, N, 128, generator=gen)).to(torch.bfloat16)
    vc = (0.5 * torch.randn(2, 2, N, 128, generator=gen)).to(torch.bfloat16)
    q = (0.5 * torch.randn(2, 8, 128, generator=gen)).to(torch.bfloat16)
    s = torch.randn(2, 2, 1, -(-N // 64), generator=gen)
    d = B.make_desc(batch=2, seq_len=1, q_offset=N - 1, n_q_heads=8, n_kv_heads=2, head_dim=128, block_size=64,
                    top_k=K)
    od = oracle.Desc(batch=2, seq_len=1, q_offset=N - 1, n_q_heads=8, n_kv_heads=2, head_dim=128, block_size=64,
                     top_k=K)
    ref = oracle.decode(od, q.float().numpy(), kc.float().numpy(), vc.float().numpy(), s.numpy())
    return d, kc.cuda(), vc.cuda(), q.cuda(), s.cuda(), ref


def test_decode_gives_up_then_recovers(short_waits):
    d, kc, vc, q, s, ref = _decode_case()
    sel = api.block_topk(d, s)
    t0 = B.sas_device_timeouts()
    out = api.sparse_decode(d, q, kc, vc, sel)
    torch.cuda.synchronize()
    assert B.sas_device_timeouts() > t0
    got = out.float().cpu().numpy()
    assert np.isnan(got).any()
    fin = ~np.isnan(got)            # groups whose CTAs all finished are still exact
    assert np.abs(got[fin] - ref[fin]).max(initial=0.0) <= TOL_BF16_O
    B.sas_set_wait_limit(0)
    t1 = B.sas_device_timeouts()
    out = api.sparse_decode(d, q, kc, vc, sel)
    torch.cuda.synchronize()
    assert B.sas_device_timeouts() == t1
    assert np.abs(out.float().cpu().numpy() - ref).max() <= TOL_BF16_O


def test_training_gives_up_then_recovers(short_waits):
    """The gathered-row forward and backward (bf16, d 128, block 64, G = 5)."""
    w = synth.Workload("mid", "train", 1, 1024, 10, 2, 128, 64, 5, "bf16", 21, 0.5, score_noise=0.1)
    x = synth.train_inputs(w)
    t0 = B.sas_device_timeouts()
    _, bad = U.run_train(w, inputs=x)
    assert B.sas_device_timeouts() > t0
    for name in ("o", "lse", "dq", "ds"):
        assert torch.isnan(bad[name].float()).all(), name
    B.sas_set_wait_limit(0)
    t1 = B.sas_device_timeouts()
    _, out = U.run_train(w, inputs=x)
    assert B.sas_device_timeouts() == t1
    G = w.group
    for g in range(w.n_kv_heads):
        d = U.group_desc(w)
        a = U.group_arrays(x, w, 0, g)
        o, _ = oracle.fwd(d, a["q"], a["k"], a["v"], a["s"])
        assert np.abs(out["o"][0, g * G:(g + 1) * G].float().numpy().transpose(1, 0, 2) - o).max() <= TOL_BF16_O
        r = oracle.bwd(d, a["q"], a["k"], a["v"], a["s"], a["dO"])
        got = {"dq": out["dq"][0, g * G:(g + 1) * G].float().numpy().transpose(1, 0, 2),
               "dk": out["dk"][:, g:g + 1].float().numpy(), "dv": out["dv"][:, g:g + 1].float().numpy(),
               "ds": out["ds"][0, g].numpy()}
        for key, val in got.items():
            assert U.normwise(val, r[key]) <= TOL_BF16_GRAD, key
