"""Boundary tests that need no GPU: libsas builds, loads, exports every symbol
include/sas.h declares, sizes workspaces, and rejects bad arguments before any
CUDA call (every call below fails validation, so no kernel is launched and no
fake pointer is ever dereferenced)."""
import ctypes
import os
import re

import pytest

from trainable_block_sparse_topk_b200 import binding as B
from trainable_block_sparse_topk_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build()
    return B.lib()


def declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"^\s*(?:const\s+)?\w+\*?\s+\**(sas_\w+)\s*\(", text, flags=re.M))
    return sorted(names)


def test_exports_every_declared_symbol(L):
    names = declared_symbols()
    assert {"sas_block_topk", "sas_gated_attn_fwd", "sas_gated_attn_bwd", "sas_sparse_decode",
            "sas_workspace_size", "sas_status_string"} <= set(names)
    for n in names:
        assert hasattr(L, n), n


def test_status_strings(L):
    for st in range(6):
        s = B.sas_status_string(st)
        assert isinstance(s, str) and s
    assert B.sas_status_string(99) == "unknown status"


def desc(**kw):
    base = dict(batch=1, seq_len=256, n_q_heads=8, n_kv_heads=2, head_dim=128, block_size=64, top_k=3)
    base.update(kw)
    return B.make_desc(**base)


def ws_size(op, d):
    n = ctypes.c_size_t(0)
    st = B.lib().sas_workspace_size(op, ctypes.byref(d), ctypes.byref(n))
    return st, n.value


def test_workspace_sizes(L):
    d = desc()
    assert ws_size(B.SAS_OP_TOPK, d) == (0, 0)
    st, n = ws_size(B.SAS_OP_BWD, d)
    assert st == 0
    # per-block token streams: capacity B*Hkv*T*(K+1) entries of 16 bytes plus
    # rvs per-head row values (rounded up to 16 bytes), per-block first entry
    # and count, per-(block, query tile) running counts and the allocation
    # counter; each piece 256-byte aligned
    NB, nT = 4, 4
    cap = 1 * 2 * 256 * (3 + 1)
    a = lambda p: (p + 255) // 256 * 256
    stream = lambda rvs: a(16 * cap) + a(4 * cap * rvs) + 2 * a(4 * 2 * NB) + a(4 * 2 * NB * nT) + 256
    # backward: column bitmap + D + Gsum + fp32 dq accumulator, then the
    # streams with the lse and D of each of the G = 4 heads (rvs 8), then the
    # 256-byte flag a CTA sets when it gives up on a wait
    parts = [8 * 1 * 2 * NB * nT, 4 * 8 * 256, 4 * 2 * 256 * 3, 4 * 8 * 256 * 128]
    assert n == sum(a(p) for p in parts) + a(stream(8)) + 256
    # forward (tensor-core shapes): column bitmap, then per query-head row the
    # shift, flagged-row list, l and the fp32 output accumulator plus the
    # flagged-row count, then the streams with the shift of each head (rvs 4)
    rows = 8 * 256
    head = a(12 * rows + 4 * rows * 128 + 16)
    assert ws_size(B.SAS_OP_FWD, d) == (0, a(8 * 1 * 2 * NB * nT) + a(head + stream(4)))
    st, n32 = ws_size(B.SAS_OP_BWD, desc(dtype="fp32"))
    assert st == 0 and n32 < n            # fp32 accumulates dq in place
    dd = desc(seq_len=1, q_offset=4095)
    st, nd = ws_size(B.SAS_OP_DECODE, dd)
    assert st == 0 and nd > 0 and nd % 256 == 0
    assert ws_size(B.SAS_OP_DECODE, desc())[0] == B.SAS_ERR_INVALID_ARG   # decode needs seq_len 1
    assert ws_size(7, d)[0] == B.SAS_ERR_INVALID_ARG


@pytest.mark.parametrize("kw,status", [
    (dict(n_q_heads=6, n_kv_heads=4), B.SAS_ERR_INVALID_ARG),
    (dict(batch=0), B.SAS_ERR_INVALID_ARG),
    (dict(top_k=0), B.SAS_ERR_INVALID_ARG),
    (dict(dtype=7), B.SAS_ERR_INVALID_ARG),
    (dict(gate=6), B.SAS_ERR_INVALID_ARG),
    (dict(softmax_scale=float("nan")), B.SAS_ERR_INVALID_ARG),
    (dict(head_dim=96), B.SAS_ERR_UNSUPPORTED),
    (dict(block_size=16), B.SAS_ERR_UNSUPPORTED),
    (dict(top_k=65), B.SAS_ERR_UNSUPPORTED),
    (dict(n_q_heads=18, n_kv_heads=2), B.SAS_ERR_UNSUPPORTED),
    (dict(seq_len=200), B.SAS_ERR_UNSUPPORTED),          # training needs T % b == 0
    (dict(q_offset=64), B.SAS_ERR_UNSUPPORTED),          # training needs q_offset == 0
])
def test_bad_descriptors_rejected(L, kw, status):
    assert ws_size(B.SAS_OP_FWD, desc(**kw))[0] == status


FAKE = 0x10000      # 16-byte aligned, never dereferenced: validation fails first
ODD = 0x10004


def P(x):
    return ctypes.c_void_p(x)


def call_topk(d, scores=FAKE, idx=FAKE, gl=FAKE, lse=FAKE, nsel=FAKE):
    return B.lib().sas_block_topk(ctypes.byref(d), P(scores), P(idx), P(gl), P(lse), P(nsel), P(0))


def test_topk_rejects_before_launch(L):
    d = desc()
    assert call_topk(d, scores=None) == B.SAS_ERR_INVALID_ARG
    assert call_topk(d, nsel=None) == B.SAS_ERR_INVALID_ARG
    assert call_topk(d, idx=ODD) == B.SAS_ERR_MISALIGNED
    assert call_topk(desc(head_dim=80)) == B.SAS_ERR_UNSUPPORTED
    assert B.lib().sas_block_topk(None, P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(0)) == B.SAS_ERR_INVALID_ARG
    # decode rows beyond the longest supported row length
    assert call_topk(desc(seq_len=1, q_offset=64 * 8193 + 5)) == B.SAS_ERR_UNSUPPORTED


def test_fwd_rejects_before_launch(L):
    d = desc()
    f = B.lib().sas_gated_attn_fwd
    args = [P(FAKE)] * 8
    assert f(ctypes.byref(d), *args[:3], None, *args[4:], P(0), 0, P(0)) == B.SAS_ERR_INVALID_ARG
    bad = list(args)
    bad[7] = P(ODD)
    assert f(ctypes.byref(d), *bad, P(0), 0, P(0)) == B.SAS_ERR_MISALIGNED
    assert f(ctypes.byref(desc(seq_len=100)), *args, P(0), 0, P(0)) == B.SAS_ERR_UNSUPPORTED


def test_bwd_rejects_before_launch(L):
    d = desc()
    f = B.lib().sas_gated_attn_bwd
    args = [P(FAKE)] * 15
    st, need = ws_size(B.SAS_OP_BWD, d)
    assert need > 0
    assert f(ctypes.byref(d), *args, None, 0, P(0)) == B.SAS_ERR_WORKSPACE
    assert f(ctypes.byref(d), *args, P(FAKE), need - 1, P(0)) == B.SAS_ERR_WORKSPACE
    assert f(ctypes.byref(d), *args, P(ODD), need, P(0)) == B.SAS_ERR_MISALIGNED
    bad = list(args)
    bad[14] = None
    assert f(ctypes.byref(d), *bad, P(FAKE), need, P(0)) == B.SAS_ERR_INVALID_ARG


def test_decode_rejects_before_launch(L):
    d = desc(seq_len=1, q_offset=1000)
    f = B.lib().sas_sparse_decode
    st, need = ws_size(B.SAS_OP_DECODE, d)
    ok = [P(FAKE)] * 3
    # cache stride shorter than N = q_offset + 1
    assert f(ctypes.byref(d), *ok, 1000, P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE), need, P(0)) == \
        B.SAS_ERR_INVALID_ARG
    # selection given without its gate / count
    assert f(ctypes.byref(d), *ok, 1001, P(FAKE), None, P(FAKE), P(FAKE), P(FAKE), need, P(0)) == \
        B.SAS_ERR_INVALID_ARG
    assert f(ctypes.byref(d), *ok, 1001, None, None, None, P(FAKE), P(FAKE), need - 256, P(0)) == \
        B.SAS_ERR_WORKSPACE
    assert f(ctypes.byref(d), P(ODD), P(FAKE), P(FAKE), 1001, None, None, None, P(FAKE), P(FAKE), need, P(0)) == \
        B.SAS_ERR_MISALIGNED
    assert f(ctypes.byref(desc(seq_len=2, q_offset=5)), *ok, 1001, None, None, None, P(FAKE), P(FAKE), need,
             P(0)) == B.SAS_ERR_INVALID_ARG


def test_binding_refuses_host_tensors(L):
    import torch
    d = desc()
    s = torch.zeros(1, 2, 256, 4)
    with pytest.raises(ValueError):
        B.sas_block_topk(d, s, s, s, s, s)


def test_kernel_timing_records_nothing_without_launches(L):
    assert B.sas_kernel_timing("*") is None
    assert B.sas_kernel_time("bwd_tc") == (0.0, 0)
    assert B.sas_kernel_timing(None) is None
    ms, n = ctypes.c_double(1.0), ctypes.c_uint32(7)
    assert L.sas_kernel_time(None, ctypes.byref(ms), ctypes.byref(n)) == B.SAS_ERR_INVALID_ARG
    assert L.sas_kernel_time(b"fwd_rows", None, ctypes.byref(n)) == B.SAS_ERR_INVALID_ARG


def test_select_heads_value_checked(L):
    d = desc()
    d.select_heads = 2            # neither 0 nor 1
    assert ws_size(B.SAS_OP_FWD, d)[0] == B.SAS_ERR_INVALID_ARG


def test_per_head_selection_workspace(L):
    """Per-query-head selection: the selection arrays and streams have Hq rows
    per position, and the backward adds fp32 dK, dV per selection group (two
    B*Hq*T*d float arrays) for the sum over the heads of each KV head."""
    d0, d1 = desc(), desc(select_heads=1)
    a = lambda p: (p + 255) // 256 * 256
    st, n0 = ws_size(B.SAS_OP_BWD, d0)
    st1, n1 = ws_size(B.SAS_OP_BWD, d1)
    assert st == 0 and st1 == 0
    Bn, Hq, Hkv, T, K, D, NB, nT = 1, 8, 2, 256, 3, 128, 4, 4
    cap1 = Bn * Hq * T * (K + 1)
    stream1 = a(16 * cap1) + a(4 * cap1 * 4) + 2 * a(4 * Hq * NB) + a(4 * Hq * NB * nT) + 256
    parts = [8 * Bn * Hq * NB * nT, 4 * Bn * Hq * T, 4 * Bn * Hq * T * K, 4 * Bn * Hq * T * D]
    assert n1 == sum(a(p) for p in parts) + 2 * a(4 * Bn * Hq * T * D) + a(stream1) + 256
    assert n1 > n0
