"""ctypes binding of libsas (include/sas.h), one Python function per C entry point.

Argument marshalling only: each function checks that the torch tensors it is
given live on the GPU, are contiguous and have the expected dtype, then passes
their device pointers and the current CUDA stream to the C function of the same
name and raises SasError on a non-OK status. All computation happens in the
library's CUDA kernels; there is no other implementation behind these names.
"""
from __future__ import annotations

import ctypes
import os

import torch

from .build import LIB

SAS_OK, SAS_ERR_INVALID_ARG, SAS_ERR_UNSUPPORTED, SAS_ERR_MISALIGNED, SAS_ERR_WORKSPACE, SAS_ERR_CUDA = range(6)
SAS_DT_BF16, SAS_DT_FP32 = 0, 1
SAS_GATE_SOFTMAX, SAS_GATE_NONE, SAS_GATE_SIGMOID, SAS_GATE_RAW, SAS_GATE_SOFTMAX_SELECTED, SAS_GATE_STE = range(6)
GATES = {"softmax": SAS_GATE_SOFTMAX, "none": SAS_GATE_NONE, "sigmoid": SAS_GATE_SIGMOID, "raw": SAS_GATE_RAW,
         "softmax_selected": SAS_GATE_SOFTMAX_SELECTED, "ste": SAS_GATE_STE}
SAS_OP_TOPK, SAS_OP_FWD, SAS_OP_BWD, SAS_OP_DECODE = range(4)


class SasError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn}: {sas_status_string(status)} (status {status})")
        self.status = status


class sas_desc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("seq_len", ctypes.c_int32), ("q_offset", ctypes.c_int32),
                ("n_q_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("block_size", ctypes.c_int32), ("top_k", ctypes.c_int32), ("softmax_scale", ctypes.c_float),
                ("dtype", ctypes.c_int32), ("gate", ctypes.c_int32), ("select_heads", ctypes.c_int32)]

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def n_sel_groups(self) -> int:
        """Rows of the selection arrays per (batch, query position): the KV
        heads, or the query heads when every query head selects its own blocks."""
        return self.n_q_heads if self.select_heads else self.n_kv_heads

    @property
    def n_blocks(self) -> int:
        return -(-(self.q_offset + self.seq_len) // self.block_size)

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == SAS_DT_FP32 else torch.bfloat16


def make_desc(batch, seq_len, n_q_heads, n_kv_heads, head_dim, block_size, top_k, q_offset=0,
              softmax_scale=0.0, dtype="bf16", gate="softmax", select_heads=False) -> sas_desc:
    dt = {"bf16": SAS_DT_BF16, "fp32": SAS_DT_FP32}[dtype] if isinstance(dtype, str) else int(dtype)
    gt = GATES[gate] if isinstance(gate, str) else int(gate)
    return sas_desc(batch, seq_len, q_offset, n_q_heads, n_kv_heads, head_dim, block_size, top_k,
                    softmax_scale, dt, gt, 1 if select_heads else 0)


_lib = None


def lib() -> ctypes.CDLL:
    """Load libsas.so; raises if it has not been built (there is no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB):
            raise RuntimeError(f"libsas.so not found at {LIB}: build it with "
                               "`python -m trainable_block_sparse_topk_b200.build`")
        L = ctypes.CDLL(LIB)
        P, D = ctypes.c_void_p, ctypes.POINTER(sas_desc)
        L.sas_workspace_size.argtypes = [ctypes.c_int32, D, ctypes.POINTER(ctypes.c_size_t)]
        L.sas_block_topk.argtypes = [D, P, P, P, P, P, P]
        L.sas_gated_attn_fwd.argtypes = [D, P, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]
        L.sas_gated_attn_bwd.argtypes = [D, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]
        L.sas_sparse_decode.argtypes = [D, P, P, P, ctypes.c_int64, P, P, P, P, P, ctypes.c_size_t, P]
        L.sas_sparse_decode_noalloc.argtypes = [D, P, P, P, ctypes.c_int64, P, P, P, P, P]
        L.sas_sparse_decode_paged.argtypes = [D, P, P, P, ctypes.c_int32, P, ctypes.c_int32, P, P, P, P, P, P,
                                              ctypes.c_size_t, P]
        L.sas_block_topk_varlen.argtypes = [D, P, P, P, P, P, P, P]
        L.sas_block_scores_pooled.argtypes = [D, P, P, ctypes.c_int64, P, P]
        L.sas_sparse_decode_pooled.argtypes = [D, P, P, P, ctypes.c_int64, P, ctypes.c_int64, P, P, P, P, P, P, P,
                                               ctypes.c_size_t, P]
        L.sas_status_string.argtypes = [ctypes.c_int]
        L.sas_status_string.restype = ctypes.c_char_p
        L.sas_device_timeouts.argtypes = [ctypes.POINTER(ctypes.c_uint32)]
        L.sas_kernel_launches.argtypes = []
        L.sas_kernel_launches.restype = ctypes.c_uint64
        L.sas_set_wait_limit.argtypes = [ctypes.c_uint64]
        L.sas_kernel_timing.argtypes = [ctypes.c_char_p]
        L.sas_kernel_time.argtypes = [ctypes.c_char_p, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_uint32)]
        for f in ("sas_workspace_size", "sas_block_topk", "sas_gated_attn_fwd", "sas_gated_attn_bwd",
                  "sas_sparse_decode", "sas_sparse_decode_noalloc", "sas_sparse_decode_paged",
                  "sas_block_topk_varlen", "sas_block_scores_pooled", "sas_sparse_decode_pooled",
                  "sas_device_timeouts", "sas_set_wait_limit",
                  "sas_kernel_timing", "sas_kernel_time"):
            getattr(L, f).restype = ctypes.c_int
        _lib = L
    return _lib


def _dev(t: torch.Tensor | None, name: str, dtype=None):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(fn: str, st: int) -> None:
    if st != SAS_OK:
        raise SasError(fn, st)


def sas_status_string(status: int) -> str:
    return lib().sas_status_string(int(status)).decode()


def sas_workspace_size(op: int, desc: sas_desc) -> int:
    n = ctypes.c_size_t(0)
    _check("sas_workspace_size", lib().sas_workspace_size(int(op), ctypes.byref(desc), ctypes.byref(n)))
    return int(n.value)


def sas_block_topk(desc, scores, idx, gate_logit, score_lse, n_sel, stream=None) -> None:
    f32, i32 = torch.float32, torch.int32
    _check("sas_block_topk", lib().sas_block_topk(
        ctypes.byref(desc), _dev(scores, "scores", f32), _dev(idx, "idx", i32),
        _dev(gate_logit, "gate_logit", f32), _dev(score_lse, "score_lse", f32), _dev(n_sel, "n_sel", i32),
        _stream(stream)))


def sas_gated_attn_fwd(desc, q, k, v, idx, gate_logit, n_sel, o, attn_lse, ws, stream=None) -> None:
    dt, f32, i32 = desc.torch_dtype, torch.float32, torch.int32
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check("sas_gated_attn_fwd", lib().sas_gated_attn_fwd(
        ctypes.byref(desc), _dev(q, "q", dt), _dev(k, "k", dt), _dev(v, "v", dt), _dev(idx, "idx", i32),
        _dev(gate_logit, "gate_logit", f32), _dev(n_sel, "n_sel", i32), _dev(o, "o", dt),
        _dev(attn_lse, "attn_lse", f32), _dev(ws, "ws"), nbytes, _stream(stream)))


def sas_gated_attn_bwd(desc, q, k, v, o, dO, attn_lse, scores, score_lse, idx, gate_logit, n_sel,
                       dq, dk, dv, dscores, ws, stream=None) -> None:
    dt, f32, i32 = desc.torch_dtype, torch.float32, torch.int32
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check("sas_gated_attn_bwd", lib().sas_gated_attn_bwd(
        ctypes.byref(desc), _dev(q, "q", dt), _dev(k, "k", dt), _dev(v, "v", dt), _dev(o, "o", dt),
        _dev(dO, "dO", dt), _dev(attn_lse, "attn_lse", f32), _dev(scores, "scores", f32),
        _dev(score_lse, "score_lse", f32), _dev(idx, "idx", i32), _dev(gate_logit, "gate_logit", f32),
        _dev(n_sel, "n_sel", i32), _dev(dq, "dq", dt), _dev(dk, "dk", dt), _dev(dv, "dv", dt),
        _dev(dscores, "dscores", f32), _dev(ws, "ws"), nbytes, _stream(stream)))


def sas_sparse_decode(desc, q, k_cache, v_cache, cache_stride_tokens, idx, gate_logit, n_sel, o, ws,
                      stream=None) -> None:
    dt, f32, i32 = desc.torch_dtype, torch.float32, torch.int32
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check("sas_sparse_decode", lib().sas_sparse_decode(
        ctypes.byref(desc), _dev(q, "q", dt), _dev(k_cache, "k_cache", dt), _dev(v_cache, "v_cache", dt),
        int(cache_stride_tokens), _dev(idx, "idx", i32), _dev(gate_logit, "gate_logit", f32),
        _dev(n_sel, "n_sel", i32), _dev(o, "o", dt), _dev(ws, "ws"), nbytes, _stream(stream)))


def sas_block_topk_varlen(desc, scores, seq_lens, idx, gate_logit, score_lse, n_sel, stream=None) -> None:
    f32, i32 = torch.float32, torch.int32
    _check("sas_block_topk_varlen", lib().sas_block_topk_varlen(
        ctypes.byref(desc), _dev(scores, "scores", f32), _dev(seq_lens, "seq_lens", i32), _dev(idx, "idx", i32),
        _dev(gate_logit, "gate_logit", f32), _dev(score_lse, "score_lse", f32), _dev(n_sel, "n_sel", i32),
        _stream(stream)))


def sas_sparse_decode_paged(desc, q, k_pages, v_pages, block_table, seq_lens, idx, gate_logit, n_sel, o, ws,
                            stream=None) -> None:
    """Decode over page pools [num_pages, Hkv, block, d] through block_table
    [B, max_blocks] (int32) with per-sequence lengths seq_lens [B] (int32)."""
    dt, f32, i32 = desc.torch_dtype, torch.float32, torch.int32
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check("sas_sparse_decode_paged", lib().sas_sparse_decode_paged(
        ctypes.byref(desc), _dev(q, "q", dt), _dev(k_pages, "k_pages", dt), _dev(v_pages, "v_pages", dt),
        int(k_pages.shape[0]), _dev(block_table, "block_table", i32), int(block_table.shape[1]),
        _dev(seq_lens, "seq_lens", i32), _dev(idx, "idx", i32), _dev(gate_logit, "gate_logit", f32),
        _dev(n_sel, "n_sel", i32), _dev(o, "o", dt), _dev(ws, "ws"), nbytes, _stream(stream)))


def sas_block_scores_pooled(desc, q, kbar, scores, stream=None) -> None:
    """Pooled-key block scores of the decode rows: kbar [B, Hkv, S, d] bf16."""
    _check("sas_block_scores_pooled", lib().sas_block_scores_pooled(
        ctypes.byref(desc), _dev(q, "q", torch.bfloat16), _dev(kbar, "kbar", torch.bfloat16), int(kbar.shape[2]),
        _dev(scores, "scores", torch.float32), _stream(stream)))


def sas_sparse_decode_pooled(desc, q, k_cache, v_cache, cache_stride_tokens, kbar, scores, idx, gate_logit,
                             score_lse, n_sel, o, ws, stream=None) -> None:
    """Pooled-key scores, top-K and sparse decode in one call."""
    dt, f32, i32 = desc.torch_dtype, torch.float32, torch.int32
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check("sas_sparse_decode_pooled", lib().sas_sparse_decode_pooled(
        ctypes.byref(desc), _dev(q, "q", dt), _dev(k_cache, "k_cache", dt), _dev(v_cache, "v_cache", dt),
        int(cache_stride_tokens), _dev(kbar, "kbar", dt), int(kbar.shape[2]), _dev(scores, "scores", f32),
        _dev(idx, "idx", i32), _dev(gate_logit, "gate_logit", f32), _dev(score_lse, "score_lse", f32),
        _dev(n_sel, "n_sel", i32), _dev(o, "o", dt), _dev(ws, "ws"), nbytes, _stream(stream)))


def sas_sparse_decode_noalloc(desc, q, k_cache, v_cache, cache_stride_tokens, idx, gate_logit, n_sel, o,
                              stream=None) -> None:
    """sas_sparse_decode without a workspace: the library's static scratch
    array holds the split partials (see include/sas.h)."""
    dt, f32, i32 = desc.torch_dtype, torch.float32, torch.int32
    _check("sas_sparse_decode_noalloc", lib().sas_sparse_decode_noalloc(
        ctypes.byref(desc), _dev(q, "q", dt), _dev(k_cache, "k_cache", dt), _dev(v_cache, "v_cache", dt),
        int(cache_stride_tokens), _dev(idx, "idx", i32), _dev(gate_logit, "gate_logit", f32),
        _dev(n_sel, "n_sel", i32), _dev(o, "o", dt), _stream(stream)))


def sas_device_timeouts() -> int:
    c = ctypes.c_uint32(0)
    _check("sas_device_timeouts", lib().sas_device_timeouts(ctypes.byref(c)))
    return int(c.value)


def sas_set_wait_limit(ns: int) -> None:
    """Bound (ns) on every device-side wait of the library's kernels; 0
    restores the default of 1 s."""
    _check("sas_set_wait_limit", lib().sas_set_wait_limit(int(ns)))


def sas_kernel_launches() -> int:
    return int(lib().sas_kernel_launches())


def sas_kernel_timing(names: str | None) -> None:
    """Record per-kernel CUDA events for the comma-separated kernel names
    ("*" for every kernel); None stops recording."""
    _check("sas_kernel_timing", lib().sas_kernel_timing(None if names is None else names.encode()))


def sas_kernel_time(kernel: str) -> tuple[float, int]:
    """(summed device ms, launches) recorded for `kernel` while timing was on."""
    ms = ctypes.c_double(0.0)
    n = ctypes.c_uint32(0)
    _check("sas_kernel_time", lib().sas_kernel_time(kernel.encode(), ctypes.byref(ms), ctypes.byref(n)))
    return float(ms.value), int(n.value)
