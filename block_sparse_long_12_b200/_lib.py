"""ctypes binding of libmsa.so (include/msa.h): argument marshalling only.

Every entry point of the C ABI is exposed under its own name and takes torch
tensors (for their device pointers) plus a ``Params`` structure; the work
itself runs in the library's CUDA kernels.  There is no fallback: if the
library is missing or the call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmsa.so")

MSA_OK, MSA_ERR_INVALID_ARG, MSA_ERR_UNSUPPORTED, MSA_ERR_WORKSPACE, MSA_ERR_CUDA, MSA_ERR_TIMEOUT = range(6)
MSA_F32, MSA_BF16 = 0, 1
MSA_SCORES_TOKEN, MSA_SCORES_BLOCKMAX, MSA_DENSE, MSA_FORCE_SINK_LOCAL = 1, 2, 8, 16
MSA_IDX_PLAIN, MSA_IDX_MXFP8 = 0, 1
(MSA_ENTRY_INDEX_SCORE, MSA_ENTRY_MAXPOOL_TOPK, MSA_ENTRY_ATTN_DECODE, MSA_ENTRY_ATTN_PREFILL,
 MSA_ENTRY_DECODE_FUSED, MSA_ENTRY_PREFILL_INDEX_TOPK) = range(6)

# every symbol include/msa.h declares
EXPORTED = ["msa_index_score", "msa_block_maxpool_topk", "msa_sparse_attn_decode", "msa_sparse_attn_prefill",
            "msa_decode_fused", "msa_prefill_index_topk", "msa_workspace_size", "msa_last_error_string",
            "msa_status_string", "msa_get_device_status", "msa_clear_device_status", "msa_set_stage_events",
            "msa_decode_fused_noalloc", "msa_noalloc_get_status", "msa_noalloc_clear_status", "msa_set_wait_limit",
            "msa_diag_wait_timeout", "msa_decode_append", "msa_quantize_index_k"]


class MsaError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"status {status}: {message}")
        self.status = status


class Params(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int), ("n_q_heads", ctypes.c_int), ("n_kv_heads", ctypes.c_int),
        ("n_idx_k_heads", ctypes.c_int), ("head_dim", ctypes.c_int), ("idx_dim", ctypes.c_int),
        ("block_size", ctypes.c_int), ("top_k", ctypes.c_int), ("q_len", ctypes.c_int), ("q_start", ctypes.c_int),
        ("max_seq_len", ctypes.c_int), ("seq_lens", ctypes.c_void_p), ("softmax_scale", ctypes.c_float),
        ("dtype", ctypes.c_int), ("flags", ctypes.c_int), ("block_table", ctypes.c_void_p), ("n_pages", ctypes.c_int),
        ("idx_format", ctypes.c_int), ("k_idx_scale", ctypes.c_void_p),
    ]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m block_sparse_long_12_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.POINTER(Params)
        vp, sz, st = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p
        sig = {
            "msa_index_score": [P, vp, vp, vp, vp, sz, st],
            "msa_block_maxpool_topk": [P, vp, vp, vp, vp, sz, st],
            "msa_sparse_attn_decode": [P, vp, vp, vp, vp, vp, vp, vp, sz, st],
            "msa_sparse_attn_prefill": [P, vp, vp, vp, vp, vp, vp, vp, sz, st],
            "msa_decode_fused": [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, st],
            "msa_decode_fused_noalloc": [P, vp, vp, vp, vp, vp, vp, vp, vp, st],
            "msa_prefill_index_topk": [P, vp, vp, vp, vp, vp, sz, st],
            "msa_get_device_status": [vp, ctypes.POINTER(ctypes.c_int), st],
            "msa_clear_device_status": [vp, st],
            "msa_set_stage_events": [ctypes.POINTER(ctypes.c_void_p), ctypes.c_int],
            "msa_noalloc_get_status": [ctypes.POINTER(ctypes.c_int), st],
            "msa_noalloc_clear_status": [st],
            "msa_set_wait_limit": [vp, ctypes.c_uint64, st],
            "msa_diag_wait_timeout": [vp, sz, st],
            "msa_decode_append": [P, vp, vp, vp, vp, vp, vp, st],
            "msa_quantize_index_k": [P, vp, ctypes.c_longlong, vp, vp, st],
        }
        for name, args in sig.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = ctypes.c_int
        L.msa_workspace_size.argtypes = [P, ctypes.c_int]
        L.msa_workspace_size.restype = ctypes.c_size_t
        L.msa_last_error_string.argtypes = []
        L.msa_last_error_string.restype = ctypes.c_char_p
        L.msa_status_string.argtypes = [ctypes.c_int]
        L.msa_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int):
    if status != MSA_OK:
        raise MsaError(status, lib().msa_last_error_string().decode())


def msa_workspace_size(params: Params, entry: int) -> int:
    n = lib().msa_workspace_size(ctypes.byref(params), entry)
    if n == ctypes.c_size_t(-1).value:
        raise MsaError(MSA_ERR_INVALID_ARG, lib().msa_last_error_string().decode())
    return n


def msa_index_score(params, q_idx, k_idx, scores_out, ws, stream=None):
    _check(lib().msa_index_score(ctypes.byref(params), _ptr(q_idx), _ptr(k_idx), _ptr(scores_out), _ptr(ws),
                                 ws.numel() if ws is not None else 0, _stream(stream)))


def msa_block_maxpool_topk(params, scores_in, ids_out, top_scores_out, ws, stream=None):
    _check(lib().msa_block_maxpool_topk(ctypes.byref(params), _ptr(scores_in), _ptr(ids_out), _ptr(top_scores_out),
                                        _ptr(ws), ws.numel() if ws is not None else 0, _stream(stream)))


def msa_sparse_attn_decode(params, q, k_cache, v_cache, ids, o, lse, ws, stream=None):
    _check(lib().msa_sparse_attn_decode(ctypes.byref(params), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(ids),
                                        _ptr(o), _ptr(lse), _ptr(ws), ws.numel() if ws is not None else 0,
                                        _stream(stream)))


def msa_sparse_attn_prefill(params, q, k_cache, v_cache, ids, o, lse, ws, stream=None):
    _check(lib().msa_sparse_attn_prefill(ctypes.byref(params), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(ids),
                                         _ptr(o), _ptr(lse), _ptr(ws), ws.numel() if ws is not None else 0,
                                         _stream(stream)))


def msa_decode_fused(params, q, q_idx, k_cache, v_cache, k_idx, o, ids_out, lse, ws, stream=None):
    _check(lib().msa_decode_fused(ctypes.byref(params), _ptr(q), _ptr(q_idx), _ptr(k_cache), _ptr(v_cache),
                                  _ptr(k_idx), _ptr(o), _ptr(ids_out), _ptr(lse), _ptr(ws),
                                  ws.numel() if ws is not None else 0, _stream(stream)))


def msa_decode_fused_noalloc(params, q, q_idx, k_cache, v_cache, k_idx, o, ids_out, lse, stream=None):
    """msa_decode_fused without a workspace argument: scratch comes from the library's fixed device array."""
    _check(lib().msa_decode_fused_noalloc(ctypes.byref(params), _ptr(q), _ptr(q_idx), _ptr(k_cache), _ptr(v_cache),
                                          _ptr(k_idx), _ptr(o), _ptr(ids_out), _ptr(lse), _stream(stream)))


def msa_prefill_index_topk(params, q_idx, k_idx, ids_out, top_scores_out, ws, stream=None):
    _check(lib().msa_prefill_index_topk(ctypes.byref(params), _ptr(q_idx), _ptr(k_idx), _ptr(ids_out),
                                        _ptr(top_scores_out), _ptr(ws), ws.numel() if ws is not None else 0,
                                        _stream(stream)))


def msa_get_device_status(ws, stream=None) -> int:
    out = ctypes.c_int(0)
    _check(lib().msa_get_device_status(_ptr(ws), ctypes.byref(out), _stream(stream)))
    return out.value


def msa_clear_device_status(ws, stream=None):
    _check(lib().msa_clear_device_status(_ptr(ws), _stream(stream)))


def msa_set_stage_events(events):
    """events: a list of 3 recorded-once torch.cuda.Event, or None to unset."""
    if not events:
        _check(lib().msa_set_stage_events(None, 0))
        return
    arr = (ctypes.c_void_p * 3)(*[e.cuda_event for e in events])
    _check(lib().msa_set_stage_events(arr, 3))


def msa_noalloc_get_status(stream=None) -> int:
    out = ctypes.c_int(0)
    _check(lib().msa_noalloc_get_status(ctypes.byref(out), _stream(stream)))
    return out.value


def msa_noalloc_clear_status(stream=None):
    _check(lib().msa_noalloc_clear_status(_stream(stream)))


def msa_set_wait_limit(ws, limit_ns: int, stream=None):
    _check(lib().msa_set_wait_limit(_ptr(ws), int(limit_ns), _stream(stream)))


def msa_diag_wait_timeout(ws, stream=None):
    _check(lib().msa_diag_wait_timeout(_ptr(ws), ws.numel() if ws is not None else 0, _stream(stream)))


def msa_decode_append(params, k_new, v_new, k_idx_new, k_cache, v_cache, k_idx, stream=None):
    _check(lib().msa_decode_append(ctypes.byref(params), _ptr(k_new), _ptr(v_new), _ptr(k_idx_new), _ptr(k_cache),
                                   _ptr(v_cache), _ptr(k_idx), _stream(stream)))


def msa_quantize_index_k(params, src, rows, codes, scales, stream=None):
    _check(lib().msa_quantize_index_k(ctypes.byref(params), _ptr(src), int(rows), _ptr(codes), _ptr(scales),
                                      _stream(stream)))
