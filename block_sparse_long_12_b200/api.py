"""Tensor-level convenience over the C ABI.

These helpers only derive shapes from torch tensors, allocate outputs and
workspace with torch, and call the library entry points of ``_lib``; every
step of MSA itself runs in the CUDA kernels of libmsa.so.
"""
from __future__ import annotations

import math

import torch

from . import _lib
from ._lib import (MSA_BF16, MSA_DENSE, MSA_ENTRY_ATTN_DECODE, MSA_ENTRY_ATTN_PREFILL, MSA_ENTRY_DECODE_FUSED,
                   MSA_ENTRY_INDEX_SCORE, MSA_ENTRY_MAXPOOL_TOPK, MSA_ENTRY_PREFILL_INDEX_TOPK, MSA_F32,
                   MSA_FORCE_SINK_LOCAL, MSA_SCORES_BLOCKMAX, MSA_SCORES_TOKEN, Params)


def dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return MSA_F32
    if t.dtype == torch.bfloat16:
        return MSA_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def make_params(*, batch, n_q_heads, n_kv_heads, n_idx_k_heads, head_dim, idx_dim, block_size, top_k,
                max_seq_len, dtype, q_len=1, q_start=0, seq_lens=None, softmax_scale=None, flags=0,
                block_table=None, n_pages=0, k_idx_scale=None) -> Params:
    """block_table (int32 [B, ceil(max_seq_len / block_size)], device) selects paged caches of n_pages pages;
    k_idx_scale (uint8 E8M0 scales, one per 32 index dims) selects MXFP8 index keys."""
    return Params(batch, n_q_heads, n_kv_heads, n_idx_k_heads, head_dim, idx_dim, block_size, top_k, q_len,
                  q_start, max_seq_len, seq_lens.data_ptr() if seq_lens is not None else None,
                  float(softmax_scale if softmax_scale is not None else 1.0 / math.sqrt(head_dim)), dtype, flags,
                  block_table.data_ptr() if block_table is not None else None, int(n_pages),
                  _lib.MSA_IDX_MXFP8 if k_idx_scale is not None else _lib.MSA_IDX_PLAIN,
                  k_idx_scale.data_ptr() if k_idx_scale is not None else None)


def quantize_index_k(k_idx: torch.Tensor, stream=None) -> tuple[torch.Tensor, torch.Tensor]:
    """MXFP8 copy of a bf16 index-key tensor [..., di]: (codes uint8 [..., di], scales uint8 [..., di / 32])."""
    di = k_idx.shape[-1]
    rows = k_idx.numel() // di
    codes = torch.empty(k_idx.shape, dtype=torch.uint8, device=k_idx.device)
    scales = torch.empty(k_idx.shape[:-1] + (di // 32,), dtype=torch.uint8, device=k_idx.device)
    p = make_params(batch=1, n_q_heads=1, n_kv_heads=1, n_idx_k_heads=1, head_dim=64, idx_dim=di, block_size=16,
                    top_k=1, max_seq_len=16, dtype=_lib.MSA_BF16)
    _lib.msa_quantize_index_k(p, k_idx.contiguous(), rows, codes, scales, stream)
    return codes, scales


def params_from(q, q_idx, k, k_idx, *, block_size, top_k, seq_lens=None, q_start=0, softmax_scale=None,
                flags=0, k_idx_scale=None) -> Params:
    """Params for q [B, Tq, Hq, D], q_idx [B, Tq, G, di], k [B, G, L, D], k_idx [B, Hik, L, di] (bf16, or
    MXFP8 codes with their scales k_idx_scale [B, Hik, L, di / 32])."""
    B, Tq, Hq, D = q.shape
    _, G, L, _ = k.shape
    return make_params(batch=B, n_q_heads=Hq, n_kv_heads=G, n_idx_k_heads=k_idx.shape[1], head_dim=D,
                       idx_dim=q_idx.shape[-1], block_size=block_size, top_k=top_k, max_seq_len=L,
                       dtype=dtype_code(q), q_len=Tq, q_start=q_start, seq_lens=seq_lens,
                       softmax_scale=softmax_scale, flags=flags, k_idx_scale=k_idx_scale)


def workspace(params, entry: int, device) -> torch.Tensor:
    """Zeroed scratch for one entry (the first word is the device status).  `params` may be
    a list: the scratch then serves every call made with any of them."""
    plist = params if isinstance(params, (list, tuple)) else [params]
    n = max(_lib.msa_workspace_size(p, entry) for p in plist)
    return torch.zeros(max(n, 256), dtype=torch.uint8, device=device)


def decode(q, q_idx, k, v, k_idx, seq_lens, *, block_size, top_k, softmax_scale=None, ws=None, out=None,
           stream=None, force_sink_local=False, k_idx_scale=None):
    """One fused MSA decode step.  Returns (o [B,1,Hq,D], ids [B,1,G,k], lse [B,1,Hq]).
    force_sink_local: the selection always keeps block 0 and the query's own block.
    k_idx_scale: k_idx holds MXFP8 codes with these scales (quantize_index_k)."""
    p = params_from(q, q_idx, k, k_idx, block_size=block_size, top_k=top_k, seq_lens=seq_lens,
                    softmax_scale=softmax_scale, flags=MSA_FORCE_SINK_LOCAL if force_sink_local else 0,
                    k_idx_scale=k_idx_scale)
    B, _, Hq, D = q.shape
    G = k.shape[1]
    if ws is None:
        ws = workspace(p, MSA_ENTRY_DECODE_FUSED, q.device)
    if out is None:
        out = (torch.empty_like(q), torch.empty(B, 1, G, top_k, dtype=torch.int32, device=q.device),
               torch.empty(B, 1, Hq, dtype=torch.float32, device=q.device))
    o, ids, lse = out
    _lib.msa_decode_fused(p, q, q_idx, k, v, k_idx, o, ids, lse, ws, stream)
    return o, ids, lse


def attend_decode(q, k, v, ids, seq_lens, *, block_size, top_k, dense=False, softmax_scale=None, ws=None,
                  stream=None):
    """Sparse (or, with dense=True, full GQA) decode attention.  Returns (o, lse)."""
    B, _, Hq, D = q.shape
    G, L = k.shape[1], k.shape[2]
    p = make_params(batch=B, n_q_heads=Hq, n_kv_heads=G, n_idx_k_heads=G, head_dim=D,
                    idx_dim=64 if q.dtype == torch.bfloat16 else 32, block_size=block_size, top_k=top_k,
                    max_seq_len=L, dtype=dtype_code(q), seq_lens=seq_lens, softmax_scale=softmax_scale,
                    flags=MSA_DENSE if dense else 0)
    if ws is None:
        ws = workspace(p, MSA_ENTRY_ATTN_DECODE, q.device)
    o = torch.empty_like(q)
    lse = torch.empty(B, 1, Hq, dtype=torch.float32, device=q.device)
    _lib.msa_sparse_attn_decode(p, q, k, v, None if dense else ids, o, lse, ws, stream)
    return o, lse


def index_scores(q_idx, k_idx, seq_lens, *, n_kv_heads, block_size, top_k=1, mode="block", stream=None):
    """Stored decode index scores: token [B,1,G,L] or block-max [B,1,G,nb] fp32."""
    B, Tq, G, di = q_idx.shape
    L = k_idx.shape[2]
    p = make_params(batch=B, n_q_heads=G, n_kv_heads=G, n_idx_k_heads=k_idx.shape[1], head_dim=64, idx_dim=di,
                    block_size=block_size, top_k=top_k, max_seq_len=L, dtype=dtype_code(q_idx), q_len=Tq,
                    seq_lens=seq_lens, flags=MSA_SCORES_TOKEN if mode == "token" else MSA_SCORES_BLOCKMAX)
    n = L if mode == "token" else -(-L // block_size)
    out = torch.empty(B, Tq, G, n, dtype=torch.float32, device=q_idx.device)
    ws = workspace(p, MSA_ENTRY_INDEX_SCORE, q_idx.device)
    _lib.msa_index_score(p, q_idx, k_idx, out, ws, stream)
    return out


def pool_topk(scores, seq_lens, *, block_size, top_k, max_seq_len, is_block, q_start=0, stream=None,
              force_sink_local=False):
    """Block max pool + TopK of stored scores [B, Tq, G, n].  Returns (ids, top_scores)."""
    B, Tq, G, _ = scores.shape
    p = make_params(batch=B, n_q_heads=G, n_kv_heads=G, n_idx_k_heads=G, head_dim=64, idx_dim=32,
                    block_size=block_size, top_k=top_k, max_seq_len=max_seq_len, dtype=MSA_F32, q_len=Tq,
                    q_start=q_start, seq_lens=seq_lens,
                    flags=(MSA_SCORES_BLOCKMAX if is_block else 0) | (MSA_FORCE_SINK_LOCAL if force_sink_local else 0))
    ids = torch.empty(B, Tq, G, top_k, dtype=torch.int32, device=scores.device)
    ts = torch.empty(B, Tq, G, top_k, dtype=torch.float32, device=scores.device)
    ws = workspace(p, MSA_ENTRY_MAXPOOL_TOPK, scores.device)
    _lib.msa_block_maxpool_topk(p, scores, ids, ts, ws, stream)
    return ids, ts
