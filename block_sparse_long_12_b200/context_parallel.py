"""Context-parallel MSA decode: one step across ranks that each hold a slice of the context.

Every rank holds the same contiguous, block-aligned slice [start, start + length) of every
sequence's K, V and index-K cache (its own caches, contiguous, [B, H, length, row]).  One decode
step (page "MiniMax wird duenn", atlascloud.ai, section 1, Steps 1 and 2) then runs as:

1. Index branch, locally: each rank scores the blocks of its slice and keeps its local TopK
   (k best blocks per (sequence, group), higher score first, ties to the lower block id), with
   block ids made global by adding the slice's first block.
2. Exchange: the ranks all-gather their k (score, id) candidates per (sequence, group); every
   rank then keeps the k best of the gathered candidates in the same order.  The result is the
   selection a single rank would make over the whole context: a block among the global k best is
   among the k best of the slice that holds it.
3. Sparse branch, locally: each rank attends the selected blocks it holds and returns, per query
   head, its output normalised over those keys and its log-sum-exp (a rank holding none gives
   log-sum-exp -inf and a zero output).
4. Exchange: the ranks all-gather their (output, log-sum-exp) partials, and every rank merges
   them by log-sum-exp into the full output.

The two exchanges move k * (4 + 4) bytes per (sequence, group) and (D + 1) * 4 bytes per
(sequence, head) per rank: a few hundred kilobytes per step at most.  Transport is
torch.distributed (NCCL between GPUs, gloo on CPU ranks); nothing here issues a peer load.

The local steps come from a backend object with two calls:

* ``block_topk(q_idx, k_idx, lens, k) -> (scores [B, G, k], ids [B, G, k])`` over the slice,
  local ids with -1 padding and -inf scores for missing blocks;
* ``attend(q, k, v, lens, ids) -> (o [B, Hq, D], lse [B, Hq])`` over the listed local blocks
  (-1 entries skipped), lse the natural-log normaliser.

``LibraryBackend`` runs them in the CUDA library (msa_index_score with block-max scores,
msa_block_maxpool_topk, msa_sparse_attn_decode); the merges below are a handful of element-wise
tensor operations on the gathered candidates and partials.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist


@dataclass(frozen=True)
class Slice:
    """A rank's part of the context: tokens [start, start + length), start a multiple of the block size."""
    start: int
    length: int

    def local_lens(self, lens: torch.Tensor) -> torch.Tensor:
        """Tokens of each sequence (cached lengths `lens`) that fall in this slice."""
        return (lens.to(torch.int64) - self.start).clamp(0, self.length).to(torch.int32)


def slices_of(max_seq_len: int, block_size: int, world: int) -> list[Slice]:
    """The context cut into `world` slices of whole blocks, as equal as the blocks allow."""
    nb = -(-max_seq_len // block_size)
    out, b0 = [], 0
    for r in range(world):
        b1 = nb * (r + 1) // world
        start, end = b0 * block_size, min(b1 * block_size, max_seq_len)
        out.append(Slice(start, max(end - start, 0)))
        b0 = b1
    return out


def select_global_topk(scores: torch.Tensor, ids: torch.Tensor, k: int) -> tuple[torch.Tensor, torch.Tensor]:
    """The k best of gathered candidates scores/ids [R, B, G, k] (global ids, -1 for none) in the
    TopK order: higher score first, then lower block id.  Returns (scores, ids) [B, G, k]."""
    R, B, G, kk = scores.shape
    s = scores.permute(1, 2, 0, 3).reshape(B, G, R * kk)
    i = ids.permute(1, 2, 0, 3).reshape(B, G, R * kk).to(torch.int64)
    s = torch.where(i >= 0, s, torch.full_like(s, float("-inf")))
    big = torch.iinfo(torch.int64).max
    # stable sort by id ascending, then stable sort by score descending keeps ties in id order
    order = torch.argsort(torch.where(i >= 0, i, torch.full_like(i, big)), dim=-1, stable=True)
    s, i = torch.gather(s, -1, order), torch.gather(i, -1, order)
    order = torch.argsort(-s, dim=-1, stable=True)
    s, i = torch.gather(s, -1, order)[..., :k], torch.gather(i, -1, order)[..., :k]
    i = torch.where(s > float("-inf"), i, torch.full_like(i, -1))
    return s, i.to(torch.int32)


def local_ids_of(global_ids: torch.Tensor, sl: Slice, block_size: int) -> torch.Tensor:
    """The selected blocks this slice holds, in its own numbering; -1 elsewhere."""
    b0 = sl.start // block_size
    nb = -(-sl.length // block_size)
    g = global_ids.to(torch.int64)
    held = (g >= b0) & (g < b0 + nb)
    return torch.where(held, g - b0, torch.full_like(g, -1)).to(torch.int32)


def merge_partials(o: torch.Tensor, lse: torch.Tensor) -> tuple[torch.Tensor, torch.Tensor]:
    """Log-sum-exp merge of per-rank partials o [R, B, Hq, D] (each normalised over its keys) and
    lse [R, B, Hq]: o = sum_r exp(lse_r - lse) o_r with lse = log sum_r exp(lse_r)."""
    m = lse.max(dim=0).values
    finite = torch.isfinite(m)
    m_safe = torch.where(finite, m, torch.zeros_like(m))
    w = torch.exp(lse - m_safe.unsqueeze(0))
    w = torch.where(torch.isfinite(lse), w, torch.zeros_like(w))
    den = w.sum(dim=0)
    out = (w.unsqueeze(-1) * o.to(w.dtype)).sum(dim=0) / torch.where(den > 0, den, torch.ones_like(den)).unsqueeze(-1)
    lse_out = torch.where(den > 0, m_safe + torch.log(torch.where(den > 0, den, torch.ones_like(den))),
                          torch.full_like(den, float("-inf")))
    return out, lse_out


def _all_gather(x: torch.Tensor, group=None) -> torch.Tensor:
    world = dist.get_world_size(group)
    out = [torch.empty_like(x) for _ in range(world)]
    dist.all_gather(out, x.contiguous(), group=group)
    return torch.stack(out)


def local_candidates(backend, q_idx, k_idx, lens, sl: Slice, *, block_size: int, top_k: int):
    """Step 1 on one slice: its k best blocks per (sequence, group) as (scores, global ids) [B, G, k]."""
    s_loc, i_loc = backend.block_topk(q_idx, k_idx, sl.local_lens(lens), top_k)
    b0 = sl.start // block_size
    return s_loc.to(torch.float64), torch.where(i_loc >= 0, i_loc + b0, i_loc).to(torch.int32)


def local_partial(backend, q, k, v, lens, sl: Slice, ids, *, block_size: int):
    """Step 2 on one slice: the partial (o, lse) over the selected blocks it holds."""
    o, lse = backend.attend(q, k, v, sl.local_lens(lens), local_ids_of(ids, sl, block_size))
    return o, lse.to(torch.float64)


def decode_step(backend, q, q_idx, k, v, k_idx, lens, sl: Slice, *, block_size: int, top_k: int, group=None):
    """One context-parallel decode step on this rank (every rank of `group` calls it with its own
    slice and the same queries).  q [B, 1, Hq, D], q_idx [B, 1, G, di]; k, v [B, G, sl.length, D]
    and k_idx [B, Hik, sl.length, di] are this rank's slice; lens [B] the whole cached lengths.
    Returns (o [B, Hq, D], lse [B, Hq], ids [B, G, k]) -- the same on every rank."""
    s_loc, i_loc = local_candidates(backend, q_idx, k_idx, lens, sl, block_size=block_size, top_k=top_k)
    _, ids = select_global_topk(_all_gather(s_loc, group), _all_gather(i_loc, group), top_k)
    o_loc, lse_loc = local_partial(backend, q, k, v, lens, sl, ids, block_size=block_size)
    o, lse = merge_partials(_all_gather(o_loc, group), _all_gather(lse_loc, group))
    return o, lse, ids


class LibraryBackend:
    """The local steps in the CUDA library (device tensors)."""

    def __init__(self, n_q_heads: int, block_size: int, softmax_scale: float | None = None):
        self.n_q_heads = n_q_heads
        self.block_size = block_size
        self.softmax_scale = softmax_scale

    def _params(self, q_idx, k_idx, lens, k, *, L, flags, head_dim):
        from . import api
        B, _, G, di = q_idx.shape
        return api.make_params(batch=B, n_q_heads=self.n_q_heads, n_kv_heads=G, n_idx_k_heads=k_idx.shape[1],
                               head_dim=head_dim, idx_dim=di, block_size=self.block_size, top_k=k,
                               max_seq_len=L, dtype=api.dtype_code(q_idx), seq_lens=lens, flags=flags,
                               softmax_scale=self.softmax_scale)

    def block_topk(self, q_idx, k_idx, lens, k):
        from . import _lib, api
        B, _, G, _ = q_idx.shape
        L = k_idx.shape[2]
        nb = -(-L // self.block_size)
        # Step 1 over the slice: block-max scores, then the slice's TopK of them
        p = self._params(q_idx, k_idx, lens, k, L=L, flags=_lib.MSA_SCORES_BLOCKMAX, head_dim=64)
        blk = torch.empty(B, 1, G, nb, dtype=torch.float32, device=q_idx.device)
        ws = api.workspace(p, _lib.MSA_ENTRY_INDEX_SCORE, q_idx.device)
        _lib.msa_index_score(p, q_idx, k_idx, blk, ws)
        ids = torch.empty(B, 1, G, k, dtype=torch.int32, device=q_idx.device)
        sc = torch.empty(B, 1, G, k, dtype=torch.float32, device=q_idx.device)
        ws2 = api.workspace(p, _lib.MSA_ENTRY_MAXPOOL_TOPK, q_idx.device)
        _lib.msa_block_maxpool_topk(p, blk, ids, sc, ws2)
        empty = (lens <= 0).view(B, 1, 1)  # a slice the sequence does not reach holds no block
        ids = torch.where(empty, torch.full_like(ids[:, 0], -1), ids[:, 0])
        sc = torch.where(empty, torch.full_like(sc[:, 0], float("-inf")), sc[:, 0])
        return sc, ids

    def attend(self, q, k, v, lens, ids):
        from . import _lib, api
        B, _, Hq, D = q.shape
        G, L = k.shape[1], k.shape[2]
        kk = ids.shape[-1]
        p = api.make_params(batch=B, n_q_heads=Hq, n_kv_heads=G, n_idx_k_heads=G, head_dim=D,
                            idx_dim=64 if q.dtype == torch.bfloat16 else 32, block_size=self.block_size, top_k=kk,
                            max_seq_len=L, dtype=api.dtype_code(q), seq_lens=lens.clamp(min=1),
                            softmax_scale=self.softmax_scale)
        ws = api.workspace(p, _lib.MSA_ENTRY_ATTN_DECODE, q.device)
        o = torch.empty_like(q)
        lse = torch.empty(B, 1, Hq, dtype=torch.float32, device=q.device)
        _lib.msa_sparse_attn_decode(p, q, k, v, ids.view(B, 1, G, kk).contiguous(), o, lse, ws)
        return o[:, 0].float(), lse[:, 0]
