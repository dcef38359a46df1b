"""Second, independent NumPy formulation of MSA, used only to cross-check the C oracle.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).  It is written
differently on purpose so that a slip in one is unlikely to be repeated in
the other:

* token scores: one matrix-vector product in float64;
* block max pool: pad the visible scores to whole blocks with -inf, reshape,
  take the row maximum ("Block Max Pool", page "MiniMax wird duenn", section 1,
  Step 1);
* TopK: rank counting -- block n is kept iff fewer than k blocks beat it in the
  order (higher score, then lower id); no sort is used;
* attention: a boolean key mask built from the selected block ids, then a
  masked softmax (section 1, Step 2: every head of the group uses the same
  list; contiguous grouping Q1..Q3 -> I1, Q4..Q6 -> I2).
"""
from __future__ import annotations

import numpy as np

from . import to_f64


def token_scores(q_idx_row: np.ndarray, k_idx_head: np.ndarray, pos: int) -> np.ndarray:
    """s = K_idx[0..pos] @ q_idx  (both already float64)."""
    return k_idx_head[: pos + 1] @ q_idx_row


def block_scores(s: np.ndarray, block_size: int) -> np.ndarray:
    nb = -(-len(s) // block_size)
    padded = np.full(nb * block_size, -np.inf)
    padded[: len(s)] = s
    return padded.reshape(nb, block_size).max(axis=1)


def rank_of(S: np.ndarray) -> np.ndarray:
    """rank[n] = #{m : S_m > S_n or (S_m == S_n and m < n)}."""
    n = np.arange(len(S))
    beats = (S[None, :] > S[:, None]) | ((S[None, :] == S[:, None]) & (n[None, :] < n[:, None]))
    return beats.sum(axis=1)


def topk(S: np.ndarray, k: int, force_sink_local: bool = False) -> np.ndarray:
    """Ids of the k best blocks in order, padded with -1.  With ``force_sink_local`` the first
    block (the sink) and the last one (the query's own) are raised to +inf before ranking."""
    if force_sink_local and len(S):
        S = S.copy()
        S[[0, -1]] = np.inf
    rank = rank_of(S)
    ids = np.full(k, -1, np.int32)
    for n in np.nonzero(rank < k)[0]:
        ids[rank[n]] = n
    return ids


def attention(q_h: np.ndarray, K: np.ndarray, V: np.ndarray, ids: np.ndarray, pos: int,
              block_size: int, scale: float):
    """Masked softmax over keys 0..pos whose block is in ``ids``.  Returns (o, lse, w)."""
    keys = np.arange(pos + 1)
    chosen = np.zeros(pos // block_size + 1, bool)
    chosen[ids[ids >= 0]] = True
    mask = chosen[keys // block_size]
    z = np.where(mask, scale * (K[: pos + 1] @ q_h), -np.inf)
    m = z.max()
    e = np.exp(z - m)
    w = e / e.sum()
    return w @ V[: pos + 1], m + np.log(e.sum()), w


def msa_row(cfg: dict, q, q_idx, k, v, k_idx, b: int, t: int, pos: int, dense: bool = False):
    """Whole MSA for one query row: returns (ids[G, k], o[Hq, D], lse[Hq])."""
    Hq, Hkv, Hik = cfg["n_q_heads"], cfg["n_kv_heads"], cfg["n_idx_k_heads"]
    r = Hq // Hkv
    qf, qif, kf, vf, kif = (to_f64(x) for x in (q, q_idx, k, v, k_idx))
    ids_all, o_all, lse_all = [], [], []
    for g in range(Hkv):
        s = token_scores(qif[b, t, g], kif[b, g % Hik], pos)
        S = block_scores(s, cfg["block_size"])
        ids = topk(S, cfg["top_k"], cfg.get("force_sink_local", False))
        ids_all.append(ids)
        use = np.arange(len(S), dtype=np.int32) if dense else ids
        for h in range(g * r, (g + 1) * r):
            o, lse, _ = attention(qf[b, t, h], kf[b, g], vf[b, g], use, pos, cfg["block_size"], cfg["softmax_scale"])
            o_all.append(o)
            lse_all.append(lse)
    return np.stack(ids_all), np.stack(o_all), np.array(lse_all)
