"""Pins for the CPU oracle (no GPU).

The oracle is checked against things other than itself: the worked examples
in tests/golden (cited there), brute force on tiny inputs, closed forms
(uniform weights when q = 0, a single visible key, projection onto a unit
index query), a textbook routine (torch's fp64 scaled_dot_product_attention
with GQA, dense and with a key mask), and invariants stated by the page
"MiniMax wird duenn" (atlascloud.ai), section 1 (Step 1: index score ->
block max pool -> TopK per group; Step 2: the group's heads share one list
and attend over the real K/V of the selected blocks).

Every pin runs against both formulations (C oracle, NumPy twin) and against a
set of deliberately broken copies of the twin, each of which some pin must
reject.
"""
from __future__ import annotations

import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from oracle import numpy_twin as tw

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------------
# implementations under test
# --------------------------------------------------------------------------

def _pos(cfg, x, b, t):
    return cfg["q_start"] + t if cfg["prefill"] else int(x["seq_lens"][b]) - 1


class COracle:
    name = "c_oracle"

    def params(self, cfg, dense=False):
        return oracle.Params(cfg["batch"], cfg["n_q_heads"], cfg["n_kv_heads"], cfg["n_idx_k_heads"],
                             cfg["head_dim"], cfg["idx_dim"], cfg["block_size"], cfg["top_k"], cfg["q_len"],
                             cfg["q_start"], cfg["max_seq_len"], cfg["dtype"], cfg["softmax_scale"],
                             prefill=cfg["prefill"], dense=dense,
                             force_sink_local=cfg.get("force_sink_local", False))

    def token_scores(self, cfg, x, b, t, g, pos):
        return oracle.token_scores(self.params(cfg), x["q_idx"], x["k_idx"], b, t, g, pos)

    def block_scores(self, cfg, s, pos):
        return oracle.block_scores(self.params(cfg), s, pos)

    def topk(self, cfg, S):
        return oracle.topk(self.params(cfg), S)[0]

    def row(self, cfg, x, b, t, dense=False):
        r = oracle.msa_rows(self.params(cfg, dense), x["seq_lens"], x["q"], x["q_idx"], x["k"], x["v"],
                            x["k_idx"], [(b, t)])
        return r["ids"][0], r["o"][0], r["lse"][0]


class Twin:
    """NumPy twin, split into overridable steps so that broken copies can be made."""
    name = "numpy_twin"

    def group_of(self, h, cfg):
        return h // (cfg["n_q_heads"] // cfg["n_kv_heads"])

    def token_scores(self, cfg, x, b, t, g, pos):
        qi = oracle.to_f64(x["q_idx"])[b, t, g]
        ki = oracle.to_f64(x["k_idx"])[b, g % cfg["n_idx_k_heads"]]
        return tw.token_scores(qi, ki, pos)

    def block_scores(self, cfg, s, pos):
        return tw.block_scores(s[: pos + 1], cfg["block_size"])

    def topk(self, cfg, S):
        return tw.topk(S, cfg["top_k"], cfg.get("force_sink_local", False))

    def attend(self, cfg, qh, K, V, ids, pos):
        return tw.attention(qh, K, V, ids, pos, cfg["block_size"], cfg["softmax_scale"])

    def row(self, cfg, x, b, t, dense=False):
        pos = _pos(cfg, x, b, t)
        G, Hq = cfg["n_kv_heads"], cfg["n_q_heads"]
        qf, kf, vf = (oracle.to_f64(x[n]) for n in ("q", "k", "v"))
        ids = np.stack([self.topk(cfg, self.block_scores(cfg, self.token_scores(cfg, x, b, t, g, pos), pos))
                        for g in range(G)])
        o, lse = [], []
        for h in range(Hq):
            g = self.group_of(h, cfg)
            use = np.arange(pos // cfg["block_size"] + 1, dtype=np.int32) if dense else ids[g]
            oh, lh, _ = self.attend(cfg, qf[b, t, h], kf[b, g], vf[b, g], use, pos)
            o.append(oh)
            lse.append(lh)
        return ids, np.stack(o), np.array(lse)


# broken copies: each plants one plausible mistake
class MutGroupModulo(Twin):
    name = "mut_group_modulo"

    def group_of(self, h, cfg):
        return h % cfg["n_kv_heads"]


class MutTieHigherId(Twin):
    name = "mut_tie_higher_id"

    def topk(self, cfg, S):
        n = len(S)
        order = sorted(range(n), key=lambda i: (-S[i], -i))[: cfg["top_k"]]
        return np.array(order + [-1] * (cfg["top_k"] - len(order)), np.int32)


class MutPoolSeesFuture(Twin):
    name = "mut_pool_sees_future"

    def token_scores(self, cfg, x, b, t, g, pos):
        qi = oracle.to_f64(x["q_idx"])[b, t, g]
        ki = oracle.to_f64(x["k_idx"])[b, g % cfg["n_idx_k_heads"]]
        return ki @ qi  # every cached token, including those after pos

    def block_scores(self, cfg, s, pos):
        bk = cfg["block_size"]
        nb = pos // bk + 1
        return np.array([s[n * bk:(n + 1) * bk].max() for n in range(nb)])


class MutMeanPool(Twin):
    name = "mut_mean_pool"

    def block_scores(self, cfg, s, pos):
        bk = cfg["block_size"]
        s = s[: pos + 1]
        return np.array([s[n * bk:(n + 1) * bk].mean() for n in range(-(-len(s) // bk))])


class MutNoScale(Twin):
    name = "mut_no_softmax_scale"

    def attend(self, cfg, qh, K, V, ids, pos):
        return tw.attention(qh, K, V, ids, pos, cfg["block_size"], 1.0)


class MutAttendFuture(Twin):
    name = "mut_attend_future_in_block"

    def attend(self, cfg, qh, K, V, ids, pos):
        bk = cfg["block_size"]
        last = min(K.shape[0] - 1, (pos // bk + 1) * bk - 1)
        return tw.attention(qh, K, V, ids, last, bk, cfg["softmax_scale"])


class MutDropIndexDim(Twin):
    name = "mut_drop_last_index_dim"

    def token_scores(self, cfg, x, b, t, g, pos):
        qi = oracle.to_f64(x["q_idx"])[b, t, g][:-1]
        ki = oracle.to_f64(x["k_idx"])[b, g % cfg["n_idx_k_heads"]][:, :-1]
        return tw.token_scores(qi, ki, pos)


class MutIndexHeadOfGroupZero(Twin):
    name = "mut_index_head_always_0"

    def token_scores(self, cfg, x, b, t, g, pos):
        qi = oracle.to_f64(x["q_idx"])[b, t, g]
        ki = oracle.to_f64(x["k_idx"])[b, 0]
        return tw.token_scores(qi, ki, pos)


class MutForcedLocalIsPrevious(Twin):
    name = "mut_forced_local_is_previous_block"

    def topk(self, cfg, S):
        if cfg.get("force_sink_local", False) and len(S):
            S = S.copy()
            S[[0, max(len(S) - 2, 0)]] = np.inf
        return tw.topk(S, cfg["top_k"])


class MutForcedKeepRealScoreOrder(Twin):
    name = "mut_forced_blocks_ranked_by_score"

    def topk(self, cfg, S):
        if not (cfg.get("force_sink_local", False) and len(S)):
            return tw.topk(S, cfg["top_k"])
        forced = sorted({0, len(S) - 1}, key=lambda n: (-S[n], n))
        rest = [n for n in tw.topk(S, len(S)) if n not in forced]
        out = (forced + rest)[: cfg["top_k"]]
        return np.array(out + [-1] * (cfg["top_k"] - len(out)), np.int32)


GOOD = [COracle(), Twin()]
MUTANTS = [MutGroupModulo(), MutTieHigherId(), MutPoolSeesFuture(), MutMeanPool(), MutNoScale(),
           MutAttendFuture(), MutDropIndexDim(), MutIndexHeadOfGroupZero(), MutForcedLocalIsPrevious(),
           MutForcedKeepRealScoreOrder()]


# --------------------------------------------------------------------------
# inputs
# --------------------------------------------------------------------------

def make_cfg(**kw):
    cfg = dict(batch=1, n_q_heads=4, n_kv_heads=2, n_idx_k_heads=2, head_dim=8, idx_dim=4, block_size=4,
               top_k=3, q_len=1, q_start=0, max_seq_len=32, dtype="f32", prefill=False)
    cfg.update(kw)
    cfg.setdefault("softmax_scale", 1.0 / math.sqrt(cfg["head_dim"]))
    return cfg


def rand_inputs(cfg, seed, seq_lens=None):
    rng = np.random.default_rng(seed)
    B, T, L = cfg["batch"], cfg["q_len"], cfg["max_seq_len"]

    def f(*shape):
        return rng.standard_normal(shape).astype(np.float32)
    x = dict(q=f(B, T, cfg["n_q_heads"], cfg["head_dim"]), q_idx=f(B, T, cfg["n_kv_heads"], cfg["idx_dim"]),
             k=f(B, cfg["n_kv_heads"], L, cfg["head_dim"]), v=f(B, cfg["n_kv_heads"], L, cfg["head_dim"]),
             k_idx=f(B, cfg["n_idx_k_heads"], L, cfg["idx_dim"]))
    x["seq_lens"] = np.array(seq_lens if seq_lens is not None else [L] * B, np.int32)
    return x


def rows_of(cfg, x):
    return [(b, t) for b in range(cfg["batch"]) for t in range(cfg["q_len"])]


# --------------------------------------------------------------------------
# pins (each returns None or raises AssertionError)
# --------------------------------------------------------------------------

def pin_golden_hand_worked(impl):
    gold = json.load(open(os.path.join(GOLDEN, "hand_worked_selection.json")))
    cfg = make_cfg(block_size=gold["block_size"], top_k=gold["top_k"])
    s = np.array(gold["token_scores"])
    S = impl.block_scores(cfg, s, gold["pos"])
    np.testing.assert_allclose(S, gold["block_scores"], rtol=0, atol=1e-15)
    assert list(impl.topk(cfg, S)) == gold["ids"]


def pin_topk_brute_force(impl):
    rng = np.random.default_rng(7)
    for trial in range(300):
        nb = int(rng.integers(1, 13))
        k = int(rng.integers(1, 5))
        # small integers force many exact ties
        S = rng.integers(-3, 4, nb).astype(np.float64) if trial % 2 else rng.standard_normal(nb)
        cfg = make_cfg(top_k=k)
        m = min(k, nb)
        best = max((sorted(((S[n], -n) for n in comb), reverse=True) for comb in itertools.combinations(range(nb), m)))
        want = [-neg for (_, neg) in best] + [-1] * (k - m)
        got = list(impl.topk(cfg, S))
        assert got == want, (S, k, got, want)


def pin_block_pool_properties(impl):
    rng = np.random.default_rng(11)
    for trial in range(50):
        bk = int(rng.integers(1, 6))
        L = int(rng.integers(1, 30))
        pos = int(rng.integers(0, L))
        s = rng.standard_normal(L)
        cfg = make_cfg(block_size=bk)
        S = impl.block_scores(cfg, s, pos)
        assert len(S) == pos // bk + 1
        for n in range(len(S)):
            vis = s[n * bk: min((n + 1) * bk, pos + 1)]
            assert np.all(S[n] >= vis) and np.any(S[n] == vis)
            # permuting the tokens inside a block leaves the pool unchanged
        perm = s.copy()
        for n in range(len(S)):
            lo, hi = n * bk, min((n + 1) * bk, pos + 1)
            perm[lo:hi] = rng.permutation(perm[lo:hi])
        np.testing.assert_array_equal(impl.block_scores(cfg, perm, pos), S)


def pin_index_score_projection(impl):
    """q_idx = unit vector e_d gives s_j = k_idx[j, d] exactly (closed form)."""
    cfg = make_cfg(idx_dim=5, max_seq_len=12)
    x = rand_inputs(cfg, 3)
    for d in range(cfg["idx_dim"]):
        for g in range(cfg["n_kv_heads"]):
            x["q_idx"][:] = 0
            x["q_idx"][0, 0, g, d] = 1.0
            s = impl.token_scores(cfg, x, 0, 0, g, 11)
            np.testing.assert_array_equal(s, x["k_idx"][0, g % cfg["n_idx_k_heads"], :12, d].astype(np.float64))


def pin_dense_equals_sdpa(impl):
    """With every block selected, MSA is plain GQA softmax attention."""
    for prefill in (False, True):
        for (Hq, Hkv) in ((4, 2), (6, 3)):
            cfg = make_cfg(n_q_heads=Hq, n_kv_heads=Hkv, n_idx_k_heads=Hkv, max_seq_len=24, block_size=4,
                           top_k=6, prefill=prefill, q_len=24 if prefill else 1, batch=2)
            x = rand_inputs(cfg, 5 + Hq, seq_lens=[24, 17])
            for b in range(2):
                L = int(x["seq_lens"][b])
                K = torch.from_numpy(oracle.to_f64(x["k"][b]))[:, :L]
                V = torch.from_numpy(oracle.to_f64(x["v"][b]))[:, :L]
                if prefill:
                    Q = torch.from_numpy(oracle.to_f64(x["q"][b]))[:L].transpose(0, 1)  # [Hq, T, D]
                    ref = F.scaled_dot_product_attention(Q[None], K[None], V[None], is_causal=True,
                                                         scale=cfg["softmax_scale"], enable_gqa=True)[0]
                    ts = [0, 3, 9, L - 1]
                else:
                    Q = torch.from_numpy(oracle.to_f64(x["q"][b, 0]))[:, None]  # [Hq, 1, D]
                    ref = F.scaled_dot_product_attention(Q[None], K[None], V[None], scale=cfg["softmax_scale"],
                                                         enable_gqa=True)[0]
                    ts = [0]
                for t in ts:
                    _, o, _ = impl.row(cfg, x, b, t, dense=True)
                    col = t if prefill else 0
                    np.testing.assert_allclose(o, ref[:, col].numpy(), rtol=0, atol=1e-12)
                    if (L - 1 if not prefill else t) // 4 + 1 <= cfg["top_k"]:
                        _, o2, _ = impl.row(cfg, x, b, t)  # k >= #valid blocks: sparse == dense
                        np.testing.assert_allclose(o2, o, rtol=0, atol=1e-12)


def pin_sparse_equals_masked_sdpa(impl):
    """Given the row's ids, Step 2 is SDPA with a key mask: keys of the group's selected blocks, j <= pos."""
    cfg = make_cfg(n_q_heads=6, n_kv_heads=2, n_idx_k_heads=2, max_seq_len=40, block_size=4, top_k=3,
                   prefill=True, q_len=40)
    x = rand_inputs(cfg, 21)
    r = cfg["n_q_heads"] // cfg["n_kv_heads"]
    for t in (5, 17, 39):
        ids, o, lse = impl.row(cfg, x, 0, t)
        mask = torch.zeros(cfg["n_q_heads"], 1, t + 1, dtype=torch.bool)
        for h in range(cfg["n_q_heads"]):
            for n in ids[h // r]:
                if n >= 0:
                    mask[h, 0, n * 4: min(n * 4 + 4, t + 1)] = True
        Q = torch.from_numpy(oracle.to_f64(x["q"][0, t]))[:, None]
        K = torch.from_numpy(oracle.to_f64(x["k"][0]))[:, : t + 1]
        V = torch.from_numpy(oracle.to_f64(x["v"][0]))[:, : t + 1]
        ref = F.scaled_dot_product_attention(Q[None], K[None], V[None], attn_mask=mask[None],
                                             scale=cfg["softmax_scale"], enable_gqa=True)[0, :, 0]
        np.testing.assert_allclose(o, ref.numpy(), rtol=0, atol=1e-12)


def pin_diagram_grouping(impl):
    """Heads Q1..Q3 attend only I1's blocks, Q4..Q6 only I2's (golden fixture)."""
    gold = json.load(open(os.path.join(GOLDEN, "diagram_grouping.json")))
    L = 24
    cfg = make_cfg(n_q_heads=gold["n_q_heads"], n_kv_heads=gold["n_index_queries"], n_idx_k_heads=1,
                   head_dim=L, idx_dim=4, max_seq_len=L, block_size=4, top_k=2)
    x = rand_inputs(cfg, 9)
    # V = identity per KV head: the output row of a head is its weight vector
    for g in range(2):
        x["v"][0, g] = np.eye(L, dtype=np.float32)
    # the two index queries point at different blocks of the one index-K head
    x["k_idx"][:] = 0
    x["k_idx"][0, 0, 0:4, 0] = 5.0      # block 0
    x["k_idx"][0, 0, 8:12, 0] = 4.0     # block 2
    x["k_idx"][0, 0, 16:20, 1] = 5.0    # block 4
    x["k_idx"][0, 0, 20:24, 1] = 4.0    # block 5
    x["q_idx"][:] = 0
    x["q_idx"][0, 0, 0, 0] = 1.0
    x["q_idx"][0, 0, 1, 1] = 1.0
    want_blocks = {0: {0, 2}, 1: {4, 5}}
    ids, o, _ = impl.row(cfg, x, 0, 0)
    assert set(ids[0].tolist()) == want_blocks[0] and set(ids[1].tolist()) == want_blocks[1]
    for h in range(gold["n_q_heads"]):
        lst = gold["list_of_head"][h]
        support = {j // 4 for j in np.nonzero(o[h] > 1e-300)[0]}
        assert support == want_blocks[lst], (h, support)
        assert abs(o[h].sum() - 1) < 1e-12 and np.all(o[h] >= 0)


def pin_uniform_when_query_zero(impl):
    """q = 0: all logits equal, so each head's output is the mean of V over the visible selected keys and LSE = log(n)."""
    L = 20
    cfg = make_cfg(n_q_heads=2, n_kv_heads=1, n_idx_k_heads=1, head_dim=L, max_seq_len=L, block_size=4,
                   top_k=2, prefill=True, q_len=L)
    x = rand_inputs(cfg, 13)
    x["q"][:] = 0
    x["v"][0, 0] = np.eye(L, dtype=np.float32)
    for t in (2, 9, 14, 19):
        ids, o, lse = impl.row(cfg, x, 0, t)
        keys = sorted(j for n in ids[0] if n >= 0 for j in range(n * 4, n * 4 + 4) if j <= t)
        want = np.zeros(L)
        want[keys] = 1.0 / len(keys)
        for h in range(2):
            np.testing.assert_allclose(o[h], want, rtol=0, atol=1e-15)
            assert abs(lse[h] - math.log(len(keys))) < 1e-12


def pin_single_key(impl):
    """k = 1, block 1, the first query of a causal chunk sees one key: O is that key's V row."""
    cfg = make_cfg(n_q_heads=2, n_kv_heads=1, n_idx_k_heads=1, block_size=1, top_k=1, prefill=True,
                   q_len=6, max_seq_len=6)
    x = rand_inputs(cfg, 17)
    ids, o, _ = impl.row(cfg, x, 0, 0)
    assert ids.tolist() == [[0]]
    for h in range(2):
        np.testing.assert_allclose(o[h], x["v"][0, 0, 0].astype(np.float64), rtol=0, atol=1e-15)


def pin_causality(impl):
    """Nothing at positions after pos (index keys, K or V) changes the row's result."""
    cfg = make_cfg(n_q_heads=4, n_kv_heads=2, n_idx_k_heads=2, max_seq_len=32, block_size=4, top_k=2,
                   prefill=True, q_len=32)
    x = rand_inputs(cfg, 19)
    for t in (5, 13, 22):
        ids, o, lse = impl.row(cfg, x, 0, t)
        y = {n: a.copy() for n, a in x.items()}
        for g in range(2):
            qn = y["q_idx"][0, t, g] / np.linalg.norm(y["q_idx"][0, t, g])
            y["k_idx"][0, g, t + 1:] = 100.0 * qn   # future tokens would win every block they touch
        y["k"][0, :, t + 1:] = 50.0
        y["v"][0, :, t + 1:] = -50.0
        ids2, o2, lse2 = impl.row(cfg, y, 0, t)
        np.testing.assert_array_equal(ids2, ids)
        np.testing.assert_allclose(o2, o, rtol=0, atol=1e-13)


def pin_selection_valid_and_scale_free(impl):
    """ids are causal-valid, unique, -1 only when fewer than k blocks exist; q_idx * c (c > 0) keeps them."""
    cfg = make_cfg(n_q_heads=4, n_kv_heads=2, n_idx_k_heads=2, max_seq_len=40, block_size=4, top_k=5,
                   prefill=True, q_len=40)
    x = rand_inputs(cfg, 23)
    y = {n: a.copy() for n, a in x.items()}
    y["q_idx"] = (y["q_idx"] * np.float32(2.0)).astype(np.float32)  # exact scaling
    for t in range(0, 40, 3):
        ids, _, _ = impl.row(cfg, x, 0, t)
        ids2, _, _ = impl.row(cfg, y, 0, t)
        np.testing.assert_array_equal(ids, ids2)
        nv = t // 4 + 1
        for g in range(2):
            sel = [n for n in ids[g] if n >= 0]
            assert len(sel) == min(nv, 5) and len(set(sel)) == len(sel)
            assert all(0 <= n <= t // 4 for n in sel)
            assert list(ids[g][len(sel):]) == [-1] * (5 - len(sel))


def pin_planted_hot_blocks(impl):
    """On planted data every selected block is hot when at least k hot blocks are visible."""
    from block_sparse_long_12_b200.inputs import WORKLOADS, make_inputs, to_numpy_raw
    w = WORKLOADS["decode_b8_ctx128k_ragged"].scaled(batch=2, max_seq_len=4096, min_seq_len=2048, block_size=64,
                                                     top_k=8, hot_blocks=12, n_q_heads=8, n_kv_heads=2,
                                                     n_idx_k_heads=2, head_dim=16, dtype="f32")
    t = make_inputs(w)
    x = {n: to_numpy_raw(t[n]) for n in ("q", "q_idx", "k", "v", "k_idx", "seq_lens")}
    cfg = make_cfg(batch=2, n_q_heads=8, n_kv_heads=2, n_idx_k_heads=2, head_dim=16, idx_dim=w.idx_dim,
                   block_size=64, top_k=8, max_seq_len=4096)
    for b in range(2):
        ids, _, _ = impl.row(cfg, x, b, 0)
        for g in range(2):
            hot = set(t["hot"][b, g].tolist()) - {-1}
            assert set(ids[g].tolist()) <= hot, (b, g, ids[g], hot)


def pin_forced_sink_local_brute_force(impl):
    """Forced blocks: block 0 and the last valid block (the query's own) come first, by id, then the
    best k - 2 of the other blocks by exhaustive search; with k = 1 the sink alone."""
    rng = np.random.default_rng(29)
    for trial in range(300):
        nb = int(rng.integers(1, 13))
        k = int(rng.integers(1, 6))
        S = rng.integers(-3, 4, nb).astype(np.float64) if trial % 2 else rng.standard_normal(nb)
        cfg = make_cfg(top_k=k, force_sink_local=True)
        forced = [0] if nb == 1 else [0, nb - 1]
        head = forced[:k]
        others = [n for n in range(nb) if n not in forced]
        m = min(k - len(head), len(others))
        best = max((sorted(((S[n], -n) for n in comb), reverse=True)
                    for comb in itertools.combinations(others, m)), default=[])
        want = head + [-neg for (_, neg) in best]
        want += [-1] * (k - len(want))
        got = list(impl.topk(cfg, S))
        assert got == want, (S, k, got, want)


def pin_forced_rows(impl):
    """On whole rows (decode and prefill) the forced flag keeps block 0 and block pos // Bk in every
    group's list, the list stays valid, and with k >= the valid blocks the output is the dense one."""
    for prefill in (False, True):
        cfg = make_cfg(n_q_heads=4, n_kv_heads=2, n_idx_k_heads=2, max_seq_len=40, block_size=4, top_k=4,
                       prefill=prefill, q_len=40 if prefill else 1, force_sink_local=True)
        x = rand_inputs(cfg, 31, seq_lens=[37])
        for t in ((0, 3, 4, 17, 36) if prefill else (0,)):
            pos = t if prefill else 36
            ids, o, _ = impl.row(cfg, x, 0, t)
            nv = pos // 4 + 1
            for g in range(2):
                sel = [n for n in ids[g] if n >= 0]
                assert ids[g][0] == 0 and (nv == 1 or ids[g][1] == nv - 1), (t, ids[g])
                assert len(sel) == min(nv, 4) and len(set(sel)) == len(sel)
                assert all(0 <= n < nv for n in sel)
            if nv <= 4:
                _, od, _ = impl.row(cfg, x, 0, t, dense=True)
                np.testing.assert_allclose(o, od, rtol=0, atol=1e-12)


PINS = [pin_golden_hand_worked, pin_topk_brute_force, pin_block_pool_properties, pin_index_score_projection,
        pin_dense_equals_sdpa, pin_sparse_equals_masked_sdpa, pin_diagram_grouping, pin_uniform_when_query_zero,
        pin_single_key, pin_causality, pin_selection_valid_and_scale_free, pin_planted_hot_blocks,
        pin_forced_sink_local_brute_force, pin_forced_rows]


@pytest.mark.parametrize("impl", GOOD, ids=lambda i: i.name)
@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_pin_holds(oracle_lib, impl, pin):
    pin(impl)


@pytest.mark.parametrize("mutant", MUTANTS, ids=lambda m: m.name)
def test_some_pin_rejects_mutant(oracle_lib, mutant):
    failed = []
    for pin in PINS:
        try:
            pin(mutant)
        except (AssertionError, IndexError, ValueError):
            failed.append(pin.__name__)
    assert failed, f"no pin caught {mutant.name}"


# --------------------------------------------------------------------------
# the two formulations agree on random inputs (both fp32 and bf16 storage)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("mode", ["decode", "prefill"])
def test_c_oracle_matches_numpy_twin(oracle_lib, dtype, mode):
    from block_sparse_long_12_b200.inputs import Workload, make_inputs, to_numpy_raw
    w = Workload("t", mode, 2, 300, 6, 3, 3 if mode == "decode" else 1, 16, 8, 16, 4, dtype, hot_blocks=3,
                 min_seq_len=150 if mode == "decode" else 0, seed=77)
    t = make_inputs(w)
    x = {n: to_numpy_raw(t[n]) for n in ("q", "q_idx", "k", "v", "k_idx", "seq_lens")}
    cfg = make_cfg(batch=2, n_q_heads=6, n_kv_heads=3, n_idx_k_heads=w.n_idx_k_heads, head_dim=16, idx_dim=8,
                   block_size=16, top_k=4, max_seq_len=300, dtype=dtype, prefill=mode == "prefill",
                   q_len=w.q_len)
    rows = [(b, t_) for b in range(2) for t_ in ((0,) if mode == "decode" else (0, 15, 16, 150, 299))]
    c, n = COracle(), Twin()
    for (b, t_) in rows:
        for dense in (False, True):
            cfg["force_sink_local"] = not dense and t_ % 2 == 0
            i1, o1, l1 = c.row(cfg, x, b, t_, dense)
            i2, o2, l2 = n.row(cfg, x, b, t_, dense)
            np.testing.assert_array_equal(i1, i2)
            np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-12)
            np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-12)


def test_kth_gap_reported(oracle_lib):
    """The k-th / (k+1)-th scores used by the near-tie rule come from the full ranking."""
    p = COracle().params(make_cfg(top_k=2))
    ids, sc, kth, kn = oracle.topk(p, np.array([1.0, 5.0, 3.0, 3.0, -2.0]))
    assert ids.tolist() == [1, 2] and sc.tolist() == [5.0, 3.0] and kth == 3.0 and kn == 3.0
    ids, sc, kth, kn = oracle.topk(p, np.array([1.0]))
    assert ids.tolist() == [0, -1] and math.isnan(kth) and math.isnan(kn)


@pytest.mark.parametrize("k", [33, 100, 1024])
def test_large_k_topk_matches_twin(oracle_lib, k):
    """TopK far beyond a warp list (the large-k regime): the C oracle's sort and the twin's rank
    counting agree on rows with many exact ties, fewer blocks than k, and forced blocks."""
    rng = np.random.default_rng(k)
    for trial in range(12):
        nb = int(rng.integers(1, 2500))
        S = rng.integers(-20, 21, nb).astype(np.float64) if trial % 2 else rng.standard_normal(nb)
        for force in (False, True):
            cfg = make_cfg(top_k=k, force_sink_local=force)
            got = COracle().topk(cfg, S)
            want = Twin().topk(cfg, S)
            np.testing.assert_array_equal(got, want)
            sel = [n for n in got if n >= 0]
            assert len(sel) == min(k, nb) and len(set(sel)) == len(sel)
            if force:
                assert got[0] == 0 and (nb == 1 or got[1] == nb - 1)
