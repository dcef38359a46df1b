"""GPU parity of the decode path (C ABI -> CUDA kernels) against the fp64 oracle.

Step 1 (index score, block max pool, TopK) and Step 2 (sparse attention of
every head of the group over the group's selected blocks), page "MiniMax wird
duenn" (atlascloud.ai), section 1.
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle
from block_sparse_long_12_b200.inputs import WORKLOADS, Workload, make_inputs

pytestmark = pytest.mark.gpu

from parity import check_forced, compare_decode, oracle_params, to_np  # noqa: E402


def _api():
    from block_sparse_long_12_b200 import api
    return api


def run_fused(inp, w, force_sink_local=False):
    api = _api()
    o, ids, lse = api.decode(inp["q"], inp["q_idx"], inp["k"], inp["v"], inp["k_idx"], inp["seq_lens"],
                             block_size=w.block_size, top_k=w.top_k, force_sink_local=force_sink_local)
    torch.cuda.synchronize()
    return o, ids, lse


def small(name="decode_b8_ctx128k_ragged", **kw):
    base = dict(batch=3, max_seq_len=5000, min_seq_len=1, n_q_heads=16, n_kv_heads=4, n_idx_k_heads=4, head_dim=128,
                idx_dim=64, block_size=64, top_k=8, hot_blocks=6, seed=11)
    base.update(kw)
    return WORKLOADS[name].scaled(**base)


def test_tiny_fp32_decode_full():
    """4096-token fp32 decode, 4 query heads on 1 KV head, k = 8 of 64 blocks."""
    w = WORKLOADS["decode_fp32_ctx4k"]
    inp = make_inputs(w, device="cuda")
    o, ids, lse = run_fused(inp, w)
    x = to_np(inp)
    res = compare_decode(x, oracle_params(x, block_size=w.block_size, top_k=w.top_k), o, ids, lse)
    assert res["err_o"] <= 1e-4


@pytest.mark.parametrize("case", [
    dict(),                                                           # ragged, partial last blocks
    dict(dtype="f32", idx_dim=32, head_dim=64),                        # fp32, D 64
    dict(n_idx_k_heads=1, hot_blocks=0),                               # one index-K head shared by all groups
    dict(n_kv_heads=8, n_q_heads=8, n_idx_k_heads=1, hot_blocks=0),    # 8 groups on one index-K stream, r = 1
    dict(block_size=16, top_k=32, max_seq_len=3000),                   # small blocks, largest k
    dict(block_size=256, top_k=1, max_seq_len=9000),                   # big blocks, k = 1
    dict(block_size=128, top_k=20, max_seq_len=1500, min_seq_len=1),  # fewer valid blocks than k: -1 padding
    dict(n_q_heads=24, n_kv_heads=4, n_idx_k_heads=4),                 # group size 6 (padded to 8)
    dict(n_q_heads=64, n_kv_heads=4, n_idx_k_heads=4, head_dim=64),    # group size 16
    dict(idx_dim=128, dtype="bf16"),                                   # 256-byte index rows
    dict(idx_dim=32, dtype="bf16"),                                    # 64-byte index rows
    dict(batch=9, max_seq_len=700, min_seq_len=1, seed=5),             # many short sequences
    # several groups on one index-K stream: tensor-core scores for bf16 rows of 128 / 256 bytes,
    # CUDA-core dot products for fp32 and for 64-byte rows
    dict(idx_dim=128, dtype="bf16", n_idx_k_heads=1),
    dict(dtype="f32", idx_dim=32, head_dim=64, n_idx_k_heads=1),
    dict(idx_dim=32, dtype="bf16", n_idx_k_heads=1),
], ids=lambda c: ",".join(f"{k}={v}" for k, v in c.items()) or "base")
def test_decode_fused_variants(case):
    w = small(**case)
    inp = make_inputs(w, device="cuda")
    o, ids, lse = run_fused(inp, w)
    x = to_np(inp)
    compare_decode(x, oracle_params(x, block_size=w.block_size, top_k=w.top_k), o, ids, lse)


def test_shared_stream_selection_in_chunks():
    """Groups on one index-K stream select from every block's score, staged in shared memory in
    chunks when the stream has more blocks than one chunk holds (16-token blocks: 6,250 blocks)."""
    w = small(block_size=16, top_k=32, max_seq_len=100000, min_seq_len=90000, batch=2, n_idx_k_heads=1, hot_blocks=12)
    inp = make_inputs(w, device="cuda")
    o, ids, lse = run_fused(inp, w)
    x = to_np(inp)
    compare_decode(x, oracle_params(x, block_size=w.block_size, top_k=w.top_k), o, ids, lse)


def test_shared_stream_selection_many_at_floor():
    """Block scores that repeat with a period of 128 blocks (the index keys of block n equal those
    of block n mod 128): the k-th best of the selecting threads' bests is then a floor that many
    blocks reach (k times the number of periods, 768), beyond what is sorted at once; ids and
    outputs against the oracle, and equal scores taken by lower id."""
    w = small(block_size=64, top_k=32, max_seq_len=196608, min_seq_len=196608, batch=1, n_idx_k_heads=1,
              hot_blocks=0)
    inp = make_inputs(w, device="cuda")
    period = 128 * w.block_size
    ki = inp["k_idx"]
    for t0 in range(period, w.max_seq_len, period):
        ki[:, :, t0:t0 + period] = ki[:, :, :period]
    o, ids, lse = run_fused(inp, w)
    x = to_np(inp)
    compare_decode(x, oracle_params(x, block_size=w.block_size, top_k=w.top_k), o, ids, lse)
    # every selected block is the lowest-id copy's class mate: within a class the lower ids come first
    idn = ids.cpu().numpy()[0, 0]
    for g in range(w.n_kv_heads):
        sel = idn[g][idn[g] >= 0]
        for c in np.unique(sel % 128):
            mates = np.sort(sel[sel % 128 == c])
            assert mates.tolist() == list(range(c, c + 128 * len(mates), 128)), (g, c, mates)


@pytest.mark.parametrize("case", [
    dict(),                                                           # ragged, partial last blocks
    dict(n_idx_k_heads=1, hot_blocks=0),                               # groups on one shared stream (tensor cores)
    dict(dtype="f32", idx_dim=32, head_dim=64),                        # fp32
    dict(block_size=128, top_k=20, max_seq_len=1500, min_seq_len=1),  # fewer valid blocks than k
    dict(block_size=256, top_k=1, max_seq_len=9000),                   # k = 1: the sink alone
    dict(block_size=16, top_k=32, max_seq_len=3000),                   # small blocks, largest k
], ids=lambda c: ",".join(f"{k}={v}" for k, v in c.items()) or "base")
def test_decode_forced_sink_local(case):
    """MSA_FORCE_SINK_LOCAL: block 0 and the query's own block lead every list, the rest is the
    best of the other blocks; ids and outputs against the oracle with the same option."""
    w = small(**case)
    inp = make_inputs(w, device="cuda")
    inp["seq_lens"][0] = 1  # one visible token: the two forced blocks are one
    o, ids, lse = run_fused(inp, w, force_sink_local=True)
    x = to_np(inp)
    compare_decode(x, oracle_params(x, block_size=w.block_size, top_k=w.top_k, force_sink_local=True), o, ids, lse)
    check_forced(ids.cpu().numpy(), lambda b, t: int(x["seq_lens"][b]) - 1, w.block_size, w.top_k)


def test_decode_exact_lengths_edges():
    """Lengths 1, Bk-1, Bk, Bk+1 and Lmax in one batch."""
    w = small(batch=5, max_seq_len=1000, block_size=64, top_k=4, hot_blocks=0)
    inp = make_inputs(w, device="cuda")
    inp["seq_lens"].copy_(torch.tensor([1, 63, 64, 65, 1000], dtype=torch.int32))
    o, ids, lse = run_fused(inp, w)
    x = to_np(inp)
    compare_decode(x, oracle_params(x, block_size=64, top_k=4), o, ids, lse)
    idn = ids.cpu().numpy()
    assert idn[0, 0, :, 0].tolist() == [0] * 4 and (idn[0, 0, :, 1:] == -1).all()


@pytest.mark.parametrize("hik,di,gk", [(4, 64, 4), (1, 64, 4), (1, 128, 4), (1, 64, 8), (1, 64, 2)],
                         ids=["hik4", "hik1", "hik1_di128", "hik1_g8", "hik1_g2"])
def test_index_scores_and_pool_topk(hik, di, gk):
    """Stored token / block scores, then the stand-alone pool + TopK entry (hik < groups: the
    groups that share one index-K stream, 2, 4 or 8 of them, are scored together on tensor cores,
    64- and 128-dim index keys)."""
    api = _api()
    w = small(dtype="bf16", hot_blocks=4, n_idx_k_heads=hik, idx_dim=di, n_kv_heads=gk, n_q_heads=4 * gk)
    inp = make_inputs(w, device="cuda")
    x = to_np(inp)
    p = oracle_params(x, block_size=w.block_size, top_k=w.top_k)
    tok = api.index_scores(inp["q_idx"], inp["k_idx"], inp["seq_lens"], n_kv_heads=w.n_kv_heads,
                           block_size=w.block_size, mode="token")
    blk = api.index_scores(inp["q_idx"], inp["k_idx"], inp["seq_lens"], n_kv_heads=w.n_kv_heads,
                           block_size=w.block_size, mode="block")
    torch.cuda.synchronize()
    tok_n, blk_n = tok.cpu().numpy(), blk.cpu().numpy()
    for b in range(w.batch):
        L = int(x["seq_lens"][b])
        for g in range(w.n_kv_heads):
            s = oracle.token_scores(p, x["q_idx"], x["k_idx"], b, 0, g, L - 1)
            S = oracle.block_scores(p, s, L - 1)
            scale = np.abs(s).max() + 1.0
            assert np.abs(tok_n[b, 0, g, :L] - s).max() <= 1e-5 * scale
            assert np.isneginf(tok_n[b, 0, g, L:]).all()
            assert np.abs(blk_n[b, 0, g, :len(S)] - S).max() <= 1e-5 * scale
            assert np.isneginf(blk_n[b, 0, g, len(S):]).all()
    # pool + TopK from the stored fp32 scores: the oracle on the same fp32 values must agree exactly
    for is_block, sc in ((False, tok), (True, blk)):
        ids, ts = api.pool_topk(sc, inp["seq_lens"], block_size=w.block_size, top_k=w.top_k,
                                max_seq_len=w.max_seq_len, is_block=is_block)
        torch.cuda.synchronize()
        ids_n, ts_n = ids.cpu().numpy(), ts.cpu().numpy()
        for b in range(w.batch):
            L = int(x["seq_lens"][b])
            for g in range(w.n_kv_heads):
                S = oracle.block_scores(p, tok_n[b, 0, g, :L].astype(np.float64), L - 1)
                ref_ids, ref_sc, _, _ = oracle.topk(p, S)
                assert ids_n[b, 0, g].tolist() == ref_ids.tolist()
                np.testing.assert_array_equal(ts_n[b, 0, g][ref_ids >= 0], ref_sc[ref_ids >= 0].astype(np.float32))


def test_pool_topk_forced_sink_local():
    """The stand-alone TopK entry with MSA_FORCE_SINK_LOCAL, decode rows (block scores) and prefill
    rows (token scores): exact against the oracle on the same fp32 values, forced scores +inf."""
    api = _api()
    B, G, L, bk, k = 3, 2, 700, 16, 6
    gen = torch.Generator(device="cuda").manual_seed(8)
    lens = torch.tensor([700, 17, 5], dtype=torch.int32, device="cuda")
    nb = -(-L // bk)
    blk = torch.randn(B, 1, G, nb, device="cuda", generator=gen).round(decimals=1)
    ids, ts = api.pool_topk(blk, lens, block_size=bk, top_k=k, max_seq_len=L, is_block=True, force_sink_local=True)
    torch.cuda.synchronize()
    p = oracle.Params(B, G, G, G, 64, 32, bk, k, 1, 0, L, "f32", 0.125, force_sink_local=True)
    bn, idn, tsn = blk.cpu().numpy(), ids.cpu().numpy(), ts.cpu().numpy()
    for b in range(B):
        n_valid = (int(lens[b]) - 1) // bk + 1
        for g in range(G):
            ref_ids, ref_sc, _, _ = oracle.topk(p, bn[b, 0, g, :n_valid].astype(np.float64))
            assert idn[b, 0, g].tolist() == ref_ids.tolist()
            np.testing.assert_array_equal(tsn[b, 0, g][ref_ids >= 0], ref_sc[ref_ids >= 0].astype(np.float32))
    check_forced(idn, lambda b, t: int(lens[b]) - 1, bk, k)
    T = 40
    sc = torch.randn(1, T, G, 300, device="cuda", generator=gen).round(decimals=1)
    ids, _ = api.pool_topk(sc, None, block_size=bk, top_k=k, max_seq_len=300, is_block=False, q_start=0,
                           force_sink_local=True)
    torch.cuda.synchronize()
    pp = oracle.Params(1, G, G, G, 64, 32, bk, k, T, 0, 300, "f32", 0.125, prefill=True, force_sink_local=True)
    scn, idn = sc.cpu().numpy(), ids.cpu().numpy()
    for t in range(T):
        for g in range(G):
            S = oracle.block_scores(pp, scn[0, t, g, :t + 1].astype(np.float64), t)
            assert idn[0, t, g].tolist() == oracle.topk(pp, S)[0].tolist()
    check_forced(idn, lambda b, t: t, bk, k)


@pytest.mark.parametrize("k", [33, 100, 1024])
def test_pool_topk_large_k(k):
    """TopK beyond the warp lists (radix select per row) from stored block and token scores,
    decode rows with ragged lengths (fewer valid blocks than k included), many exact ties; with
    and without forced blocks; exact against the oracle on the same fp32 values."""
    api = _api()
    B, G, L, bk = 3, 2, 40000, 16
    gen = torch.Generator(device="cuda").manual_seed(k)
    lens = torch.tensor([40000, 5000, 700], dtype=torch.int32, device="cuda")
    nb = -(-L // bk)
    tok = torch.randn(B, 1, G, L, device="cuda", generator=gen).round(decimals=2)
    for force in (False, True):
        p = oracle.Params(B, G, G, G, 64, 32, bk, k, 1, 0, L, "f32", 0.125, force_sink_local=force)
        tok_n = tok.cpu().numpy()
        want = {}
        for b in range(B):
            Lb = int(lens[b])
            for g in range(G):
                S = oracle.block_scores(p, tok_n[b, 0, g, :Lb].astype(np.float64), Lb - 1)
                want[b, g] = (S, oracle.topk(p, S))
        blk = torch.full((B, 1, G, nb), float("nan"), device="cuda")  # entries past a row's blocks are not read
        for (b, g), (S, _) in want.items():
            blk[b, 0, g, :len(S)] = torch.from_numpy(S.astype(np.float32))
        for is_block, sc in ((True, blk), (False, tok)):
            ids, ts = api.pool_topk(sc, lens, block_size=bk, top_k=k, max_seq_len=L, is_block=is_block,
                                    force_sink_local=force)
            torch.cuda.synchronize()
            idn, tsn = ids.cpu().numpy(), ts.cpu().numpy()
            for (b, g), (S, (ref_ids, ref_sc, _, _)) in want.items():
                assert idn[b, 0, g].tolist() == ref_ids.tolist(), (is_block, force, b, g)
                np.testing.assert_array_equal(tsn[b, 0, g][ref_ids >= 0], ref_sc[ref_ids >= 0].astype(np.float32))
                assert np.isneginf(tsn[b, 0, g][ref_ids < 0]).all()
            if force:
                check_forced(idn, lambda b, t: int(lens[b]) - 1, bk, k)


def test_pool_topk_large_k_long_rows():
    """Rows of more blocks than the select keeps in registers (40,000 and 20,001 blocks): the keys
    are re-read from memory in every radix pass; exact against the oracle, ties included."""
    api = _api()
    B, G, bk, k = 2, 2, 16, 500
    L = 40000 * bk
    gen = torch.Generator(device="cuda").manual_seed(21)
    lens = torch.tensor([L, 20001 * bk - 3], dtype=torch.int32, device="cuda")
    nb = L // bk
    blk = torch.randn(B, 1, G, nb, device="cuda", generator=gen).round(decimals=2)
    for force in (False, True):
        ids, ts = api.pool_topk(blk, lens, block_size=bk, top_k=k, max_seq_len=L, is_block=True,
                                force_sink_local=force)
        torch.cuda.synchronize()
        p = oracle.Params(B, G, G, G, 64, 32, bk, k, 1, 0, L, "f32", 0.125, force_sink_local=force)
        bn, idn, tsn = blk.cpu().numpy(), ids.cpu().numpy(), ts.cpu().numpy()
        for b in range(B):
            n_valid = (int(lens[b]) - 1) // bk + 1
            for g in range(G):
                ref_ids, ref_sc, _, _ = oracle.topk(p, bn[b, 0, g, :n_valid].astype(np.float64))
                assert idn[b, 0, g].tolist() == ref_ids.tolist(), (force, b, g)
                np.testing.assert_array_equal(tsn[b, 0, g], ref_sc.astype(np.float32))


def test_pool_topk_large_k_prefill_rows():
    """The large-k TopK on prefill rows (pos = q_start + t) from stored token scores."""
    api = _api()
    B, T, G, L, bk, k = 1, 24, 2, 3000, 16, 64
    gen = torch.Generator(device="cuda").manual_seed(12)
    sc = torch.randn(B, T, G, L, device="cuda", generator=gen).round(decimals=1)
    ids, _ = api.pool_topk(sc, None, block_size=bk, top_k=k, max_seq_len=L, is_block=False, q_start=2000)
    torch.cuda.synchronize()
    p = oracle.Params(B, G, G, G, 64, 32, bk, k, T, 2000, L, "f32", 0.125, prefill=True)
    scn, idn = sc.cpu().numpy(), ids.cpu().numpy()
    for t in range(T):
        pos = 2000 + t
        for g in range(G):
            S = oracle.block_scores(p, scn[0, t, g, :pos + 1].astype(np.float64), pos)
            assert idn[0, t, g].tolist() == oracle.topk(p, S)[0].tolist()


@pytest.mark.parametrize("case", [
    dict(block_size=64, top_k=100, max_seq_len=20000),                       # ragged batch of 3
    dict(block_size=64, top_k=1024, max_seq_len=100000, batch=2, hot_blocks=40),  # k 1024
    dict(block_size=64, top_k=300, max_seq_len=12000, min_seq_len=1),         # fewer valid blocks than k
    dict(block_size=64, top_k=48, dtype="f32", idx_dim=32, head_dim=64),      # fp32 attention kernel
    dict(block_size=128, top_k=64, n_idx_k_heads=1, hot_blocks=0),             # shared stream (tensor cores)
    dict(block_size=64, top_k=128, max_seq_len=30000, force=True),            # forced sink / local blocks
], ids=lambda c: ",".join(f"{k}={v}" for k, v in c.items()))
def test_decode_fused_large_k(case):
    """Fused decode with k beyond the warp lists: the scan stores every block score, a radix select
    writes each group's list, the attention splits the blocks over many CTAs; ids and outputs
    against the oracle."""
    case = dict(case)
    force = case.pop("force", False)
    w = small(**case)
    inp = make_inputs(w, device="cuda")
    o, ids, lse = run_fused(inp, w, force_sink_local=force)
    x = to_np(inp)
    compare_decode(x, oracle_params(x, block_size=w.block_size, top_k=w.top_k, force_sink_local=force), o, ids, lse)
    if force:
        check_forced(ids.cpu().numpy(), lambda b, t: int(x["seq_lens"][b]) - 1, w.block_size, w.top_k)


def test_pool_topk_prefill_rows():
    """The stand-alone TopK entry on prefill rows (pos = q_start + t) from stored token scores."""
    api = _api()
    B, T, G, L, bk, k = 1, 40, 2, 300, 16, 5
    gen = torch.Generator(device="cuda").manual_seed(3)
    sc = torch.randn(B, T, G, L, device="cuda", generator=gen).round(decimals=1)  # many exact ties
    ids, ts = api.pool_topk(sc, None, block_size=bk, top_k=k, max_seq_len=L, is_block=False, q_start=200)
    torch.cuda.synchronize()
    p = oracle.Params(B, G, G, G, 64, 32, bk, k, T, 200, L, "f32", 0.125, prefill=True)
    scn, idn = sc.cpu().numpy(), ids.cpu().numpy()
    for t in range(T):
        pos = 200 + t
        for g in range(G):
            S = oracle.block_scores(p, scn[0, t, g, :pos + 1].astype(np.float64), pos)
            assert idn[0, t, g].tolist() == oracle.topk(p, S)[0].tolist()


@pytest.mark.parametrize("case", [
    dict(),                                              # D 128, block 64, k 6
    dict(head_dim=64, block_size=128),                   # D 64 (the many-tile kernel's 64-key tiles)
    dict(block_size=16, top_k=40),                       # k > 32 given: ids read by split; tiles of 16 keys
    dict(head_dim=64, block_size=256, top_k=48),         # D 64, 256-token blocks, k > 32, lists mostly -1
], ids=lambda c: ",".join(f"{k}={v}" for k, v in c.items()) or "base")
def test_attend_decode_given_ids_and_dense(case):
    api = _api()
    w = small(batch=4, max_seq_len=3000, **{"top_k": 6, "hot_blocks": 0, **case})
    inp = make_inputs(w, device="cuda")
    x = to_np(inp)
    gen = np.random.default_rng(5)
    ids = np.full((w.batch, 1, w.n_kv_heads, w.top_k), -1, np.int32)
    for b in range(w.batch):
        nb = -(-int(x["seq_lens"][b]) // w.block_size)
        for g in range(w.n_kv_heads):
            m = min(nb, int(gen.integers(1, w.top_k + 1)))
            ids[b, 0, g, :m] = gen.choice(nb, m, replace=False)
            gen.shuffle(ids[b, 0, g])  # -1 entries anywhere in the list
    o, lse = api.attend_decode(inp["q"], inp["k"], inp["v"], torch.from_numpy(ids).cuda(), inp["seq_lens"],
                               block_size=w.block_size, top_k=w.top_k)
    torch.cuda.synchronize()
    p = oracle_params(x, block_size=w.block_size, top_k=w.top_k)
    rows = [(b, 0) for b in range(w.batch)]
    ref = oracle.msa_rows(p, x["seq_lens"], x["q"], x["q_idx"], x["k"], x["v"], x["k_idx"], rows,
                          ids_in=ids[:, 0])
    assert np.abs(o.float().cpu().numpy()[:, 0] - ref["o"]).max() <= 2e-2
    assert np.abs(lse.cpu().numpy()[:, 0] - ref["lse"]).max() <= 1e-3
    od, lsed = api.attend_decode(inp["q"], inp["k"], inp["v"], None, inp["seq_lens"], block_size=w.block_size,
                                 top_k=w.top_k, dense=True)
    torch.cuda.synchronize()
    pd = oracle_params(x, block_size=w.block_size, top_k=w.top_k, dense=True)
    refd = oracle.msa_rows(pd, x["seq_lens"], x["q"], x["q_idx"], x["k"], x["v"], x["k_idx"], rows)
    assert np.abs(od.float().cpu().numpy()[:, 0] - refd["o"]).max() <= 2e-2
    assert np.abs(lsed.cpu().numpy()[:, 0] - refd["lse"]).max() <= 1e-3


def test_dense_equals_sparse_when_k_covers_all():
    """With k >= number of blocks, MSA decode equals the dense GQA decode (both GPU paths)."""
    api = _api()
    w = small(batch=2, max_seq_len=1024, block_size=64, top_k=16, hot_blocks=0)
    inp = make_inputs(w, device="cuda")
    o, ids, lse = run_fused(inp, w)
    od, lsed = api.attend_decode(inp["q"], inp["k"], inp["v"], None, inp["seq_lens"], block_size=64, top_k=16,
                                 dense=True)
    torch.cuda.synchronize()
    assert (o.float() - od.float()).abs().max().item() <= 2e-2
    # the two paths merge different numbers of fp32 splits: compare at the LSE tolerance used against the oracle
    assert (lse - lsed).abs().max().item() <= 1e-3


def test_repeat_calls_same_workspace():
    """The workspace is rewritten by each call: two calls give identical results."""
    api = _api()
    w = small()
    inp = make_inputs(w, device="cuda")
    p = api.params_from(inp["q"], inp["q_idx"], inp["k"], inp["k_idx"], block_size=w.block_size, top_k=w.top_k,
                        seq_lens=inp["seq_lens"])
    ws = api.workspace(p, api.MSA_ENTRY_DECODE_FUSED, "cuda")
    a = api.decode(inp["q"], inp["q_idx"], inp["k"], inp["v"], inp["k_idx"], inp["seq_lens"],
                   block_size=w.block_size, top_k=w.top_k, ws=ws)
    a = [t.clone() for t in a]
    b = api.decode(inp["q"], inp["q_idx"], inp["k"], inp["v"], inp["k_idx"], inp["seq_lens"],
                   block_size=w.block_size, top_k=w.top_k, ws=ws)
    torch.cuda.synchronize()
    for t1, t2 in zip(a, b):
        assert torch.equal(t1, t2)
    from block_sparse_long_12_b200 import _lib
    assert _lib.msa_get_device_status(ws) == 0


def test_workspace_reused_across_shapes():
    """One workspace serves calls of different shapes in turn (its layout moves with the
    shape): every call equals a call on a fresh workspace, and the status stays clean."""
    api = _api()
    from block_sparse_long_12_b200 import _lib
    wa, wb = small(batch=4, seed=5), small(batch=1, max_seq_len=7000, seed=6, n_kv_heads=2, n_q_heads=8,
                                           n_idx_k_heads=2)
    ia, ib = make_inputs(wa, device="cuda"), make_inputs(wb, device="cuda")

    def params(inp, w):
        return api.params_from(inp["q"], inp["q_idx"], inp["k"], inp["k_idx"], block_size=w.block_size,
                               top_k=w.top_k, seq_lens=inp["seq_lens"])

    shared = api.workspace([params(ia, wa), params(ib, wb)], api.MSA_ENTRY_DECODE_FUSED, "cuda")
    for inp, w in ((ia, wa), (ib, wb), (ia, wa), (ib, wb)):
        got = api.decode(inp["q"], inp["q_idx"], inp["k"], inp["v"], inp["k_idx"], inp["seq_lens"],
                         block_size=w.block_size, top_k=w.top_k, ws=shared)
        got = [t.clone() for t in got]
        ref = run_fused(inp, w)
        for t1, t2 in zip(got, ref):
            assert torch.equal(t1, t2)
    assert _lib.msa_get_device_status(shared) == 0


@pytest.mark.parametrize("name", ["decode_b8_ctx128k_ragged", "decode_ctx1m", "decode_b4_ctx1m", "decode_ctx1m_large_k",
                                  "decode_ctx1m_shared_idx"])
def test_full_size_decode(name):
    """The benchmark workloads at full size, checked against the oracle on every (sequence, group)."""
    w = WORKLOADS[name]
    inp = make_inputs(w, device="cuda")
    o, ids, lse = run_fused(inp, w)
    x = to_np(inp)
    hot = inp["hot"].cpu().numpy()
    del inp
    torch.cuda.empty_cache()
    compare_decode(x, oracle_params(x, block_size=w.block_size, top_k=w.top_k), o, ids, lse)
    # planted data: every selected block is hot (k <= hot blocks), or every hot block is selected
    idn = ids.cpu().numpy()
    for b in range(w.batch):
        for g in range(w.n_kv_heads):
            sel, hb = set(idn[b, 0, g].tolist()), set(hot[b, g % w.n_idx_k_heads].tolist()) - {-1}
            assert sel <= hb if w.top_k <= len(hb) else hb <= sel
