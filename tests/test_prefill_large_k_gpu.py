"""GPU parity of prefill with lists of more than 32 blocks (large k) against the fp64 oracle.

Page "MiniMax wird duenn" (atlascloud.ai), section 1, Step 1 (TopK per group over the block
scores) and Step 2 (attention over the selected blocks); section 3 back-calculates that a query at
1M tokens keeps about 6-7 % of 16,384 blocks of 64 tokens, a k near 1000, and the index branch
runs in prefill as well as in decode.  Above 32 blocks per row the index epilogue stores every
visible block score and a radix select per row keeps the k best; the sparse branch runs in passes
of fewer rows and merges each row's k partials in chunks of 32."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from block_sparse_long_12_b200.inputs import WORKLOADS, make_inputs, to_numpy_raw

pytestmark = pytest.mark.gpu

from parity import check_forced, check_ids_row  # noqa: E402
from test_prefill_attn_gpu import compare, gpu_attend, gpu_index, oracle_attend, random_ids  # noqa: E402
from test_prefill_index_gpu import check_rows, prefill_ids  # noqa: E402


@pytest.mark.parametrize("case", [
    dict(block_size=32, top_k=64),
    dict(block_size=32, top_k=100),   # not a power of two
    dict(block_size=64, top_k=64),
    dict(block_size=128, top_k=40),
    dict(block_size=256, top_k=33),
    dict(block_size=32, top_k=256, n_idx_k_heads=1),
], ids=lambda c: ",".join(f"{k}={v}" for k, v in c.items()))
def test_prefill_index_large_k_chunk(case):
    """A ragged chunk (1000 rows from 9000) of a 12,000-token batch-2 sequence: every row's list
    against the oracle (near ties by the tie rule), scores sorted and -inf exactly at padding."""
    hik = case.pop("n_idx_k_heads", 8)
    w = WORKLOADS["prefill_causal_1m"].scaled(max_seq_len=12000, batch=2, n_idx_k_heads=hik, hot_blocks=8, seed=41)
    inp = make_inputs(w, device="cuda")
    q_start, T, k, bk = 9000, 1000, case["top_k"], case["block_size"]
    ids, ts = prefill_ids(inp, w, q_start, T, top_k=k, block_size=bk, scores=True)
    rows = [(b, t) for b in range(2) for t in range(T)]
    check_rows(inp, w, q_start, T, ids, rows, top_k=k, block_size=bk)
    tsn, idn = ts.cpu().numpy(), ids.cpu().numpy()
    finite = np.where(np.isneginf(tsn), np.float32(-3e38), tsn)
    assert (np.diff(finite, axis=-1) <= 0).all()
    assert ((idn == -1) == np.isneginf(tsn)).all()


def test_prefill_index_k1024_long_context():
    """k 1024 of up to 1,250 blocks of 32 tokens (rows at 39,400..40,000): sampled rows, including
    both ends of the chunk, against the oracle."""
    w = WORKLOADS["prefill_causal_1m"].scaled(max_seq_len=40000, batch=1, hot_blocks=6, seed=43)
    inp = make_inputs(w, device="cuda")
    q_start, T, k, bk = 39400, 600, 1024, 32
    ids, _ = prefill_ids(inp, w, q_start, T, top_k=k, block_size=bk)
    rng = np.random.default_rng(11)
    rows = [(0, int(t)) for t in sorted(set(rng.choice(T, 40, replace=False).tolist()) | {0, 255, 256, T - 1})]
    check_rows(inp, w, q_start, T, ids, rows, top_k=k, block_size=bk)


def test_prefill_index_large_k_first_rows_padding():
    """Rows that see fewer blocks than k take every visible block, then -1."""
    w = WORKLOADS["prefill_causal_1m"].scaled(max_seq_len=4096, batch=1, hot_blocks=0, seed=4)
    inp = make_inputs(w, device="cuda")
    k, bk = 64, 32
    ids, _ = prefill_ids(inp, w, 0, 2600, top_k=k, block_size=bk)
    idn = ids.cpu().numpy()
    for t in (0, 1, 31, 32, 1000, 2047, 2048, 2599):
        nvalid = min(t // bk + 1, k)
        for g in range(w.n_kv_heads):
            got = idn[0, t, g]
            assert (got[nvalid:] == -1).all()
            if t // bk + 1 <= k:
                assert sorted(got[:nvalid].tolist()) == list(range(nvalid))
    check_rows(inp, w, 0, 2600, ids, [(0, t) for t in range(0, 2600, 7)], top_k=k, block_size=bk)


@pytest.mark.parametrize("case", [
    dict(block_size=64, top_k=64, q_start=0, T=3000),     # first rows: the forced pair is most of the list
    dict(block_size=32, top_k=200, q_start=9000, T=1000),
], ids=lambda c: ",".join(f"{k}={v}" for k, v in c.items()))
def test_prefill_index_large_k_forced_sink_local(case):
    """MSA_FORCE_SINK_LOCAL with large k: block 0 and each row's own block lead its list with +inf,
    the rest against the oracle with the same option."""
    w = WORKLOADS["prefill_causal_1m"].scaled(max_seq_len=12000, batch=1, hot_blocks=5, seed=47)
    inp = make_inputs(w, device="cuda")
    q_start, T, k, bk = case["q_start"], case["T"], case["top_k"], case["block_size"]
    ids, ts = prefill_ids(inp, w, q_start, T, top_k=k, block_size=bk, scores=True, force=True)
    rng = np.random.default_rng(13)
    rows = [(0, int(t)) for t in sorted(set(rng.choice(T, 150, replace=False).tolist()) | {0, 1, T - 1})]
    check_rows(inp, w, q_start, T, ids, rows, top_k=k, block_size=bk, force=True)
    idn, tsn = ids.cpu().numpy(), ts.cpu().numpy()
    check_forced(idn, lambda b, t: q_start + t, bk, k)
    assert np.isposinf(tsn[..., 0]).all()


@pytest.mark.parametrize("case", [
    dict(head_dim=128, block_size=64, n_q_heads=64, n_kv_heads=8, top_k=64),
    dict(head_dim=128, block_size=128, n_q_heads=16, n_kv_heads=4, top_k=40),
    dict(head_dim=64, block_size=64, n_q_heads=32, n_kv_heads=2, top_k=200),   # group size 16
], ids=lambda c: ",".join(f"{k}={v}" for k, v in c.items()))
def test_prefill_attention_large_k_given_ids(case):
    """Step 2 alone with long random lists (ragged, -1 padded, some shuffled): every pass of the
    smaller pass size and the chunked merge against the oracle on the same ids."""
    w = WORKLOADS["prefill_causal_1m"].scaled(max_seq_len=16000, batch=2, hot_blocks=0, seed=53,
                                               n_idx_k_heads=case["n_kv_heads"], **case)
    inp = make_inputs(w, device="cuda")
    q_start, T = 12000, 4000  # k 200: passes of 1,310 rows; k 64: 4,096
    ids = random_ids(2, T, w.n_kv_heads, w.top_k, q_start, w.block_size, seed=7)
    o, lse = gpu_attend(inp, w, q_start, T, torch.from_numpy(ids).cuda())
    rng = np.random.default_rng(17)
    rows = [(b, int(t)) for b in range(2) for t in rng.choice(T, 60, replace=False)]
    rows += [(0, 0), (1, T - 1), (0, 1309), (0, 1310)]  # k 200: the first pass ends at row 1,309
    ref = oracle_attend(inp, w, q_start, T, rows, ids)
    compare(o, lse, ref, rows)


def _pipeline_vs_oracle(w, q_start, T, rows):
    """Index and sparse branch on the GPU; rows against the oracle's own selection, near-tie rows
    re-run with the GPU's ids."""
    inp = make_inputs(w, device="cuda")
    ids = gpu_index(inp, w, q_start, T)
    o, lse = gpu_attend(inp, w, q_start, T, ids)
    x = {n: to_numpy_raw(inp[n]) for n in ("q", "q_idx", "k", "v", "k_idx")}
    x["q"], x["q_idx"] = x["q"][:, q_start:q_start + T], x["q_idx"][:, q_start:q_start + T]
    p = oracle.Params(1, w.n_q_heads, w.n_kv_heads, w.n_idx_k_heads, w.head_dim, w.idx_dim, w.block_size, w.top_k,
                      T, q_start, w.max_seq_len, "bf16", w.softmax_scale, prefill=True)
    ref = oracle.msa_rows(p, None, x["q"], x["q_idx"], x["k"], x["v"], x["k_idx"], rows)
    idn = ids.cpu().numpy()
    xo = {"q_idx": x["q_idx"], "k_idx": x["k_idx"]}
    tie = []
    for i, (b, t) in enumerate(rows):
        for g in range(w.n_kv_heads):
            if not check_ids_row(p, xo, b, t, g, q_start + t, idn[b, t, g], ref["ids"][i, g], ref["kth"][i, g],
                                 ref["kth_next"][i, g], where=f"t={t} g={g}", ref_scores=ref["top_scores"][i, g]):
                tie.append(i)
    if tie:
        ids_in = ref["ids"].copy()
        for i in sorted(set(tie)):
            b, t = rows[i]
            ids_in[i] = idn[b, t]
        rerun = oracle.msa_rows(p, None, x["q"], x["q_idx"], x["k"], x["v"], x["k_idx"], rows, ids_in=ids_in)
        for i in sorted(set(tie)):
            ref["o"][i], ref["lse"][i] = rerun["o"][i], rerun["lse"][i]
    compare(o, lse, ref, rows)


def test_prefill_large_k_pipeline_64k():
    """64K context in 64-token blocks (1,024 blocks), k 64 (6.25 %, the pages' density): the last
    4,096 rows through both branches, 512 sampled rows against the oracle's own selection."""
    w = WORKLOADS["prefill_causal_16k"].scaled(max_seq_len=65536, top_k=64, seed=59)
    q_start, T = 65536 - 4096, 4096
    rng = np.random.default_rng(19)
    rows = [(0, int(t)) for t in sorted(set(rng.choice(T, 512, replace=False).tolist()) | {0, T - 1})]
    _pipeline_vs_oracle(w, q_start, T, rows)


def test_prefill_large_k_pipeline_k1024():
    """k 1024 of up to 1,250 blocks of 64 tokens (80K context): the last 512 rows (two passes of
    256) through both branches, sampled rows against the oracle's own selection."""
    w = WORKLOADS["prefill_causal_16k"].scaled(max_seq_len=80000, top_k=1024, seed=61)
    q_start, T = 80000 - 512, 512
    rng = np.random.default_rng(23)
    rows = [(0, int(t)) for t in sorted(set(rng.choice(T, 24, replace=False).tolist()) | {0, 255, 256, T - 1})]
    _pipeline_vs_oracle(w, q_start, T, rows)
