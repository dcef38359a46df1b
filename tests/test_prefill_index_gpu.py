"""GPU parity of the fused prefill index branch (tensor-core index scores, block
max pool, TopK) against the fp64 oracle.  Page "MiniMax wird duenn"
(atlascloud.ai), section 1, Step 1, and section 3 (in prefill the index
branch still scans the whole visible input)."""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

import oracle
from block_sparse_long_12_b200.inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

from parity import check_forced, check_ids_row  # noqa: E402


def prefill_ids(inp, w, q_start, T, top_k=None, block_size=None, scores=False, force=False):
    from block_sparse_long_12_b200 import _lib, api
    k = top_k or w.top_k
    bk = block_size or w.block_size
    B = inp["q_idx"].shape[0]
    qi = inp["q_idx"][:, q_start:q_start + T].contiguous()
    p = api.make_params(batch=B, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads, n_idx_k_heads=w.n_idx_k_heads,
                        head_dim=w.head_dim, idx_dim=w.idx_dim, block_size=bk, top_k=k, max_seq_len=w.max_seq_len,
                        dtype=_lib.MSA_BF16, q_len=T, q_start=q_start,
                        flags=_lib.MSA_FORCE_SINK_LOCAL if force else 0)
    ids = torch.full((B, T, w.n_kv_heads, k), -7, dtype=torch.int32, device="cuda")
    ts = torch.empty(B, T, w.n_kv_heads, k, dtype=torch.float32, device="cuda") if scores else None
    ws = api.workspace(p, _lib.MSA_ENTRY_PREFILL_INDEX_TOPK, "cuda")
    _lib.msa_prefill_index_topk(p, qi, inp["k_idx"], ids, ts, ws)
    torch.cuda.synchronize()
    assert _lib.msa_get_device_status(ws) == 0
    return ids, ts


def check_rows(inp, w, q_start, T, ids, rows, top_k=None, block_size=None, force=False):
    """Compare GPU ids with the oracle on the given chunk rows (t relative to the chunk)."""
    from block_sparse_long_12_b200.inputs import to_numpy_raw
    k = top_k or w.top_k
    bk = block_size or w.block_size
    B = inp["q_idx"].shape[0]
    xo = {"q_idx": to_numpy_raw(inp["q_idx"][:, q_start:q_start + T]), "k_idx": to_numpy_raw(inp["k_idx"])}
    unused = np.zeros(8, np.uint16)  # Step 1 only: q, k, v are not read
    p = oracle.Params(B, w.n_q_heads, w.n_kv_heads, w.n_idx_k_heads, w.head_dim, w.idx_dim, bk, k, T, q_start,
                      w.max_seq_len, "bf16", w.softmax_scale, prefill=True, force_sink_local=force)
    ref = oracle.msa_rows(p, None, unused, xo["q_idx"], unused, unused, xo["k_idx"], rows, attention=False)
    idn = ids.cpu().numpy()
    ties = 0
    for i, (b, t) in enumerate(rows):
        for g in range(w.n_kv_heads):
            exact = check_ids_row(p, xo, b, t, g, q_start + t, idn[b, t, g], ref["ids"][i, g], ref["kth"][i, g],
                                  ref["kth_next"][i, g], where=f"b={b} t={t} g={g}",
                                  ref_scores=ref["top_scores"][i, g])
            ties += not exact
    return ties


def test_prefill_16k_all_rows():
    """16K causal prefill, 16 heads / 2 groups, block 64, k 16: every row checked."""
    w = WORKLOADS["prefill_causal_16k"]
    inp = make_inputs(w, device="cuda")
    ids, _ = prefill_ids(inp, w, 0, w.max_seq_len)
    rows = [(0, t) for t in range(w.max_seq_len)]
    check_rows(inp, w, 0, w.max_seq_len, ids, rows)


@pytest.mark.parametrize("case", [
    dict(block_size=128, top_k=16),
    dict(block_size=64, top_k=8),
    dict(block_size=32, top_k=32),
    dict(block_size=256, top_k=4),
    dict(block_size=128, top_k=1),
    dict(block_size=128, top_k=16, n_idx_k_heads=1),
], ids=lambda c: ",".join(f"{k}={v}" for k, v in c.items()))
def test_prefill_index_chunk_variants(case):
    """A ragged chunk (1000 rows starting at 1500) of a 3000-token batch-2 sequence."""
    hik = case.pop("n_idx_k_heads", 8)
    w = WORKLOADS["prefill_causal_1m"].scaled(max_seq_len=3000, batch=2, n_idx_k_heads=hik, hot_blocks=5, seed=21)
    inp = make_inputs(w, device="cuda")
    q_start, T = 1500, 1000
    ids, ts = prefill_ids(inp, w, q_start, T, top_k=case["top_k"], block_size=case["block_size"], scores=True)
    rows = [(b, t) for b in range(2) for t in range(T)]
    check_rows(inp, w, q_start, T, ids, rows, top_k=case["top_k"], block_size=case["block_size"])
    # scores come out sorted (desc) and are -inf exactly where ids are -1
    tsn, idn = ts.cpu().numpy(), ids.cpu().numpy()
    finite = np.where(np.isneginf(tsn), np.float32(-3e38), tsn)
    assert (np.diff(finite, axis=-1) <= 0).all()
    assert ((idn == -1) == np.isneginf(tsn)).all()


def test_prefill_index_first_rows_and_padding():
    """The first rows of a sequence see fewer blocks than k: the lists are padded with -1."""
    w = WORKLOADS["prefill_causal_1m"].scaled(max_seq_len=2048, batch=1, hot_blocks=0, seed=4)
    inp = make_inputs(w, device="cuda")
    ids, _ = prefill_ids(inp, w, 0, 600)
    idn = ids.cpu().numpy()
    for t in (0, 1, 127, 128, 599):
        nvalid = t // w.block_size + 1
        for g in range(w.n_kv_heads):
            assert sorted(idn[0, t, g, :nvalid].tolist()) == list(range(nvalid))
            assert (idn[0, t, g, nvalid:] == -1).all()
    check_rows(inp, w, 0, 600, ids, [(0, t) for t in range(600)])


def test_prefill_1m_sampled_rows():
    """The 1M-token workload chunk by chunk (8192 rows each): the first chunk fully and
    rows sampled across the whole sequence are checked against the oracle."""
    w = WORKLOADS["prefill_causal_1m"]
    inp = make_inputs(w, device="cuda")
    T = w.chunk
    rng = np.random.default_rng(1005)
    chunks = sorted(set([0] + rng.choice(w.max_seq_len // T, 6, replace=False).tolist()))
    for c in chunks:
        ids, _ = prefill_ids(inp, w, c * T, T)
        if c == 0:
            rows = [(0, t) for t in range(T)]
        else:
            rows = [(0, int(t)) for t in rng.choice(T, 16, replace=False)]
        check_rows(inp, w, c * T, T, ids, rows)


@pytest.mark.parametrize("case", [
    dict(block_size=128, top_k=16),
    dict(block_size=256, top_k=8),
    dict(block_size=32, top_k=32),
    dict(block_size=64, top_k=16, n_idx_k_heads=1),
], ids=lambda c: ",".join(f"{k}={v}" for k, v in c.items()))
def test_prefill_index_key_segments(case):
    """Few query rows against a long context: the kernel cuts every unit's keys into
    segments, keeps one list per segment and merges them; sampled rows (including the
    ragged last row tile) against the oracle."""
    from block_sparse_long_12_b200 import _lib, api
    hik = case.pop("n_idx_k_heads", 8)
    w = WORKLOADS["prefill_causal_1m"].scaled(max_seq_len=40000, batch=1, n_idx_k_heads=hik, hot_blocks=6, seed=77)
    inp = make_inputs(w, device="cuda")
    q_start, T = 39000, 1000
    p = api.make_params(batch=1, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads, n_idx_k_heads=hik,
                        head_dim=w.head_dim, idx_dim=w.idx_dim, block_size=case["block_size"], top_k=case["top_k"],
                        max_seq_len=w.max_seq_len, dtype=_lib.MSA_BF16, q_len=T, q_start=q_start)
    units = (T + 255) // 256 * w.n_kv_heads
    # the workspace holds per-segment lists only when units are split
    assert _lib.lib().msa_workspace_size(ctypes.byref(p), _lib.MSA_ENTRY_PREFILL_INDEX_TOPK) > 256 + (units * 4 + 255) // 256 * 256
    ids, ts = prefill_ids(inp, w, q_start, T, top_k=case["top_k"], block_size=case["block_size"], scores=True)
    rng = np.random.default_rng(5)
    rows = [(0, int(t)) for t in sorted(set(rng.choice(T, 160, replace=False).tolist()) | {0, 255, 256, 767, 768, T - 1})]
    check_rows(inp, w, q_start, T, ids, rows, top_k=case["top_k"], block_size=case["block_size"])
    tsn, idn = ts.cpu().numpy(), ids.cpu().numpy()
    assert ((idn == -1) == np.isneginf(tsn)).all()
    assert (idn >= -1).all() and (idn <= (q_start + T - 1) // case["block_size"]).all()


@pytest.mark.parametrize("case", [
    dict(block_size=128, top_k=16, q_start=0, T=700),      # first rows: one or few valid blocks
    dict(block_size=64, top_k=8, q_start=1500, T=1000),
    dict(block_size=128, top_k=1, q_start=1500, T=1000),   # k = 1: the sink alone
    dict(block_size=32, top_k=32, q_start=39000, T=1000),  # long context: split key segments
], ids=lambda c: ",".join(f"{k}={v}" for k, v in c.items()))
def test_prefill_index_forced_sink_local(case):
    """MSA_FORCE_SINK_LOCAL in the fused prefill index: block 0 and each row's own (diagonal) block
    lead the row's list, reported with +inf; the rest against the oracle with the same option."""
    L = 40000 if case["q_start"] >= 39000 else 3000
    w = WORKLOADS["prefill_causal_1m"].scaled(max_seq_len=L, batch=1, hot_blocks=5, seed=31)
    inp = make_inputs(w, device="cuda")
    q_start, T, k, bk = case["q_start"], case["T"], case["top_k"], case["block_size"]
    ids, ts = prefill_ids(inp, w, q_start, T, top_k=k, block_size=bk, scores=True, force=True)
    rng = np.random.default_rng(9)
    rows = [(0, int(t)) for t in sorted(set(rng.choice(T, 200, replace=False).tolist()) | {0, 1, 255, 256, T - 1})]
    check_rows(inp, w, q_start, T, ids, rows, top_k=k, block_size=bk, force=True)
    idn, tsn = ids.cpu().numpy(), ts.cpu().numpy()
    check_forced(idn, lambda b, t: q_start + t, bk, k)
    assert np.isposinf(tsn[..., 0]).all()
