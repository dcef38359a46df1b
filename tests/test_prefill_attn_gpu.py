"""GPU parity of the prefill sparse branch (tensor-core sparse attention over
each token's selected blocks) against the fp64 oracle.  Page "MiniMax wird
duenn" (atlascloud.ai), section 1, Step 2: the heads of a group share the
group's list; attention runs on the real K/V of the selected blocks."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from block_sparse_long_12_b200.inputs import WORKLOADS, make_inputs, to_numpy_raw

pytestmark = pytest.mark.gpu

from parity import TOL_O, check_ids_row  # noqa: E402


def _lib_api():
    from block_sparse_long_12_b200 import _lib, api
    return _lib, api


def params(w, B, q_start, T, *, top_k=None, block_size=None):
    _lib, api = _lib_api()
    return api.make_params(batch=B, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads, n_idx_k_heads=w.n_idx_k_heads,
                           head_dim=w.head_dim, idx_dim=w.idx_dim, block_size=block_size or w.block_size,
                           top_k=top_k or w.top_k, max_seq_len=w.max_seq_len, dtype=_lib.MSA_BF16, q_len=T,
                           q_start=q_start)


def gpu_attend(inp, w, q_start, T, ids, *, top_k=None, block_size=None):
    _lib, api = _lib_api()
    B = inp["q"].shape[0]
    p = params(w, B, q_start, T, top_k=top_k, block_size=block_size)
    q = inp["q"][:, q_start:q_start + T].contiguous()
    o = torch.full_like(q, float("nan"))
    lse = torch.full((B, T, w.n_q_heads), float("nan"), device="cuda")
    ws = api.workspace(p, _lib.MSA_ENTRY_ATTN_PREFILL, "cuda")
    _lib.msa_sparse_attn_prefill(p, q, inp["k"], inp["v"], ids, o, lse, ws)
    torch.cuda.synchronize()
    assert _lib.msa_get_device_status(ws) == 0
    return o, lse


def gpu_index(inp, w, q_start, T, *, top_k=None, block_size=None):
    _lib, api = _lib_api()
    B = inp["q"].shape[0]
    p = params(w, B, q_start, T, top_k=top_k, block_size=block_size)
    ids = torch.empty(B, T, w.n_kv_heads, top_k or w.top_k, dtype=torch.int32, device="cuda")
    ws = api.workspace(p, _lib.MSA_ENTRY_PREFILL_INDEX_TOPK, "cuda")
    _lib.msa_prefill_index_topk(p, inp["q_idx"][:, q_start:q_start + T].contiguous(), inp["k_idx"], ids, None, ws)
    torch.cuda.synchronize()
    return ids


def oracle_attend(inp, w, q_start, T, rows, ids_np, *, top_k=None, block_size=None):
    """Oracle Step 2 for `rows` driven by the given ids ([B, T, G, k])."""
    k = top_k or w.top_k
    B = inp["q"].shape[0]
    x = {"q": to_numpy_raw(inp["q"][:, q_start:q_start + T]), "k": to_numpy_raw(inp["k"]),
         "v": to_numpy_raw(inp["v"])}
    unused = np.zeros(8, np.uint16)
    p = oracle.Params(B, w.n_q_heads, w.n_kv_heads, w.n_idx_k_heads, w.head_dim, w.idx_dim,
                      block_size or w.block_size, k, T, q_start, w.max_seq_len, "bf16", w.softmax_scale, prefill=True)
    ids_in = np.stack([ids_np[b, t] for (b, t) in rows])
    return oracle.msa_rows(p, None, x["q"], unused, x["k"], x["v"], unused, rows, ids_in=ids_in)


def compare(o, lse, ref, rows):
    on, ln = o.float().cpu().numpy(), lse.cpu().numpy()
    got_o = np.stack([on[b, t] for (b, t) in rows])
    got_l = np.stack([ln[b, t] for (b, t) in rows])
    err = np.abs(got_o - ref["o"]).max()
    assert err <= TOL_O["bf16"], f"max |o - oracle| = {err}"
    assert np.abs(got_l - ref["lse"]).max() <= 1e-2


def random_ids(B, T, G, k, q_start, bk, seed, n_valid_max=None):
    """Per token: up to k distinct causal-valid blocks (some rows with fewer, -1 padded, shuffled)."""
    rng = np.random.default_rng(seed)
    ids = np.full((B, T, G, k), -1, np.int32)
    for b in range(B):
        for t in range(T):
            nb = (q_start + t) // bk + 1
            for g in range(G):
                m = min(nb, int(rng.integers(1, k + 1)))
                ids[b, t, g, :m] = rng.choice(nb, m, replace=False)
                if t % 7 == 0:
                    rng.shuffle(ids[b, t, g])
    return ids


@pytest.mark.parametrize("case", [
    dict(head_dim=128, block_size=128, n_q_heads=64, n_kv_heads=8, top_k=16),
    dict(head_dim=128, block_size=64, n_q_heads=64, n_kv_heads=8, top_k=16),
    dict(head_dim=64, block_size=128, n_q_heads=32, n_kv_heads=4, top_k=8),
    dict(head_dim=128, block_size=128, n_q_heads=16, n_kv_heads=4, top_k=16),   # group size 4
    dict(head_dim=128, block_size=128, n_q_heads=32, n_kv_heads=2, top_k=32),   # group size 16
], ids=lambda c: ",".join(f"{k}={v}" for k, v in c.items()))
def test_prefill_attention_given_ids(case):
    """Step 2 alone: both sides attend with the same (random, ragged, -1 padded) ids."""
    w = WORKLOADS["prefill_causal_1m"].scaled(max_seq_len=3000, batch=2, hot_blocks=0, seed=31,
                                               n_idx_k_heads=case["n_kv_heads"], **case)
    inp = make_inputs(w, device="cuda")
    q_start, T = 1100, 900
    ids = random_ids(2, T, w.n_kv_heads, w.top_k, q_start, w.block_size, seed=5)
    o, lse = gpu_attend(inp, w, q_start, T, torch.from_numpy(ids).cuda())
    rows = [(b, t) for b in range(2) for t in range(0, T, 3)] + [(1, T - 1), (0, T - 1)]
    ref = oracle_attend(inp, w, q_start, T, rows, ids)
    compare(o, lse, ref, rows)


def test_prefill_attention_first_rows():
    """Chunk at the start of the sequence: the first tokens see only part of block 0."""
    w = WORKLOADS["prefill_causal_1m"].scaled(max_seq_len=1024, batch=1, hot_blocks=0, seed=8)
    inp = make_inputs(w, device="cuda")
    T = 300
    ids = random_ids(1, T, w.n_kv_heads, w.top_k, 0, w.block_size, seed=2)
    o, lse = gpu_attend(inp, w, 0, T, torch.from_numpy(ids).cuda())
    rows = [(0, t) for t in range(T)]
    ref = oracle_attend(inp, w, 0, T, rows, ids)
    compare(o, lse, ref, rows)


def test_prefill_16k_pipeline():
    """16K causal prefill end to end on the GPU (index branch, then sparse branch); sampled rows
    against the oracle's own selection (near-tie rows re-run with the GPU's ids)."""
    w = WORKLOADS["prefill_causal_16k"]
    inp = make_inputs(w, device="cuda")
    T = w.max_seq_len
    ids = gpu_index(inp, w, 0, T)
    o, lse = gpu_attend(inp, w, 0, T, ids)
    rng = np.random.default_rng(2)
    rows = [(0, int(t)) for t in sorted(set(rng.choice(T, 1024, replace=False).tolist()) | {0, 1, 63, 64, T - 1})]
    x = {n: to_numpy_raw(inp[n]) for n in ("q", "q_idx", "k", "v", "k_idx")}
    p = oracle.Params(1, w.n_q_heads, w.n_kv_heads, w.n_idx_k_heads, w.head_dim, w.idx_dim, w.block_size, w.top_k,
                      T, 0, T, "bf16", w.softmax_scale, prefill=True)
    ref = oracle.msa_rows(p, None, x["q"], x["q_idx"], x["k"], x["v"], x["k_idx"], rows)
    idn = ids.cpu().numpy()
    xo = {"q_idx": x["q_idx"], "k_idx": x["k_idx"]}
    tie = []
    for i, (b, t) in enumerate(rows):
        for g in range(w.n_kv_heads):
            if not check_ids_row(p, xo, b, t, g, t, idn[b, t, g], ref["ids"][i, g], ref["kth"][i, g],
                                 ref["kth_next"][i, g], where=f"t={t} g={g}", ref_scores=ref["top_scores"][i, g]):
                tie.append(i)
    if tie:
        ids_in = ref["ids"].copy()
        for i in tie:
            b, t = rows[i]
            ids_in[i] = idn[b, t]
        rerun = oracle.msa_rows(p, None, x["q"], x["q_idx"], x["k"], x["v"], x["k_idx"], rows, ids_in=ids_in)
        for i in tie:
            ref["o"][i], ref["lse"][i] = rerun["o"][i], rerun["lse"][i]
    compare(o, lse, ref, rows)


def test_prefill_1m_last_chunk_sampled():
    """The last 8192-token chunk of the 1M-token workload: index + attention on the GPU,
    sampled rows against the oracle driven by the GPU's ids."""
    w = WORKLOADS["prefill_causal_1m"]
    inp = make_inputs(w, device="cuda")
    T = w.chunk
    q_start = w.max_seq_len - T
    ids = gpu_index(inp, w, q_start, T)
    o, lse = gpu_attend(inp, w, q_start, T, ids)
    rng = np.random.default_rng(3)
    rows = [(0, int(t)) for t in rng.choice(T, 64, replace=False)] + [(0, T - 1)]
    ref = oracle_attend(inp, w, q_start, T, rows, ids.cpu().numpy())
    compare(o, lse, ref, rows)
