"""Prefill parity at the coverage of the workloads' own statement.

The whole prefill pipeline runs on the GPU through the C ABI (index branch,
then sparse branch, chunk by chunk); the fp64 oracle runs Steps 1 and 2 on
the same bytes with its OWN selection, and both the block ids and the outputs
are compared:

* 16K causal prefill (16 heads / 2 groups, block 64, k 16): every one of the
  16,384 rows;
* 1M-token causal prefill in 8192-token chunks (64 heads / 8 groups, block
  128, k 16): the whole first chunk, plus 4,096 seeded rows spread over all
  128 chunks (32 per chunk).

Rows whose oracle k-th and (k+1)-th block scores lie within the 1e-3 relative
tie band may hold another valid selection; those rows are compared with the
oracle re-run on the GPU's ids (page "MiniMax wird duenn", atlascloud.ai,
section 1, Steps 1 and 2).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from block_sparse_long_12_b200.inputs import WORKLOADS, make_inputs, to_numpy_raw
from parity import TOL_O, check_ids_row

pytestmark = pytest.mark.gpu

TOL_LSE_PREFILL = 1e-2  # P is rounded to bf16 before P.V on the tensor cores


def gpu_prefill(inp, w, chunk):
    """Index branch then sparse branch for every chunk; returns ids, o, lse of the whole sequence."""
    from block_sparse_long_12_b200 import _lib, api
    T = w.max_seq_len
    ids = torch.full((1, T, w.n_kv_heads, w.top_k), -7, dtype=torch.int32, device="cuda")
    o = torch.full_like(inp["q"], float("nan"))
    lse = torch.full((1, T, w.n_q_heads), float("nan"), device="cuda")
    plist = []
    for c0 in range(0, T, chunk):
        n = min(chunk, T - c0)
        plist.append((c0, n, api.make_params(batch=1, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads,
                                             n_idx_k_heads=w.n_idx_k_heads, head_dim=w.head_dim, idx_dim=w.idx_dim,
                                             block_size=w.block_size, top_k=w.top_k, max_seq_len=T,
                                             dtype=_lib.MSA_BF16, q_len=n, q_start=c0)))
    ws_i = api.workspace([p for _, _, p in plist], _lib.MSA_ENTRY_PREFILL_INDEX_TOPK, "cuda")
    ws_a = api.workspace([p for _, _, p in plist], _lib.MSA_ENTRY_ATTN_PREFILL, "cuda")
    for c0, n, p in plist:
        _lib.msa_prefill_index_topk(p, inp["q_idx"][:, c0:c0 + n], inp["k_idx"], ids[:, c0:c0 + n], None, ws_i)
        _lib.msa_sparse_attn_prefill(p, inp["q"][:, c0:c0 + n], inp["k"], inp["v"], ids[:, c0:c0 + n],
                                     o[:, c0:c0 + n], lse[:, c0:c0 + n], ws_a)
    torch.cuda.synchronize()
    assert _lib.msa_get_device_status(ws_i) == 0 and _lib.msa_get_device_status(ws_a) == 0
    return ids, o, lse


def check_chunk(w, x_full, q_chunk, qi_chunk, c0, n, ts, ids_g, o_g, lse_g):
    """Oracle Steps 1 and 2 for chunk rows ts (relative to c0, sorted); ids_g/o_g/lse_g hold the GPU's
    values of those rows.  Returns (tie rows, max |o| error, max |lse| error)."""
    p = oracle.Params(1, w.n_q_heads, w.n_kv_heads, w.n_idx_k_heads, w.head_dim, w.idx_dim, w.block_size, w.top_k,
                      n, c0, w.max_seq_len, "bf16", w.softmax_scale, prefill=True)
    rows = [(0, int(t)) for t in ts]
    ref = oracle.msa_rows(p, None, q_chunk, qi_chunk, x_full["k"], x_full["v"], x_full["k_idx"], rows)
    xo = {"q_idx": qi_chunk, "k_idx": x_full["k_idx"]}
    tie = []
    for i, t in enumerate(ts):
        for g in range(w.n_kv_heads):
            if not check_ids_row(p, xo, 0, int(t), g, c0 + int(t), ids_g[i, g], ref["ids"][i, g], ref["kth"][i, g],
                                 ref["kth_next"][i, g], where=f"pos={c0 + int(t)} g={g}",
                                 ref_scores=ref["top_scores"][i, g]):
                tie.append(i)
    tie = sorted(set(tie))
    o_ref, lse_ref = ref["o"], ref["lse"]
    if tie:
        ids_in = ref["ids"].copy()
        for i in tie:
            ids_in[i] = ids_g[i]
        rerun = oracle.msa_rows(p, None, q_chunk, qi_chunk, x_full["k"], x_full["v"], x_full["k_idx"], rows,
                                ids_in=ids_in)
        for i in tie:
            o_ref[i], lse_ref[i] = rerun["o"][i], rerun["lse"][i]
    err_o = float(np.abs(o_g - o_ref).max())
    err_l = float(np.abs(lse_g - lse_ref).max())
    assert err_o <= TOL_O["bf16"], f"chunk at {c0}: max |o - oracle| = {err_o}"
    assert err_l <= TOL_LSE_PREFILL, f"chunk at {c0}: max |lse - oracle| = {err_l}"
    return len(tie), err_o, err_l


def test_prefill_16k_every_row_ids_and_outputs():
    """16K causal prefill, whole sequence as one chunk: ids, outputs and LSE of all 16,384 rows."""
    w = WORKLOADS["prefill_causal_16k"]
    inp = make_inputs(w, device="cuda")
    T = w.max_seq_len
    ids, o, lse = gpu_prefill(inp, w, T)
    x = {n: to_numpy_raw(inp[n]) for n in ("q", "q_idx", "k", "v", "k_idx")}
    ts = np.arange(T)
    check_chunk(w, x, x["q"], x["q_idx"], 0, T, ts, ids[0].cpu().numpy(), o[0].float().cpu().numpy(),
                lse[0].cpu().numpy())


def test_prefill_1m_first_chunk_and_4096_rows_over_all_chunks():
    """1M-token prefill in 8192-token chunks: the first chunk row by row, then 32 seeded rows of every
    one of the 128 chunks, ids and outputs against the oracle's own selection."""
    w = WORKLOADS["prefill_causal_1m"]
    inp = make_inputs(w, device="cuda")
    C, T = w.chunk, w.max_seq_len
    ids, o, lse = gpu_prefill(inp, w, C)
    del inp["hot"]
    x = {n: to_numpy_raw(inp[n]) for n in ("k", "v", "k_idx")}
    rng = np.random.default_rng(5005)
    q_buf = np.zeros((1, C, w.n_q_heads, w.head_dim), np.uint16)
    checked = 0
    for c in range(T // C):
        c0 = c * C
        if c == 0:
            ts = np.arange(C)
        else:
            ts = np.sort(rng.choice(C, 32, replace=False))
        sel = torch.from_numpy(ts).cuda() + c0
        q_buf[0, ts] = to_numpy_raw(inp["q"][0, sel])
        qi_chunk = to_numpy_raw(inp["q_idx"][:, c0:c0 + C])
        check_chunk(w, x, q_buf, qi_chunk, c0, C, ts, ids[0, sel].cpu().numpy(), o[0, sel].float().cpu().numpy(),
                    lse[0, sel].cpu().numpy())
        q_buf[0, ts] = 0
        checked += len(ts)
    assert checked == C + 32 * (T // C - 1)
