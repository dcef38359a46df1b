"""Shared helpers of the GPU parity tests: run the oracle on the exact bytes
the GPU saw and compare, with the near-tie rule for block ids.

Rule for ids: bit-exact, except in a row whose oracle k-th and (k+1)-th block
scores are within 1e-3 relative of each other.  There the GPU ids must be
unique and causal-valid, contain every block the oracle ranks above the tie
band, take the rest from inside the band, and that row's outputs are then
compared against the oracle re-run with the GPU's own ids.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
from block_sparse_long_12_b200.inputs import to_numpy_raw

TIE_REL = 1e-3
TOL_O = {"f32": 1e-4, "bf16": 2e-2}
TOL_LSE = {"f32": 1e-4, "bf16": 1e-3}


def oracle_params(x: dict, *, block_size, top_k, prefill=False, q_start=0, dense=False, softmax_scale=None,
                  force_sink_local=False):
    B, Tq, Hq, D = x["q"].shape
    G, L = x["k"].shape[1], x["k"].shape[2]
    dtype = "f32" if x["q"].dtype == np.float32 else "bf16"
    return oracle.Params(B, Hq, G, x["k_idx"].shape[1], D, x["q_idx"].shape[-1], block_size, top_k, Tq, q_start, L,
                         dtype, softmax_scale if softmax_scale is not None else 1.0 / math.sqrt(D),
                         prefill=prefill, dense=dense, force_sink_local=force_sink_local)


def check_forced(ids: np.ndarray, pos_of, block_size: int, top_k: int):
    """Every row of ids [B, T, G, k] holds block 0 first and the row's own block second (when it
    has two valid blocks and k >= 2); pos_of(b, t) gives the row's position."""
    B, T, G, _ = ids.shape
    for b in range(B):
        for t in range(T):
            pos = pos_of(b, t)
            if pos < 0:
                continue
            own = pos // block_size
            for g in range(G):
                assert ids[b, t, g, 0] == 0, (b, t, g, ids[b, t, g])
                if own > 0 and top_k >= 2:
                    assert ids[b, t, g, 1] == own, (b, t, g, ids[b, t, g])


def to_np(inputs: dict) -> dict:
    return {n: to_numpy_raw(inputs[n]) for n in ("q", "q_idx", "k", "v", "k_idx", "seq_lens")}


def oracle_block_score(p: oracle.Params, x: dict, b: int, t: int, g: int, pos: int, n: int) -> float:
    s = oracle.token_scores(p, x["q_idx"], x["k_idx"], b, t, g, pos)
    return float(oracle.block_scores(p, s, pos)[n])


def _close(a, b):
    return abs(a - b) <= TIE_REL * max(abs(a), abs(b))


def check_ids_row(p, x, b, t, g, pos, gpu_ids, ref_ids, kth, kth_next, where="", ref_scores=None):
    """Returns True if the row is exact, False if it passed under the near-tie rule (raises otherwise).

    The same set in another order is exact when every position that differs
    holds two blocks whose oracle scores are within the tie tolerance (the
    list is ordered by score, which fp32 and fp64 may order differently)."""
    gpu_ids = [int(i) for i in gpu_ids]
    ref_ids = [int(i) for i in ref_ids]
    if gpu_ids == ref_ids:
        return True
    cache = {}

    def block_score(i):
        # the row's block scores, computed once (long rows and large k make per-id calls costly)
        if "S" not in cache:
            s = oracle.token_scores(p, x["q_idx"], x["k_idx"], b, t, g, pos)
            cache["S"] = oracle.block_scores(p, s, pos)
        return float(cache["S"][i])
    if sorted(gpu_ids) == sorted(ref_ids):
        def score(i):
            if ref_scores is not None:
                return float(ref_scores[ref_ids.index(i)])
            return block_score(i)
        for a_, r_ in zip(gpu_ids, ref_ids):
            if a_ != r_:
                assert a_ >= 0 and r_ >= 0 and _close(score(a_), score(r_)), \
                    f"{where}: order differs beyond ties: gpu {gpu_ids} oracle {ref_ids}"
        return True
    tie = (not math.isnan(kth) and not math.isnan(kth_next)
           and abs(kth - kth_next) <= TIE_REL * max(abs(kth), abs(kth_next)))
    assert tie, f"{where}: ids differ without a near-tie: gpu {gpu_ids} oracle {ref_ids} (kth {kth}, next {kth_next})"
    nb = pos // p.block_size + 1
    sel = [i for i in gpu_ids if i >= 0]
    assert len(sel) == len(set(sel)) == min(nb, p.top_k), f"{where}: gpu ids not unique/complete {gpu_ids}"
    assert all(0 <= i < nb for i in sel), f"{where}: gpu id not causal-valid {gpu_ids}"
    band_lo = kth_next - TIE_REL * max(abs(kth), abs(kth_next))
    band_hi = kth + TIE_REL * max(abs(kth), abs(kth_next))
    sel_set, ref_set = set(sel), set(ref_ids)
    for i in ref_ids:
        if i >= 0 and block_score(i) > band_hi:
            assert i in sel_set, f"{where}: block {i} above the tie band missing from gpu ids {gpu_ids}"
    for i in sel:
        if i not in ref_set:
            sc = block_score(i)
            assert band_lo <= sc <= band_hi, f"{where}: gpu block {i} (score {sc}) outside the tie band"
    return False


def compare_decode(x: dict, p: oracle.Params, o_gpu, ids_gpu, lse_gpu, batches=None, tol=None, tol_lse=None):
    """Compare a decode step ([B,1,...] tensors) with the oracle on every sequence in `batches`."""
    B = p.batch
    batches = list(range(B)) if batches is None else batches
    tol_o = tol if tol is not None else TOL_O[p.dtype]
    tol_l = tol_lse if tol_lse is not None else TOL_LSE[p.dtype]
    rows = [(b, 0) for b in batches]
    ref = oracle.msa_rows(p, x["seq_lens"], x["q"], x["q_idx"], x["k"], x["v"], x["k_idx"], rows)
    o = o_gpu.float().cpu().numpy()
    lse = lse_gpu.float().cpu().numpy() if lse_gpu is not None else None
    ids = ids_gpu.cpu().numpy() if ids_gpu is not None else None
    G = p.n_kv_heads
    r = p.n_q_heads // G
    tie_rows = []
    for i, b in enumerate(batches):
        pos = int(x["seq_lens"][b]) - 1
        if ids is not None and not p.dense:
            for g in range(G):
                exact = check_ids_row(p, x, b, 0, g, pos, ids[b, 0, g], ref["ids"][i, g], ref["kth"][i, g],
                                      ref["kth_next"][i, g], where=f"b={b} g={g}", ref_scores=ref["top_scores"][i, g])
                if not exact:
                    tie_rows.append((i, b, g))
    o_ref = ref["o"].copy()
    lse_ref = ref["lse"].copy()
    if tie_rows:
        ids_in = ref["ids"].copy()
        for (i, b, g) in tie_rows:
            ids_in[i, g] = ids[b, 0, g]
        rerun = oracle.msa_rows(p, x["seq_lens"], x["q"], x["q_idx"], x["k"], x["v"], x["k_idx"], rows, ids_in=ids_in)
        for (i, b, g) in tie_rows:
            o_ref[i, g * r:(g + 1) * r] = rerun["o"][i, g * r:(g + 1) * r]
            lse_ref[i, g * r:(g + 1) * r] = rerun["lse"][i, g * r:(g + 1) * r]
    err_o = np.abs(o[batches, 0] - o_ref).max()
    assert err_o <= tol_o, f"max |o - oracle| = {err_o} > {tol_o}"
    if lse is not None:
        err_l = np.abs(lse[batches, 0] - lse_ref).max()
        assert err_l <= tol_l, f"max |lse - oracle| = {err_l}"
    return {"err_o": float(err_o), "tie_rows": len(tie_rows)}


def cuda_inputs(w, seed=None):
    from block_sparse_long_12_b200.inputs import make_inputs
    return make_inputs(w, device="cuda", seed=seed)


def sync():
    torch.cuda.synchronize()
