"""Context-parallel decode on CPU ranks (gloo): the exchange of TopK candidates and of (output,
log-sum-exp) partials, with every local step done by the fp64 oracle on the rank's slice.  The
ranks' common result must be the single-rank oracle's: block ids bit for bit, outputs and log-sum-
exps to 1e-12 (page "MiniMax wird duenn", atlascloud.ai, section 1, Steps 1 and 2: a selection of
the k best blocks per group, then exact softmax attention over them)."""
from __future__ import annotations

import math
import os
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


class OracleBackend:
    """The two local steps of a rank by the fp64 oracle (decode rows, contiguous slice caches)."""

    def __init__(self, w):
        self.w = w

    def _params(self, x, k):
        import oracle
        w = self.w
        B, _, Hq, D = x["q"].shape
        G, L = x["k"].shape[1], x["k"].shape[2]
        return oracle.Params(B, Hq, G, x["k_idx"].shape[1], D, x["q_idx"].shape[-1], w.block_size, k, 1, 0, L,
                             w.dtype, 1.0 / math.sqrt(D))

    def block_topk(self, q_idx, k_idx, lens, k):
        import oracle
        from block_sparse_long_12_b200.inputs import to_numpy_raw
        B, _, G, _ = q_idx.shape
        scores = torch.full((B, G, k), float("-inf"), dtype=torch.float64)
        ids = torch.full((B, G, k), -1, dtype=torch.int32)
        x = {"q": np.zeros((B, 1, G, 8), np.uint16), "q_idx": to_numpy_raw(q_idx), "k": np.zeros((B, G, k_idx.shape[2], 8), np.uint16),
             "k_idx": to_numpy_raw(k_idx)}
        rows = [(b, 0) for b in range(B) if int(lens[b]) > 0]
        if rows:
            p = self._params(x, k)
            unused = np.zeros(8, np.uint16)
            ref = oracle.msa_rows(p, lens.numpy(), unused, x["q_idx"], unused, unused, x["k_idx"], rows,
                                  attention=False)
            for i, (b, _) in enumerate(rows):
                scores[b] = torch.from_numpy(ref["top_scores"][i])
                ids[b] = torch.from_numpy(ref["ids"][i])
        return scores, ids

    def attend(self, q, k, v, lens, ids):
        import oracle
        from block_sparse_long_12_b200.inputs import to_numpy_raw
        B, _, Hq, D = q.shape
        o = torch.zeros(B, Hq, D, dtype=torch.float64)
        lse = torch.full((B, Hq), float("-inf"), dtype=torch.float64)
        x = {"q": to_numpy_raw(q), "k": to_numpy_raw(k), "v": to_numpy_raw(v),
             "q_idx": np.zeros((B, 1, k.shape[1], 8), np.uint16), "k_idx": np.zeros((B, k.shape[1], k.shape[2], 8), np.uint16)}
        rows = [(b, 0) for b in range(B) if int(lens[b]) > 0]
        if rows:
            p = self._params(x, ids.shape[-1])
            unused = np.zeros(8, np.uint16)
            ref = oracle.msa_rows(p, lens.numpy(), x["q"], unused, x["k"], x["v"], unused, rows,
                                  ids_in=np.stack([ids[b].numpy() for (b, _) in rows]))
            for i, (b, _) in enumerate(rows):
                got = torch.from_numpy(ref["lse"][i])
                lse[b] = got
                o[b] = torch.where(torch.isfinite(got).unsqueeze(-1), torch.from_numpy(ref["o"][i]), torch.zeros(1, dtype=torch.float64))
        return o, lse


def workload():
    from block_sparse_long_12_b200.inputs import WORKLOADS
    return WORKLOADS["decode_b8_ctx128k_ragged"].scaled(batch=3, max_seq_len=2900, min_seq_len=300, n_q_heads=8,
                                                        n_kv_heads=2, n_idx_k_heads=2, head_dim=64, idx_dim=32,
                                                        block_size=64, top_k=6, hot_blocks=5, seed=77)


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        oracle.build()
        from block_sparse_long_12_b200 import context_parallel as cp
        from block_sparse_long_12_b200.inputs import make_inputs
        w = workload()
        x = make_inputs(w)  # the same seeded values on every rank
        sl = cp.slices_of(w.max_seq_len, w.block_size, world)[rank]
        part = lambda t: t[:, :, sl.start:sl.start + sl.length].contiguous()  # noqa: E731
        o, lse, ids = cp.decode_step(OracleBackend(w), x["q"], x["q_idx"], part(x["k"]), part(x["v"]),
                                     part(x["k_idx"]), x["seq_lens"], sl, block_size=w.block_size, top_k=w.top_k)
        out[rank] = (o.numpy(), lse.numpy(), ids.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_context_parallel_decode_equals_single_rank_oracle(world):
    import oracle
    sys.path.insert(0, ROOT)
    from block_sparse_long_12_b200.inputs import make_inputs, to_numpy_raw
    port = 29600 + world * 17 + (os.getpid() % 500)
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    w = workload()
    x = {n: to_numpy_raw(t) for n, t in make_inputs(w).items() if n != "hot"}
    oracle.build()
    p = oracle.Params(w.batch, w.n_q_heads, w.n_kv_heads, w.n_idx_k_heads, w.head_dim, w.idx_dim, w.block_size,
                      w.top_k, 1, 0, w.max_seq_len, w.dtype, w.softmax_scale)
    ref = oracle.msa_rows(p, x["seq_lens"], x["q"], x["q_idx"], x["k"], x["v"], x["k_idx"],
                          [(b, 0) for b in range(w.batch)])
    o0, lse0, ids0 = out[0]
    for r in range(1, world):  # every rank holds the same result
        assert np.array_equal(out[r][2], ids0) and np.array_equal(out[r][0], o0) and np.array_equal(out[r][1], lse0)
    assert np.array_equal(ids0, ref["ids"]), "block ids differ from the single-rank oracle"
    assert np.abs(o0 - ref["o"]).max() <= 1e-12
    assert np.abs(lse0 - ref["lse"]).max() <= 1e-12
    # the selection was spread: more than one rank held selected blocks of some group
    nb_rank = [s.length // w.block_size for s in __import__("block_sparse_long_12_b200.context_parallel",
                                                               fromlist=["x"]).slices_of(w.max_seq_len, w.block_size, world)]
    edges = np.cumsum([0] + nb_rank)
    owners = {int(np.searchsorted(edges, i, side="right")) for i in ids0[ids0 >= 0].ravel()}
    assert len(owners) > 1


def test_global_topk_merge_keeps_the_order():
    """Candidates with equal scores on different ranks: ties go to the lower block id."""
    sys.path.insert(0, ROOT)
    from block_sparse_long_12_b200.context_parallel import select_global_topk
    s = torch.tensor([[[[5.0, 3.0, 3.0, float("-inf")]]], [[[3.0, 3.0, 1.0, 0.5]]]], dtype=torch.float64)
    i = torch.tensor([[[[7, 2, 9, -1]]], [[[4, 11, 30, 31]]]], dtype=torch.int32)
    sc, ids = select_global_topk(s, i, 4)
    assert ids.tolist() == [[[7, 2, 4, 9]]]
    assert sc.tolist() == [[[5.0, 3.0, 3.0, 3.0]]]
    sc, ids = select_global_topk(s[:, :, :, :2], i[:, :, :, :2], 4)  # fewer candidates than k: padded
    assert ids.tolist() == [[[7, 2, 4, 11]]]
