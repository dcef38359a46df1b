"""Context-parallel decode with the CUDA library doing every local step, the ranks emulated one
after another on one GPU (no collective): each slice's TopK candidates and (output, log-sum-exp)
partials are stacked as the all-gathers would stack them.  The selection must be bit for bit the
unsharded fused decode's (the block scores are the same fp32 sums), the outputs must match it and
the fp64 oracle at the bf16 tolerance."""
from __future__ import annotations

import pytest
import torch

from block_sparse_long_12_b200.inputs import WORKLOADS, make_inputs
from parity import compare_decode, oracle_params, to_np

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("world,case", [
    (2, dict(batch=3, max_seq_len=40000, min_seq_len=9000, hot_blocks=12)),
    (4, dict(batch=2, max_seq_len=65536, min_seq_len=20000, hot_blocks=16, n_idx_k_heads=1)),
], ids=["world2", "world4-shared-index-head"])
def test_emulated_ranks_match_the_fused_decode(world, case):
    from block_sparse_long_12_b200 import api
    from block_sparse_long_12_b200 import context_parallel as cp
    w = WORKLOADS["decode_b8_ctx128k_ragged"].scaled(**case)
    inp = make_inputs(w, device="cuda")
    q, q_idx, k, v, ki, lens = (inp[n] for n in ("q", "q_idx", "k", "v", "k_idx", "seq_lens"))
    o_ref, ids_ref, lse_ref = api.decode(q, q_idx, k, v, ki, lens, block_size=w.block_size, top_k=w.top_k)
    backend = cp.LibraryBackend(w.n_q_heads, w.block_size)
    slices = cp.slices_of(w.max_seq_len, w.block_size, world)
    part = lambda t, sl: t[:, :, sl.start:sl.start + sl.length].contiguous()  # noqa: E731
    cands = [cp.local_candidates(backend, q_idx, part(ki, sl), lens, sl, block_size=w.block_size, top_k=w.top_k)
             for sl in slices]
    _, ids = cp.select_global_topk(torch.stack([c[0] for c in cands]), torch.stack([c[1] for c in cands]), w.top_k)
    parts = [cp.local_partial(backend, q, part(k, sl), part(v, sl), lens, sl, ids, block_size=w.block_size)
             for sl in slices]
    o, lse = cp.merge_partials(torch.stack([p[0] for p in parts]), torch.stack([p[1] for p in parts]))
    torch.cuda.synchronize()
    assert torch.equal(ids, ids_ref[:, 0]), "selection differs from the unsharded decode"
    assert (o - o_ref[:, 0].double()).abs().max().item() <= 2e-2
    assert (lse - lse_ref[:, 0].double()).abs().max().item() <= 1e-3
    x = to_np(inp)
    compare_decode(x, oracle_params(x, block_size=w.block_size, top_k=w.top_k), o.unsqueeze(1).to(torch.bfloat16),
                   ids.unsqueeze(1), lse.unsqueeze(1).float())
