"""msa_decode_append: the new token's K, V and index key land at position seq_lens[b] - 1 of every
sequence, in contiguous and in paged caches, and nothing else of the caches changes."""
from __future__ import annotations

import pytest
import torch

from block_sparse_long_12_b200.inputs import WORKLOADS, make_inputs
from test_paged_gpu import paginate

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("paged", [False, True], ids=["contiguous", "paged"])
@pytest.mark.parametrize("name", ["decode_b8_ctx128k_ragged", "decode_fp32_ctx4k"])
def test_append_writes_the_new_token_only(paged, name):
    from block_sparse_long_12_b200 import _lib, api
    w = WORKLOADS[name]
    if name == "decode_b8_ctx128k_ragged":
        w = w.scaled(batch=3, max_seq_len=5000, min_seq_len=100, hot_blocks=0)
    inp = make_inputs(w, device="cuda")
    lens = inp["seq_lens"]
    gen = torch.Generator(device="cuda").manual_seed(7)
    dt = inp["k"].dtype
    k_new = torch.randn(w.batch, w.n_kv_heads, w.head_dim, generator=gen, device="cuda").to(dt)
    v_new = torch.randn(w.batch, w.n_kv_heads, w.head_dim, generator=gen, device="cuda").to(dt)
    ki_new = torch.randn(w.batch, w.n_idx_k_heads, w.idx_dim, generator=gen, device="cuda").to(dt)
    pg = paginate(inp, w.block_size, seed=2) if paged else None
    k, v, ki = (inp["k"].clone(), inp["v"].clone(), inp["k_idx"].clone()) if pg is None else pg[:3]
    before = (k.clone(), v.clone(), ki.clone())
    p = api.make_params(batch=w.batch, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads, n_idx_k_heads=w.n_idx_k_heads,
                        head_dim=w.head_dim, idx_dim=w.idx_dim, block_size=w.block_size, top_k=w.top_k,
                        max_seq_len=w.max_seq_len, dtype=api.dtype_code(inp["q"]), seq_lens=lens,
                        block_table=None if pg is None else pg[3], n_pages=0 if pg is None else pg[4])
    _lib.msa_decode_append(p, k_new, v_new, ki_new, k, v, ki)
    torch.cuda.synchronize()
    want = [t.clone() for t in before]
    for b in range(w.batch):
        pos = int(lens[b]) - 1
        if pg is None:
            want[0][b, :, pos], want[1][b, :, pos], want[2][b, :, pos] = k_new[b], v_new[b], ki_new[b]
        else:
            page = int(pg[3][b, pos // w.block_size])
            off = pos % w.block_size
            want[0][page, :, off], want[1][page, :, off], want[2][page, :, off] = k_new[b], v_new[b], ki_new[b]
    for got, exp in zip((k, v, ki), want):
        assert torch.equal(got.view(torch.int16 if dt == torch.bfloat16 else torch.int32),
                           exp.view(torch.int16 if dt == torch.bfloat16 else torch.int32))
