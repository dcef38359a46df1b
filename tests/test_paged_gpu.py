"""Paged caches: the K, V and index-K caches as pools of block-sized pages named by a block table.

Every entry reads a page where it would have read a block of the contiguous cache, so on the same
values a paged call must give bit-for-bit the contiguous call's ids and outputs (the work split
depends only on the lengths); the contiguous path itself is checked against the fp64 oracle, and
one case here is checked against the oracle directly.  Pages are laid out in a seeded random order
with unused pages between them."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from block_sparse_long_12_b200.inputs import WORKLOADS, make_inputs
from parity import compare_decode, oracle_params, to_np

pytestmark = pytest.mark.gpu


def paginate(inp, block_size, seed=0, spare=7):
    """Pools [n_pages, H, Bk, row] holding every block of k, v and k_idx at a random page, and the table."""
    k, v, ki = inp["k"], inp["v"], inp["k_idx"]
    B, G, L, D = k.shape
    nb = -(-L // block_size)
    n_pages = B * nb + spare
    g = torch.Generator().manual_seed(seed)
    perm = torch.randperm(n_pages, generator=g)[: B * nb].to(torch.int32)
    table = perm.view(B, nb).contiguous()
    pad = nb * block_size - L

    def pool(x):
        H, row = x.shape[1], x.shape[3]
        xp = torch.nn.functional.pad(x, (0, 0, 0, pad)) if pad else x
        blocks = xp.view(B, H, nb, block_size, row).permute(0, 2, 1, 3, 4).reshape(B * nb, H, block_size, row)
        out = torch.full((n_pages, H, block_size, row), float("nan"), dtype=x.dtype, device=x.device)
        out[table.view(-1).long().to(x.device)] = blocks
        return out
    return pool(k), pool(v), pool(ki), table.to(k.device), n_pages


def fused(inp, w, paged=None, top_k=None, force=False):
    from block_sparse_long_12_b200 import _lib, api
    q, q_idx, lens = inp["q"], inp["q_idx"], inp["seq_lens"]
    k, v, ki = (inp["k"], inp["v"], inp["k_idx"]) if paged is None else paged[:3]
    kk = top_k or w.top_k
    flags = _lib.MSA_FORCE_SINK_LOCAL if force else 0
    p = api.make_params(batch=w.batch, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads, n_idx_k_heads=w.n_idx_k_heads,
                        head_dim=w.head_dim, idx_dim=w.idx_dim, block_size=w.block_size, top_k=kk,
                        max_seq_len=w.max_seq_len, dtype=api.dtype_code(q), seq_lens=lens, flags=flags,
                        block_table=None if paged is None else paged[3], n_pages=0 if paged is None else paged[4])
    ws = api.workspace(p, _lib.MSA_ENTRY_DECODE_FUSED, "cuda")
    o = torch.empty_like(q)
    ids = torch.empty(w.batch, 1, w.n_kv_heads, kk, dtype=torch.int32, device="cuda")
    lse = torch.empty(w.batch, 1, w.n_q_heads, device="cuda")
    _lib.msa_decode_fused(p, q, q_idx, k, v, ki, o, ids, lse, ws)
    torch.cuda.synchronize()
    assert _lib.msa_get_device_status(ws) == 0
    return o, ids, lse


@pytest.mark.parametrize("case", [
    dict(name="decode_b8_ctx128k_ragged", batch=3, max_seq_len=40000, min_seq_len=1000, hot_blocks=10),
    dict(name="decode_b8_ctx128k_ragged", batch=2, max_seq_len=20000, min_seq_len=3000, hot_blocks=6, block_size=64,
         top_k=300),                                                   # large k: radix select, many-tile attention
    dict(name="decode_ctx1m_shared_idx", max_seq_len=50000, hot_blocks=8),  # one index-K head for all groups
    dict(name="decode_fp32_ctx4k"),                                  # fp32, 64-token blocks
    dict(name="decode_b8_ctx128k_ragged", batch=2, max_seq_len=30000, min_seq_len=9000, hot_blocks=4, force=True),
], ids=lambda c: "-".join(f"{k}={v}" for k, v in c.items()))
def test_paged_fused_decode_is_bitwise_the_contiguous_one(case):
    case = dict(case)
    name, force = case.pop("name"), case.pop("force", False)
    w = WORKLOADS[name].scaled(**case)
    inp = make_inputs(w, device="cuda")
    ref = fused(inp, w, force=force)
    got = fused(inp, w, paginate(inp, w.block_size, seed=3), force=force)
    assert torch.equal(got[1], ref[1]), "block ids differ"
    assert torch.equal(got[0], ref[0]), "outputs differ"
    assert torch.equal(got[2], ref[2]), "lse differs"


def test_paged_fused_decode_against_the_oracle():
    w = WORKLOADS["decode_b8_ctx128k_ragged"].scaled(batch=2, max_seq_len=24000, min_seq_len=7000, hot_blocks=6)
    inp = make_inputs(w, device="cuda")
    o, ids, lse = fused(inp, w, paginate(inp, w.block_size, seed=11))
    x = to_np(inp)  # the de-paged cache is the contiguous one
    compare_decode(x, oracle_params(x, block_size=w.block_size, top_k=w.top_k), o, ids, lse)


def test_paged_dense_and_given_ids_attention():
    from block_sparse_long_12_b200 import _lib, api
    w = WORKLOADS["decode_b8_ctx128k_ragged"].scaled(batch=2, max_seq_len=20000, min_seq_len=5000, hot_blocks=0)
    inp = make_inputs(w, device="cuda")
    paged = paginate(inp, w.block_size, seed=5)
    rng = np.random.default_rng(0)
    nb = (inp["seq_lens"].cpu().numpy() + w.block_size - 1) // w.block_size
    ids = torch.from_numpy(np.stack([[rng.choice(nb[b], w.top_k, replace=False) for _ in range(w.n_kv_heads)]
                                     for b in range(w.batch)])[:, None].astype(np.int32)).cuda()
    for dense in (False, True):
        outs = []
        for pg in (None, paged):
            k, v = (inp["k"], inp["v"]) if pg is None else pg[:2]
            p = api.make_params(batch=w.batch, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads,
                                n_idx_k_heads=w.n_idx_k_heads, head_dim=w.head_dim, idx_dim=w.idx_dim,
                                block_size=w.block_size, top_k=w.top_k, max_seq_len=w.max_seq_len,
                                dtype=_lib.MSA_BF16, seq_lens=inp["seq_lens"], flags=_lib.MSA_DENSE if dense else 0,
                                block_table=None if pg is None else pg[3], n_pages=0 if pg is None else pg[4])
            ws = api.workspace(p, _lib.MSA_ENTRY_ATTN_DECODE, "cuda")
            o = torch.empty_like(inp["q"])
            lse = torch.empty(w.batch, 1, w.n_q_heads, device="cuda")
            _lib.msa_sparse_attn_decode(p, inp["q"], k, v, None if dense else ids, o, lse, ws)
            torch.cuda.synchronize()
            outs.append((o, lse))
        assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1]), f"dense={dense}"


def test_paged_prefill_chunk_is_bitwise_the_contiguous_one():
    from block_sparse_long_12_b200 import _lib, api
    w = WORKLOADS["prefill_causal_1m"].scaled(max_seq_len=20000, batch=2, hot_blocks=6, seed=41)
    inp = make_inputs(w, device="cuda")
    paged = paginate(inp, w.block_size, seed=9)
    q_start, T = 11000, 5000
    res = []
    for pg in (None, paged):
        k, v, ki = (inp["k"], inp["v"], inp["k_idx"]) if pg is None else pg[:3]
        p = api.make_params(batch=2, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads, n_idx_k_heads=w.n_idx_k_heads,
                            head_dim=w.head_dim, idx_dim=w.idx_dim, block_size=w.block_size, top_k=w.top_k,
                            max_seq_len=w.max_seq_len, dtype=_lib.MSA_BF16, q_len=T, q_start=q_start,
                            block_table=None if pg is None else pg[3], n_pages=0 if pg is None else pg[4])
        ids = torch.empty(2, T, w.n_kv_heads, w.top_k, dtype=torch.int32, device="cuda")
        o = torch.empty(2, T, w.n_q_heads, w.head_dim, dtype=torch.bfloat16, device="cuda")
        lse = torch.empty(2, T, w.n_q_heads, device="cuda")
        wi = api.workspace(p, _lib.MSA_ENTRY_PREFILL_INDEX_TOPK, "cuda")
        wa = api.workspace(p, _lib.MSA_ENTRY_ATTN_PREFILL, "cuda")
        _lib.msa_prefill_index_topk(p, inp["q_idx"][:, q_start:q_start + T].contiguous(), ki, ids, None, wi)
        _lib.msa_sparse_attn_prefill(p, inp["q"][:, q_start:q_start + T].contiguous(), k, v, ids, o, lse, wa)
        torch.cuda.synchronize()
        assert _lib.msa_get_device_status(wi) == 0 and _lib.msa_get_device_status(wa) == 0
        res.append((ids, o, lse))
    assert torch.equal(res[0][0], res[1][0]), "prefill ids differ"
    assert torch.equal(res[0][1], res[1][1]), "prefill outputs differ"
    assert torch.equal(res[0][2], res[1][2]), "prefill lse differs"
