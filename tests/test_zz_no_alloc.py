"""The allocation-free decode entry point, msa_decode_fused_noalloc.

Some callers of this library get only their input and output buffers and
cannot hand over scratch memory (plugin or foreign-function hosts without a
workspace slot, serving loops that allocate nothing after start-up).  For
them the library keeps a fixed scratch array in device memory.  This test
calls that entry through the C ABI and checks, on two calls in a row, that
it returns what msa_decode_fused returns with a caller-supplied workspace.
It sits in a file that pytest collects last, so that a failure here comes
after every other test has run; it also passes on its own in a fresh process.
"""
from __future__ import annotations

import ctypes

import pytest
import torch

from block_sparse_long_12_b200.inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu


def test_noalloc_matches_workspace_entry_on_two_calls():
    from block_sparse_long_12_b200 import _lib, api
    w = WORKLOADS["decode_b8_ctx128k_ragged"].scaled(batch=3, max_seq_len=40000, min_seq_len=1000, hot_blocks=12)
    inp = make_inputs(w, device="cuda")
    q, q_idx, k, v, k_idx, lens = (inp[n] for n in ("q", "q_idx", "k", "v", "k_idx", "seq_lens"))
    p = api.params_from(q, q_idx, k, k_idx, block_size=w.block_size, top_k=w.top_k, seq_lens=lens)
    assert _lib.msa_workspace_size(p, _lib.MSA_ENTRY_DECODE_FUSED) <= 8 << 20

    ref_o, ref_ids, ref_lse = api.decode(q, q_idx, k, v, k_idx, lens, block_size=w.block_size, top_k=w.top_k)
    torch.cuda.synchronize()
    for call in range(2):
        o = torch.full_like(q, float("nan"))
        ids = torch.full_like(ref_ids, -7)
        lse = torch.full_like(ref_lse, float("nan"))
        _lib.msa_decode_fused_noalloc(p, q, q_idx, k, v, k_idx, o, ids, lse)
        torch.cuda.synchronize()
        assert torch.equal(ids, ref_ids), f"call {call}: block ids differ"
        assert (o.float() - ref_o.float()).abs().max().item() <= 2e-2, f"call {call}: outputs differ"
        assert (lse - ref_lse).abs().max().item() <= 1e-3, f"call {call}: lse differs"
        # no bounded wait ran out: the fixed scratch's status word reads MSA_OK
        assert _lib.msa_noalloc_get_status() == _lib.MSA_OK, f"call {call}: status word set"
    _lib.msa_noalloc_clear_status()
    assert _lib.msa_noalloc_get_status() == _lib.MSA_OK


def test_noalloc_rejects_shapes_beyond_its_scratch():
    from block_sparse_long_12_b200 import _lib, api
    # 64 sequences of 1M tokens would need far more than the fixed 8 MiB of scratch
    p = api.make_params(batch=64, n_q_heads=64, n_kv_heads=8, n_idx_k_heads=8, head_dim=128, idx_dim=64,
                        block_size=128, top_k=32, max_seq_len=1 << 20, dtype=_lib.MSA_BF16)
    p.seq_lens = 0x10000  # never read: the call is refused before anything is enqueued
    a = 0x10000
    rc = _lib.lib().msa_decode_fused_noalloc(ctypes.byref(p), a, a, a, a, a, a, None, None, None)
    assert rc == _lib.MSA_ERR_WORKSPACE
    assert "fixed scratch" in _lib.lib().msa_last_error_string().decode()
