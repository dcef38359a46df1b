"""Failure detection on the GPU without a fault.

Every device wait of the kernels is bounded; when one runs out the kernel
writes MSA_ERR_TIMEOUT into the workspace's status word and returns.  Here a
diagnostic entry waits on an mbarrier phase that nothing completes, under a
1 ms limit, so the timeout path runs for real: the status must read
MSA_ERR_TIMEOUT, clearing it must work, and the same workspace must then give
a decode step that matches the fp64 oracle."""
from __future__ import annotations

import time

import pytest
import torch

from block_sparse_long_12_b200.inputs import WORKLOADS, make_inputs
from parity import compare_decode, oracle_params, to_np

pytestmark = pytest.mark.gpu


def test_wait_timeout_reaches_status_and_workspace_recovers():
    from block_sparse_long_12_b200 import _lib, api
    w = WORKLOADS["decode_b8_ctx128k_ragged"].scaled(batch=2, max_seq_len=20000, min_seq_len=5000, hot_blocks=8)
    inp = make_inputs(w, device="cuda")
    q, q_idx, k, v, k_idx, lens = (inp[n] for n in ("q", "q_idx", "k", "v", "k_idx", "seq_lens"))
    p = api.params_from(q, q_idx, k, k_idx, block_size=w.block_size, top_k=w.top_k, seq_lens=lens)
    ws = api.workspace(p, _lib.MSA_ENTRY_DECODE_FUSED, "cuda")
    assert _lib.msa_get_device_status(ws) == _lib.MSA_OK

    _lib.msa_set_wait_limit(ws, 1_000_000)  # 1 ms
    t0 = time.perf_counter()
    _lib.msa_diag_wait_timeout(ws)
    torch.cuda.synchronize()
    took = time.perf_counter() - t0
    assert _lib.msa_get_device_status(ws) == _lib.MSA_ERR_TIMEOUT
    assert took < 0.5, f"the 1 ms wait took {took:.3f} s"
    # the context is still usable
    assert torch.cuda.synchronize() is None and float(torch.ones(4, device="cuda").sum()) == 4.0

    _lib.msa_clear_device_status(ws)  # also restores the default wait limit
    assert _lib.msa_get_device_status(ws) == _lib.MSA_OK

    o, ids, lse = api.decode(q, q_idx, k, v, k_idx, lens, block_size=w.block_size, top_k=w.top_k, ws=ws)
    torch.cuda.synchronize()
    assert _lib.msa_get_device_status(ws) == _lib.MSA_OK
    x = to_np(inp)
    compare_decode(x, oracle_params(x, block_size=w.block_size, top_k=w.top_k), o, ids, lse)


def test_default_wait_limit_restored_by_zero():
    """A limit of 0 means the default (one second): the diagnostic then takes about a second."""
    from block_sparse_long_12_b200 import _lib
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    _lib.msa_set_wait_limit(ws, 50_000_000)  # 50 ms
    t0 = time.perf_counter()
    _lib.msa_diag_wait_timeout(ws)
    torch.cuda.synchronize()
    took = time.perf_counter() - t0
    assert _lib.msa_get_device_status(ws) == _lib.MSA_ERR_TIMEOUT
    assert 0.04 <= took < 0.6, took
    _lib.msa_clear_device_status(ws)
    _lib.msa_set_wait_limit(ws, 0)
    t0 = time.perf_counter()
    _lib.msa_diag_wait_timeout(ws)
    torch.cuda.synchronize()
    took = time.perf_counter() - t0
    assert _lib.msa_get_device_status(ws) == _lib.MSA_ERR_TIMEOUT
    assert 0.9 <= took < 3.0, took
    _lib.msa_clear_device_status(ws)
    assert _lib.msa_get_device_status(ws) == _lib.MSA_OK
