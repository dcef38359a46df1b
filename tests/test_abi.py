"""The C ABI library without a GPU: it loads, exports what include/msa.h
declares, and rejects bad arguments before anything reaches the device."""
from __future__ import annotations

import ctypes
import os
import re
import subprocess

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from block_sparse_long_12_b200 import _lib, build
    build.build()
    return _lib


def declared_symbols():
    hdr = open(os.path.join(ROOT, "include", "msa.h")).read()
    return sorted(set(re.findall(r"MSA_API\s+[\w\s\*]+?\b(msa_\w+)\s*\(", hdr)))


def test_header_declares_the_bound_entry_points(lib):
    assert declared_symbols() == sorted(lib.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    L = lib.lib()
    for name in declared_symbols():
        assert hasattr(L, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", lib.LIB_PATH], capture_output=True, text=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    assert set(declared_symbols()) <= exported
    # nothing else of ours leaks out of the library
    assert {s for s in exported if s.startswith("msa_")} == set(declared_symbols())


def test_flag_values_match_the_header(lib):
    hdr = open(os.path.join(ROOT, "include", "msa.h")).read()
    for name in ("MSA_SCORES_TOKEN", "MSA_SCORES_BLOCKMAX", "MSA_DENSE", "MSA_FORCE_SINK_LOCAL"):
        m = re.search(r"\b" + name + r"\s*=\s*(\d+)", hdr)
        assert m is not None, name
        assert int(m.group(1)) == getattr(lib, name), name


def test_status_strings(lib):
    L = lib.lib()
    for code, name in enumerate(["MSA_OK", "MSA_ERR_INVALID_ARG", "MSA_ERR_UNSUPPORTED", "MSA_ERR_WORKSPACE",
                                 "MSA_ERR_CUDA", "MSA_ERR_TIMEOUT"]):
        assert L.msa_status_string(code).decode() == name


def good_params(lib, **kw):
    from block_sparse_long_12_b200.api import make_params
    base = dict(batch=1, n_q_heads=64, n_kv_heads=8, n_idx_k_heads=8, head_dim=128, idx_dim=64, block_size=128,
                top_k=16, max_seq_len=4096, dtype=lib.MSA_BF16, seq_lens=None)
    base.update(kw)
    p = make_params(**base)
    if p.seq_lens is None:
        p.seq_lens = 0x1000  # a fake device address: never dereferenced, every case below fails first
    return p


BAD = [
    (dict(batch=0), "INVALID_ARG"),
    (dict(n_q_heads=12), "INVALID_ARG"),
    (dict(n_idx_k_heads=3), "INVALID_ARG"),
    (dict(head_dim=96), "UNSUPPORTED"),
    (dict(idx_dim=48), "UNSUPPORTED"),
    (dict(block_size=100), "UNSUPPORTED"),
    (dict(block_size=512), "UNSUPPORTED"),
    (dict(top_k=0), "INVALID_ARG"),
    (dict(top_k=1025), "UNSUPPORTED"),
    (dict(max_seq_len=0), "INVALID_ARG"),
    (dict(softmax_scale=-1.0), "INVALID_ARG"),
    (dict(softmax_scale=float("inf")), "INVALID_ARG"),
    (dict(dtype=7), "INVALID_ARG"),
    (dict(flags=64), "INVALID_ARG"),
    (dict(q_len=2), "INVALID_ARG"),               # decode entries take one query
    (dict(n_q_heads=8 * 32), "UNSUPPORTED"),      # group size 32
    (dict(batch=5000), "UNSUPPORTED"),
]


@pytest.mark.skipif(torch.cuda.is_available(), reason="fake pointers: host-only argument checks")
@pytest.mark.parametrize("kw,status", BAD, ids=lambda v: str(v))
def test_bad_params_rejected_before_launch(lib, kw, status):
    p = good_params(lib, **kw)
    code = getattr(lib, "MSA_ERR_" + status)
    fake = 0x10000
    L = lib.lib()
    ws = ctypes.c_size_t(1 << 30)
    rc = L.msa_decode_fused(ctypes.byref(p), fake, fake, fake, fake, fake, fake, None, None, fake, ws, None)
    assert rc == code, (rc, L.msa_last_error_string())
    assert L.msa_last_error_string().decode() != ""
    with pytest.raises(lib.MsaError):
        lib.msa_workspace_size(p, lib.MSA_ENTRY_DECODE_FUSED)


@pytest.mark.skipif(torch.cuda.is_available(), reason="fake pointers: host-only argument checks")
def test_bad_pointers_rejected_before_launch(lib):
    p = good_params(lib)
    L = lib.lib()
    a, mis = 0x10000, 0x10008
    ws = ctypes.c_size_t(1 << 30)
    ptrs = [a, a, a, a, a, a, None, None, a]
    for i in range(len(ptrs)):
        for bad in ((None,) if ptrs[i] is not None else ()) + (mis,):
            args = list(ptrs)
            args[i] = bad
            rc = L.msa_decode_fused(ctypes.byref(p), *args, ws, None)
            assert rc == lib.MSA_ERR_INVALID_ARG, (i, bad, L.msa_last_error_string())
    # prefill entries check their own shapes: rows beyond the caches
    pp = good_params(lib, q_len=100, q_start=4000)
    rc = L.msa_prefill_index_topk(ctypes.byref(pp), a, a, a, None, a, ws, None)
    assert rc == lib.MSA_ERR_INVALID_ARG
    # large k in prefill: lists of more than 32 blocks pass the checks (then fail on the fake pointers'
    # workspace size, not on top_k)
    pk = good_params(lib, q_len=100, top_k=64)
    assert L.msa_sparse_attn_prefill(ctypes.byref(pk), a, a, a, a, a, None, a, ctypes.c_size_t(64),
                                     None) == lib.MSA_ERR_WORKSPACE
    # index scores need exactly one score granularity
    rc = L.msa_index_score(ctypes.byref(p), a, a, a, a, ws, None)
    assert rc == lib.MSA_ERR_INVALID_ARG
    ps = good_params(lib, flags=lib.MSA_SCORES_TOKEN | lib.MSA_SCORES_BLOCKMAX)
    assert L.msa_index_score(ctypes.byref(ps), a, a, a, a, ws, None) == lib.MSA_ERR_INVALID_ARG
    # fused decode takes only the forced-block flag
    pd = good_params(lib, flags=lib.MSA_DENSE)
    assert L.msa_decode_fused(ctypes.byref(pd), *ptrs, ws, None) == lib.MSA_ERR_INVALID_ARG
    pd = good_params(lib, flags=lib.MSA_DENSE | lib.MSA_FORCE_SINK_LOCAL)
    assert L.msa_decode_fused(ctypes.byref(pd), *ptrs, ws, None) == lib.MSA_ERR_INVALID_ARG
    # forcing blocks applies to selections, not to scores or to attention from given ids
    pf = good_params(lib, flags=lib.MSA_SCORES_BLOCKMAX | lib.MSA_FORCE_SINK_LOCAL)
    assert L.msa_index_score(ctypes.byref(pf), a, a, a, a, ws, None) == lib.MSA_ERR_INVALID_ARG
    pf = good_params(lib, flags=lib.MSA_FORCE_SINK_LOCAL)
    assert L.msa_sparse_attn_decode(ctypes.byref(pf), a, a, a, a, a, None, a, ws, None) == lib.MSA_ERR_INVALID_ARG


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_no_device_reports_cuda_error(lib):
    p = good_params(lib)
    L = lib.lib()
    a = 0x10000
    rc = L.msa_decode_fused(ctypes.byref(p), a, a, a, a, a, a, None, None, a, ctypes.c_size_t(1 << 30), None)
    assert rc == lib.MSA_ERR_CUDA


@pytest.mark.skipif(torch.cuda.is_available(), reason="fake pointers: host-only argument checks")
def test_failure_detection_calls_check_arguments(lib):
    L = lib.lib()
    a = 0x10000
    assert L.msa_set_wait_limit(None, 1000, None) == lib.MSA_ERR_INVALID_ARG
    assert L.msa_set_wait_limit(a + 16, 1000, None) == lib.MSA_ERR_INVALID_ARG  # not 256-byte aligned
    assert L.msa_diag_wait_timeout(None, 256, None) == lib.MSA_ERR_INVALID_ARG
    assert L.msa_diag_wait_timeout(a, 64, None) == lib.MSA_ERR_WORKSPACE
    assert L.msa_noalloc_get_status(None, None) == lib.MSA_ERR_INVALID_ARG
    # valid arguments reach the device, which is missing here
    assert L.msa_diag_wait_timeout(a, 256, None) == lib.MSA_ERR_CUDA
    assert L.msa_noalloc_clear_status(None) == lib.MSA_ERR_CUDA


@pytest.mark.skipif(torch.cuda.is_available(), reason="fake pointers: host-only argument checks")
def test_paged_params_rejected_before_launch(lib):
    L = lib.lib()
    a = 0x10000
    ws = ctypes.c_size_t(1 << 30)
    ptrs = [a, a, a, a, a, a, None, None, a]
    p = good_params(lib)
    p.block_table = a
    p.n_pages = 0
    assert L.msa_decode_fused(ctypes.byref(p), *ptrs, ws, None) == lib.MSA_ERR_INVALID_ARG
    p.n_pages = 64
    p.block_table = a + 2  # not 4-byte aligned
    assert L.msa_decode_fused(ctypes.byref(p), *ptrs, ws, None) == lib.MSA_ERR_INVALID_ARG
    p.block_table = a
    p.n_pages = 1 << 22  # pools of more than 2^31 rows
    assert L.msa_decode_fused(ctypes.byref(p), *ptrs, ws, None) == lib.MSA_ERR_UNSUPPORTED
    # the prefill index reads 128-key tiles: pages must hold at least 128 keys
    pp = good_params(lib, q_len=100, block_size=64)
    pp.block_table, pp.n_pages = a, 64
    assert L.msa_prefill_index_topk(ctypes.byref(pp), a, a, a, None, a, ws, None) == lib.MSA_ERR_UNSUPPORTED


def test_prefill_attention_workspace_does_not_grow_with_k(lib):
    """Passes hold 8192 * 32 / k rows beyond k = 32, so the per-pair partials keep one size."""
    base = lib.msa_workspace_size(good_params(lib, q_len=16384, q_start=0, max_seq_len=16384, top_k=32),
                                  lib.MSA_ENTRY_ATTN_PREFILL)
    for k in (64, 256, 1024):
        n = lib.msa_workspace_size(good_params(lib, q_len=16384, q_start=0, max_seq_len=16384, top_k=k),
                                   lib.MSA_ENTRY_ATTN_PREFILL)
        assert base * 0.99 <= n <= base * 1.01, (k, n, base)


@pytest.mark.skipif(torch.cuda.is_available(), reason="fake pointers: host-only argument checks")
@pytest.mark.parametrize("kw,fmt,scale,status", [
    (dict(), 2, 0x10000, "INVALID_ARG"),                        # unknown index-key format
    (dict(), 1, None, "INVALID_ARG"),                           # MXFP8 without scales
    (dict(), 1, 0x10008, "INVALID_ARG"),                        # scales not 16-byte aligned
    (dict(dtype=0), 1, 0x10000, "UNSUPPORTED"),                 # MXFP8 keys beside fp32 tensors
    (dict(max_seq_len=4100), 1, 0x10000, "UNSUPPORTED"),        # scale rows not in whole 16-row units
    (dict(idx_dim=32), 1, 0x10000, "UNSUPPORTED"),              # a 32-byte code row
], ids=lambda v: str(v))
def test_mxfp8_params_rejected_before_launch(lib, kw, fmt, scale, status):
    p = good_params(lib, **kw)
    p.idx_format, p.k_idx_scale = fmt, scale
    fake = 0x10000
    L = lib.lib()
    rc = L.msa_decode_fused(ctypes.byref(p), fake, fake, fake, fake, fake, fake, None, None, fake,
                            ctypes.c_size_t(1 << 30), None)
    assert rc == getattr(lib, "MSA_ERR_" + status), (rc, L.msa_last_error_string())
    # the prefill entries do not read MXFP8 keys
    pp = good_params(lib, q_len=100)
    pp.idx_format, pp.k_idx_scale = 1, 0x10000
    assert L.msa_prefill_index_topk(ctypes.byref(pp), fake, fake, fake, None, fake, ctypes.c_size_t(1 << 30),
                                    None) == lib.MSA_ERR_UNSUPPORTED
