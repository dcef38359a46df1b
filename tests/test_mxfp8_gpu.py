"""GPU parity of MXFP8 index keys: the quantiser bit for bit against the oracle's, the cache append,
stored index scores and the fused decode step against the fp64 oracle run on the exactly decoded
keys.  Reading: MXFP8 (docs.clore.ai "MiniMax M3", the official checkpoints' format) taken as the
microscaling format, 32 E4M3 elements per E8M0 scale, here the storage of the index-key cache read
by Step 1 (page "MiniMax wird duenn", atlascloud.ai, section 1, Step 1)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from oracle import mxfp8
from block_sparse_long_12_b200.inputs import WORKLOADS, make_inputs, to_numpy_raw

pytestmark = pytest.mark.gpu

from parity import compare_decode, oracle_params  # noqa: E402


def _api():
    from block_sparse_long_12_b200 import _lib, api
    return _lib, api


def bf16_to_f32(raw: np.ndarray) -> np.ndarray:
    return (raw.astype(np.uint32) << 16).view(np.float32)


def f32_inputs(inp, codes, scales) -> dict:
    """The oracle's copy of a decode step: bf16 tensors widened exactly to fp32, the index keys
    decoded exactly from their MXFP8 codes."""
    x = {n: bf16_to_f32(to_numpy_raw(inp[n])) for n in ("q", "q_idx", "k", "v")}
    x["k_idx"] = mxfp8.decode(codes.cpu().numpy(), scales.cpu().numpy())
    x["seq_lens"] = to_numpy_raw(inp["seq_lens"])
    return x


def test_quantizer_bit_exact():
    """Rows spanning many magnitudes, all-zero and sign-only blocks, exact ties and saturating
    block maxima: codes and scales equal the oracle's bit for bit."""
    _lib, api = _api()
    rng = np.random.default_rng(7)
    rows = 4096
    v = rng.standard_normal((rows, 64)) * np.exp2(rng.integers(-40, 40, (rows, 1))).astype(np.float64)
    v[0] = 0.0
    v[1, :32] = -0.0
    v[2, :32] = 1.99 * 2.0 ** 5                      # block maximum just below a power of two: saturates
    pos = mxfp8.E4M3_TABLE[:127]
    mids = (pos[:-1] + pos[1:]) / 2
    v[3, :32] = np.concatenate([[448.0], mids[-31:]]) * 2.0 ** -3   # ties of the round to nearest even
    v[4, :32] = np.concatenate([[300.0], mids[:31]])                 # subnormal ties
    src = torch.tensor(v, dtype=torch.float32).to(torch.bfloat16)
    ref_c, ref_s = mxfp8.quantize(src.double().numpy())
    codes, scales = api.quantize_index_k(src.cuda())
    torch.cuda.synchronize()
    assert np.array_equal(scales.cpu().numpy(), ref_s)
    assert np.array_equal(codes.cpu().numpy(), ref_c)


def small(**kw):
    base = dict(batch=3, max_seq_len=5008, min_seq_len=1, n_q_heads=16, n_kv_heads=4, n_idx_k_heads=4, head_dim=128,
                idx_dim=64, block_size=64, top_k=8, hot_blocks=6, seed=12)
    base.update(kw)
    return WORKLOADS["decode_b8_ctx128k_ragged"].scaled(**base)


def test_index_scores_mxfp8():
    """Token and block scores from MXFP8 keys against the oracle's on the decoded keys."""
    _lib, api = _api()
    w = small()
    inp = make_inputs(w, device="cuda")
    codes, scales = api.quantize_index_k(inp["k_idx"])
    x = f32_inputs(inp, codes, scales)
    p_or = oracle_params(x, block_size=w.block_size, top_k=w.top_k)
    for flags, width in ((_lib.MSA_SCORES_TOKEN, w.max_seq_len), (_lib.MSA_SCORES_BLOCKMAX, -(-w.max_seq_len // w.block_size))):
        p = api.params_from(inp["q"], inp["q_idx"], inp["k"], codes, block_size=w.block_size, top_k=w.top_k,
                            seq_lens=inp["seq_lens"], flags=flags, k_idx_scale=scales)
        out = torch.empty(w.batch, 1, w.n_kv_heads, width, dtype=torch.float32, device="cuda")
        ws = api.workspace(p, _lib.MSA_ENTRY_INDEX_SCORE, "cuda")
        _lib.msa_index_score(p, inp["q_idx"], codes, out, ws)
        torch.cuda.synchronize()
        got = out.cpu().numpy()
        for b in range(w.batch):
            pos = int(x["seq_lens"][b]) - 1
            for g in range(w.n_kv_heads):
                s = oracle.token_scores(p_or, x["q_idx"], x["k_idx"], b, 0, g, pos)
                ref = s if flags == _lib.MSA_SCORES_TOKEN else oracle.block_scores(p_or, s, pos)
                n = len(ref)
                err = np.abs(got[b, 0, g, :n] - ref) / np.maximum(np.abs(ref), 1.0)
                assert err.max() <= 1e-5, (flags, b, g, err.max())


def test_index_scores_mxfp8_wide_magnitudes():
    """Index keys whose rows span 2^-30 .. 2^30 (block scales from tiny to large, many subnormal
    E4M3 codes beside each block's maximum): token scores against the oracle on the decoded keys."""
    _lib, api = _api()
    w = small(batch=2, max_seq_len=2048, min_seq_len=2048)
    inp = make_inputs(w, device="cuda")
    g = torch.Generator(device="cpu").manual_seed(9)
    mag = torch.pow(2.0, torch.randint(-30, 31, (w.batch, w.n_idx_k_heads, w.max_seq_len, 1), generator=g).float())
    spread = torch.pow(2.0, torch.randint(-12, 1, (w.batch, w.n_idx_k_heads, w.max_seq_len, w.idx_dim), generator=g).float())
    k_idx = (inp["k_idx"].float().cpu() * mag * spread).to(torch.bfloat16).cuda()
    codes, scales = api.quantize_index_k(k_idx)
    inp = dict(inp, k_idx=k_idx)
    x = f32_inputs(inp, codes, scales)
    p_or = oracle_params(x, block_size=w.block_size, top_k=w.top_k)
    p = api.params_from(inp["q"], inp["q_idx"], inp["k"], codes, block_size=w.block_size, top_k=w.top_k,
                        seq_lens=inp["seq_lens"], flags=_lib.MSA_SCORES_TOKEN, k_idx_scale=scales)
    out = torch.empty(w.batch, 1, w.n_kv_heads, w.max_seq_len, dtype=torch.float32, device="cuda")
    _lib.msa_index_score(p, inp["q_idx"], codes, out, api.workspace(p, _lib.MSA_ENTRY_INDEX_SCORE, "cuda"))
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    assert (mxfp8.E4M3_TABLE[codes.cpu().numpy() & 0x7F] < 2.0 ** -6).mean() > 0.01, "few subnormal codes"
    for b in range(w.batch):
        pos = int(x["seq_lens"][b]) - 1
        for gg in range(w.n_kv_heads):
            ref = oracle.token_scores(p_or, x["q_idx"], x["k_idx"], b, 0, gg, pos)
            # relative to the row's key magnitude: fp32 sums of products spanning 2^24
            scale = np.abs(x["k_idx"][b, gg % w.n_idx_k_heads, :pos + 1]).max(axis=-1) * 8.0
            err = np.abs(got[b, 0, gg, :pos + 1] - ref) / np.maximum(scale, 1e-30)
            assert err.max() <= 1e-5, (b, gg, err.max())


def test_index_scores_mxfp8_exact_products():
    """The scan's products of bf16 query elements and E4M3 codes are exact in fp32 (8 + 4
    significant bits) and its sums run in a fixed order, so the index query times 2^20 (beyond f16's
    range) gives exactly 2^20 times the scores, bit for bit; the scores against the oracle on the
    decoded keys."""
    _lib, api = _api()
    w = small(batch=2, max_seq_len=3008, min_seq_len=3008)
    inp = make_inputs(w, device="cuda")
    q = inp["q_idx"]
    q = torch.where(q.abs() < 2.0 ** -14, torch.zeros_like(q), q)  # no tiny elements: no underflow
    codes, scales = api.quantize_index_k(inp["k_idx"])
    outs = []
    for qq in (q, q * 2.0 ** 20):
        p = api.params_from(inp["q"], qq, inp["k"], codes, block_size=w.block_size, top_k=w.top_k,
                            seq_lens=inp["seq_lens"], flags=_lib.MSA_SCORES_TOKEN, k_idx_scale=scales)
        out = torch.empty(w.batch, 1, w.n_kv_heads, w.max_seq_len, dtype=torch.float32, device="cuda")
        _lib.msa_index_score(p, qq, codes, out, api.workspace(p, _lib.MSA_ENTRY_INDEX_SCORE, "cuda"))
        outs.append(out)
    torch.cuda.synchronize()
    assert torch.equal(outs[1], outs[0] * 2.0 ** 20)
    x = f32_inputs(dict(inp, q_idx=q), codes, scales)
    p_or = oracle_params(x, block_size=w.block_size, top_k=w.top_k)
    got = outs[0].cpu().numpy()
    for b in range(w.batch):
        pos = int(x["seq_lens"][b]) - 1
        for g in range(w.n_kv_heads):
            ref = oracle.token_scores(p_or, x["q_idx"], x["k_idx"], b, 0, g, pos)
            err = np.abs(got[b, 0, g, :pos + 1] - ref) / np.maximum(np.abs(ref), 1.0)
            assert err.max() <= 1e-5, (b, g, err.max())


@pytest.mark.parametrize("case", [
    dict(),                                                             # ragged batch, per-group index heads
    dict(n_idx_k_heads=1, hot_blocks=0),                                # one index head shared by 4 groups
    dict(n_kv_heads=8, n_q_heads=64, n_idx_k_heads=1, hot_blocks=0),    # 8 groups on one stream
    dict(idx_dim=128, block_size=128, top_k=16),                        # 128-dim index keys
    dict(block_size=16, top_k=32, max_seq_len=3008),                    # small blocks, chunks of 16 rows
    dict(block_size=32, top_k=100, max_seq_len=6000),                   # large k (radix select)
], ids=lambda c: ",".join(f"{k}={v}" for k, v in c.items()) or "default")
def test_fused_decode_mxfp8(case):
    _lib, api = _api()
    w = small(**case)
    inp = make_inputs(w, device="cuda")
    codes, scales = api.quantize_index_k(inp["k_idx"])
    o, ids, lse = api.decode(inp["q"], inp["q_idx"], inp["k"], inp["v"], codes, inp["seq_lens"],
                             block_size=w.block_size, top_k=w.top_k, k_idx_scale=scales)
    torch.cuda.synchronize()
    x = f32_inputs(inp, codes, scales)
    compare_decode(x, oracle_params(x, block_size=w.block_size, top_k=w.top_k), o, ids, lse, tol=2e-2, tol_lse=1e-3)


def test_append_quantizes_the_new_token():
    """msa_decode_append with MXFP8 keys writes the quantised new key at seq_lens - 1 and nothing else."""
    _lib, api = _api()
    w = small()
    inp = make_inputs(w, device="cuda")
    codes, scales = api.quantize_index_k(inp["k_idx"])
    c0, s0 = codes.clone(), scales.clone()
    B, Hik, di = w.batch, w.n_idx_k_heads, w.idx_dim
    g = torch.Generator(device="cpu").manual_seed(3)
    kn = torch.randn(B, w.n_kv_heads, w.head_dim, generator=g).to(torch.bfloat16).cuda()
    vn = torch.randn(B, w.n_kv_heads, w.head_dim, generator=g).to(torch.bfloat16).cuda()
    kin = (torch.randn(B, Hik, di, generator=g) * 30).to(torch.bfloat16).cuda()
    p = api.params_from(inp["q"], inp["q_idx"], inp["k"], codes, block_size=w.block_size, top_k=w.top_k,
                        seq_lens=inp["seq_lens"], k_idx_scale=scales)
    _lib.msa_decode_append(p, kn, vn, kin, inp["k"], inp["v"], codes)
    torch.cuda.synchronize()
    ref_c, ref_s = mxfp8.quantize(kin.double().cpu().numpy())
    lens = inp["seq_lens"].cpu().numpy()
    for b in range(B):
        pos = int(lens[b]) - 1
        assert np.array_equal(codes[b, :, pos].cpu().numpy(), ref_c[b])
        assert np.array_equal(scales[b, :, pos].cpu().numpy(), ref_s[b])
        c0[b, :, pos] = codes[b, :, pos]
        s0[b, :, pos] = scales[b, :, pos]
    assert torch.equal(c0, codes) and torch.equal(s0, scales)


def test_full_size_decode_mxfp8():
    """The 1M decode workload with MXFP8 index keys: every group's ids and outputs against the oracle
    on the decoded keys; the planted hot blocks are still the ones selected."""
    _lib, api = _api()
    w = WORKLOADS["decode_ctx1m"]
    inp = make_inputs(w, device="cuda")
    codes, scales = api.quantize_index_k(inp["k_idx"])
    o, ids, lse = api.decode(inp["q"], inp["q_idx"], inp["k"], inp["v"], codes, inp["seq_lens"],
                             block_size=w.block_size, top_k=w.top_k, k_idx_scale=scales)
    torch.cuda.synchronize()
    hot = inp["hot"].cpu().numpy()
    x = f32_inputs(inp, codes, scales)
    del inp
    torch.cuda.empty_cache()
    compare_decode(x, oracle_params(x, block_size=w.block_size, top_k=w.top_k), o, ids, lse, tol=2e-2, tol_lse=1e-3)
    idn = ids.cpu().numpy()
    for g in range(w.n_kv_heads):
        assert set(idn[0, 0, g].tolist()) <= set(hot[0, g % w.n_idx_k_heads].tolist()) - {-1}
