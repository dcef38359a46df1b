"""Small, self-contained runs of the MSA kernels for profilers (ncu).

  python profile_run.py decode --context 262144 --steps 3
  python profile_run.py prefill_index --context 65536 --chunk 8192 --steps 1
  python profile_run.py prefill_attn --context 65536 --chunk 8192 --steps 1
  python profile_run.py prefill_chunks --context 1048576 --chunks 16,64,127 --steps 1
  python profile_run.py scan_shared --context 1048576 --steps 3
  python profile_run.py large_k --context 262144 --steps 3
  python profile_run.py decode_mxfp8 --context 262144 --steps 3

Inputs are the seeded synthetic workloads of ``inputs`` at the requested
size (1M-token shapes: 64 query heads, 8 KV groups, head dim 128, index dim
64, block 128, top-k 16; large_k: block 64, top-k 1024), kept small enough
for a profiler's replay passes.
"""
from __future__ import annotations

import argparse

import torch

from block_sparse_long_12_b200 import _lib, api
from block_sparse_long_12_b200.inputs import WORKLOADS, make_inputs


def run_decode(args, name="decode_ctx1m"):
    w = WORKLOADS[name].scaled(max_seq_len=args.context, batch=args.batch)
    inp = make_inputs(w, device="cuda")
    q, q_idx, k, v, k_idx, lens = (inp[n] for n in ("q", "q_idx", "k", "v", "k_idx", "seq_lens"))
    scale = None
    if w.idx_format == "mxfp8":
        k_idx, scale = api.quantize_index_k(k_idx)
    p = api.params_from(q, q_idx, k, k_idx, block_size=w.block_size, top_k=w.top_k, seq_lens=lens,
                        k_idx_scale=scale)
    ws = api.workspace(p, _lib.MSA_ENTRY_DECODE_FUSED, "cuda")
    o = torch.empty_like(q)
    ids = torch.empty(w.batch, 1, w.n_kv_heads, w.top_k, dtype=torch.int32, device="cuda")
    for _ in range(args.steps):
        _lib.msa_decode_fused(p, q, q_idx, k, v, k_idx, o, ids, None, ws)
    torch.cuda.synchronize()
    print("decode done", ids[0, 0, 0].tolist())


def run_prefill_index(args):
    w = WORKLOADS["prefill_causal_1m"].scaled(max_seq_len=args.context)
    inp = make_inputs(w, device="cuda")
    q_idx, k_idx = inp["q_idx"], inp["k_idx"]
    T = args.chunk
    for step in range(args.steps):
        q_start = args.context - T
        qi = q_idx[:, q_start:q_start + T].contiguous()
        p = api.make_params(batch=1, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads, n_idx_k_heads=w.n_idx_k_heads,
                            head_dim=w.head_dim, idx_dim=w.idx_dim, block_size=w.block_size, top_k=w.top_k,
                            max_seq_len=w.max_seq_len, dtype=_lib.MSA_BF16, q_len=T, q_start=q_start)
        ids = torch.empty(1, T, w.n_kv_heads, w.top_k, dtype=torch.int32, device="cuda")
        ws = api.workspace(p, _lib.MSA_ENTRY_PREFILL_INDEX_TOPK, "cuda")
        _lib.msa_prefill_index_topk(p, qi, k_idx, ids, None, ws)
    torch.cuda.synchronize()
    print("prefill index done")


def run_prefill_attn(args):
    """Index branch, then the sparse branch, for the last chunk of the context."""
    w = WORKLOADS["prefill_causal_1m"].scaled(max_seq_len=args.context)
    inp = make_inputs(w, device="cuda")
    T = args.chunk
    q_start = args.context - T
    p = api.make_params(batch=1, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads, n_idx_k_heads=w.n_idx_k_heads,
                        head_dim=w.head_dim, idx_dim=w.idx_dim, block_size=w.block_size, top_k=w.top_k,
                        max_seq_len=w.max_seq_len, dtype=_lib.MSA_BF16, q_len=T, q_start=q_start)
    qi = inp["q_idx"][:, q_start:q_start + T].contiguous()
    q = inp["q"][:, q_start:q_start + T].contiguous()
    ids = torch.empty(1, T, w.n_kv_heads, w.top_k, dtype=torch.int32, device="cuda")
    o = torch.empty_like(q)
    ws_i = api.workspace(p, _lib.MSA_ENTRY_PREFILL_INDEX_TOPK, "cuda")
    ws_a = api.workspace(p, _lib.MSA_ENTRY_ATTN_PREFILL, "cuda")
    for _ in range(args.steps):
        _lib.msa_prefill_index_topk(p, qi, inp["k_idx"], ids, None, ws_i)
        _lib.msa_sparse_attn_prefill(p, q, inp["k"], inp["v"], ids, o, None, ws_a)
    torch.cuda.synchronize()
    print("prefill attention done", int(_lib.msa_get_device_status(ws_a)))


def run_prefill_chunks(args):
    """Index branch, then the sparse branch, for a few 8192-token chunks of the 1M-token causal
    prefill (the chunks listed in --chunks), so that a launch list shows every kernel of a chunk
    early, in the middle and at the end of the sequence."""
    w = WORKLOADS["prefill_causal_1m"].scaled(max_seq_len=args.context)
    inp = make_inputs(w, device="cuda")
    T = args.chunk
    todo = [int(c) for c in args.chunks.split(",")]
    plist = []
    for c in todo:
        plist.append(api.make_params(batch=1, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads,
                                     n_idx_k_heads=w.n_idx_k_heads, head_dim=w.head_dim, idx_dim=w.idx_dim,
                                     block_size=w.block_size, top_k=w.top_k, max_seq_len=w.max_seq_len,
                                     dtype=_lib.MSA_BF16, q_len=T, q_start=c * T))
    ws_i = api.workspace(plist, _lib.MSA_ENTRY_PREFILL_INDEX_TOPK, "cuda")
    ws_a = api.workspace(plist, _lib.MSA_ENTRY_ATTN_PREFILL, "cuda")
    ids = torch.empty(1, T, w.n_kv_heads, w.top_k, dtype=torch.int32, device="cuda")
    o = torch.empty(1, T, w.n_q_heads, w.head_dim, dtype=torch.bfloat16, device="cuda")
    for _ in range(args.steps):
        for c, p in zip(todo, plist):
            q0 = c * T
            _lib.msa_prefill_index_topk(p, inp["q_idx"][:, q0:q0 + T], inp["k_idx"], ids, None, ws_i)
            _lib.msa_sparse_attn_prefill(p, inp["q"][:, q0:q0 + T], inp["k"], inp["v"], ids, o, None, ws_a)
    torch.cuda.synchronize()
    print("prefill chunks done", todo, int(_lib.msa_get_device_status(ws_a)))


def run_scan_shared(args):
    """The index scan of one index-K head shared by the 8 groups (stored block scores, so that only
    the index keys are on the device)."""
    w = WORKLOADS["decode_ctx1m_shared_idx"].scaled(max_seq_len=args.context, batch=args.batch)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(w.seed)
    q_idx = torch.randn(w.batch, 1, w.n_kv_heads, w.idx_dim, generator=gen, device="cuda").to(torch.bfloat16)
    k_idx = torch.randn(w.batch, 1, w.max_seq_len, w.idx_dim, generator=gen, device="cuda").to(torch.bfloat16)
    lens = torch.full((w.batch,), w.max_seq_len, dtype=torch.int32, device="cuda")
    for _ in range(args.steps):
        out = api.index_scores(q_idx, k_idx, lens, n_kv_heads=w.n_kv_heads, block_size=w.block_size, mode="block")
    torch.cuda.synchronize()
    print("scan done", float(out[0, 0, 0, :4].sum()))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("what", choices=["decode", "prefill_index", "prefill_attn", "prefill_chunks", "scan_shared",
                                     "large_k", "decode_mxfp8"])
    ap.add_argument("--context", type=int, default=262144)
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--chunk", type=int, default=8192)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--chunks", default="16,64,127", help="prefill_chunks: chunk indices to run")
    args = ap.parse_args()
    {"decode": run_decode, "prefill_index": run_prefill_index, "prefill_attn": run_prefill_attn,
     "prefill_chunks": run_prefill_chunks,
     "scan_shared": run_scan_shared,
     "large_k": lambda a: run_decode(a, "decode_ctx1m_large_k"),
     "decode_mxfp8": lambda a: run_decode(a, "decode_ctx1m_mxfp8_idx")}[args.what](args)


if __name__ == "__main__":
    main()
