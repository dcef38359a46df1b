"""Seeded synthetic MSA workloads.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic, so both the CUDA path and the CPU oracle take their
inputs from it.  The workloads stand in for the pages' "1M-token" long-context
runs (no dataset is named there): shapes, dtypes and the planted "hot block"
structure are fixed here, every value comes from one torch generator seeded
per workload.

Layouts (contiguous):
  q [B, Tq, Hq, D]      q_idx [B, Tq, G, di]      (G = Hkv groups)
  k, v [B, Hkv, Lmax, D]                          k_idx [B, Hik, Lmax, di]
  seq_lens int32 [B]  (cached length, current token(s) included)

Draw order (fixed): seq_lens (ragged workloads only); per (b, index-K head)
a unit direction u and the hot block ids; then q, q_idx, k, v, k_idx, each
drawn in slices of 65536 rows (k, v, k_idx per (b, head)).  Values are N(0, 1)
in fp32, cast to the workload dtype after any hot offset is added.

Hot blocks: every index-K row of a hot block gets + hot_scale * sqrt(di) * u,
and the index queries of every group reading that index-K head get
+ sqrt(di) * u, so a hot block's score rises by about hot_scale * di while the
background maximum over a million tokens stays near 5 * sqrt(2 * di).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    mode: str               # "decode" or "prefill"
    batch: int
    max_seq_len: int        # Lmax; prefill: sequence length T
    n_q_heads: int
    n_kv_heads: int
    n_idx_k_heads: int
    head_dim: int
    idx_dim: int
    block_size: int
    top_k: int
    dtype: str              # "f32" or "bf16"
    hot_blocks: int = 0     # planted per (b, index-K head); 0 = i.i.d. only
    hot_scale: float = 3.0
    min_seq_len: int = 0    # >0: decode lengths drawn uniformly in [min, max]
    chunk: int = 0          # prefill query chunk length (0 = whole sequence)
    seed: int = 0
    idx_format: str = "plain"  # "mxfp8": the index keys are stored as MXFP8 (quantised from these draws)

    @property
    def softmax_scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)

    @property
    def q_len(self) -> int:
        return 1 if self.mode == "decode" else self.max_seq_len

    def scaled(self, **kw) -> "Workload":
        return replace(self, **kw)


# The workloads: tiny fp32 decode, 16K causal prefill, ragged batched 128K
# decode, 1M decode (batch 1 and 4), 1M chunked causal prefill, 1M decode
# with one index-K head shared by every group, and the large-k regime in
# decode (1M) and prefill (128K), and the 1M decode with MXFP8 index keys.
WORKLOADS = {
    "decode_fp32_ctx4k": Workload("decode_fp32_ctx4k", "decode", 1, 4096, 4, 1, 1, 64, 32, 64, 8,
                                  "f32", seed=1001),
    "prefill_causal_16k": Workload("prefill_causal_16k", "prefill", 1, 16384, 16, 2, 2, 128, 64, 64, 16,
                                   "bf16", hot_blocks=12, seed=1002),
    "decode_b8_ctx128k_ragged": Workload("decode_b8_ctx128k_ragged", "decode", 8, 131072, 64, 8, 8, 128, 64,
                                         128, 16, "bf16", hot_blocks=24, min_seq_len=65536, seed=1003),
    "decode_ctx1m": Workload("decode_ctx1m", "decode", 1, 1048576, 64, 8, 8, 128, 64, 128, 16, "bf16",
                             hot_blocks=32, seed=1004),
    "decode_b4_ctx1m": Workload("decode_b4_ctx1m", "decode", 4, 1048576, 64, 8, 8, 128, 64, 128, 16, "bf16",
                                hot_blocks=32, seed=1004),
    "prefill_causal_1m": Workload("prefill_causal_1m", "prefill", 1, 1048576, 64, 8, 8, 128, 64, 128, 16,
                                  "bf16", hot_blocks=32, chunk=8192, seed=1005),
    # one index-K head shared by the 8 groups (the pages' literal reading): 1/8 of the index bytes
    "decode_ctx1m_shared_idx": Workload("decode_ctx1m_shared_idx", "decode", 1, 1048576, 64, 8, 1, 128, 64, 128,
                                        16, "bf16", hot_blocks=32, seed=1006),
    # the large-k regime the pages back-calculate (section 3): 64-token blocks, 16,384 of them at
    # 1M tokens, about 6 % selected (k 1024)
    "decode_ctx1m_large_k": Workload("decode_ctx1m_large_k", "decode", 1, 1048576, 64, 8, 8, 128, 64, 64, 1024,
                                     "bf16", hot_blocks=32, seed=1007),
    # the same density in prefill: 128K tokens in 64-token blocks (2,048 of them), k 128 (6.25 %),
    # 8192-token chunks
    "prefill_ctx128k_large_k": Workload("prefill_ctx128k_large_k", "prefill", 1, 131072, 64, 8, 8, 128, 64, 64, 128,
                                        "bf16", hot_blocks=32, chunk=8192, seed=1008),
    # the 1M decode with the index-key cache stored as MXFP8 (66 bytes per 64-dim key instead of 128)
    "decode_ctx1m_mxfp8_idx": Workload("decode_ctx1m_mxfp8_idx", "decode", 1, 1048576, 64, 8, 8, 128, 64, 128, 16,
                                       "bf16", hot_blocks=32, seed=1004, idx_format="mxfp8"),
}


def torch_dtype(w: Workload) -> torch.dtype:
    return torch.float32 if w.dtype == "f32" else torch.bfloat16


_SLICE_ROWS = 1 << 16  # rows per random draw for the large tensors


def make_inputs(w: Workload, device="cpu", seed: int | None = None) -> dict:
    """Draw one workload's tensors on ``device`` (same seed -> same values per device type)."""
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed if seed is None else seed)
    dt = torch_dtype(w)
    B, L, Tq = w.batch, w.max_seq_len, w.q_len
    G, Hik = w.n_kv_heads, w.n_idx_k_heads
    root_di = math.sqrt(w.idx_dim)

    def randn(*shape):
        return torch.randn(*shape, generator=gen, device=device, dtype=torch.float32)

    if w.mode == "decode" and w.min_seq_len > 0:
        seq_lens = torch.randint(w.min_seq_len, L + 1, (B,), generator=gen, device=device).to(torch.int32)
    else:
        seq_lens = torch.full((B,), L, dtype=torch.int32, device=device)

    # hot directions u[b, h] and hot block ids, drawn first so that every
    # large tensor can be written slice by slice
    u = torch.zeros(B, Hik, w.idx_dim, device=device)
    hot = torch.full((B, Hik, max(w.hot_blocks, 1)), -1, dtype=torch.int64, device=device)
    if w.hot_blocks > 0:
        lens_host = seq_lens.tolist()
        for b in range(B):
            nb = -(-lens_host[b] // w.block_size)
            for h in range(Hik):
                d = randn(w.idx_dim)
                u[b, h] = d / d.norm()
                ids = torch.randperm(nb, generator=gen, device=device)[: w.hot_blocks]
                hot[b, h, : len(ids)] = ids

    def fill(dst: torch.Tensor, add=None):
        """dst[rows] = N(0,1) (+ add(row0, x)) drawn in fixed slices of rows."""
        flat = dst.view(-1, dst.shape[-1])
        for r0 in range(0, flat.shape[0], _SLICE_ROWS):
            x = randn(min(_SLICE_ROWS, flat.shape[0] - r0), flat.shape[1])
            if add is not None:
                add(r0, x)
            flat[r0: r0 + x.shape[0]].copy_(x.to(dt))

    q = torch.empty(B, Tq, w.n_q_heads, w.head_dim, dtype=dt, device=device)
    fill(q)
    q_idx = torch.empty(B, Tq, G, w.idx_dim, dtype=dt, device=device)
    if w.hot_blocks > 0:
        # index queries of group g lean towards the direction of index head g mod Hik
        bias = torch.stack([u[:, g % Hik] for g in range(G)], dim=1) * root_di  # [B, G, di]
        rows_per_b = Tq * G

        def add_q_bias(r0, x):
            r = torch.arange(r0, r0 + x.shape[0], device=device)
            x += bias[r // rows_per_b, r % G]
        fill(q_idx, add_q_bias)
    else:
        fill(q_idx)
    k = torch.empty(B, G, L, w.head_dim, dtype=dt, device=device)
    v = torch.empty_like(k)
    for dst in (k, v):
        for b in range(B):
            for h in range(G):
                fill(dst[b, h])
    k_idx = torch.empty(B, Hik, L, w.idx_dim, dtype=dt, device=device)
    for b in range(B):
        for h in range(Hik):
            if w.hot_blocks > 0:
                is_hot = torch.zeros(-(-L // w.block_size), dtype=torch.bool, device=device)
                ids = hot[b, h]
                is_hot[ids[ids >= 0]] = True
                off = w.hot_scale * root_di * u[b, h]

                def add_hot(r0, x, is_hot=is_hot, off=off):
                    rows = torch.arange(r0, r0 + x.shape[0], device=device)
                    x += is_hot[rows // w.block_size, None].to(x.dtype) * off
                fill(k_idx[b, h], add_hot)
            else:
                fill(k_idx[b, h])
    return {"q": q, "q_idx": q_idx, "k": k, "v": v, "k_idx": k_idx, "seq_lens": seq_lens, "hot": hot}


def to_numpy_raw(x: torch.Tensor):
    """Exact bits of a tensor as NumPy: float32 stays float32, bf16 -> uint16 patterns."""
    x = x.detach().contiguous().cpu()
    if x.dtype == torch.bfloat16:
        return x.view(torch.int16).numpy().view("uint16")
    return x.numpy()
