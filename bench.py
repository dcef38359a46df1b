"""Benchmark of the MSA hot path on B200: one JSON line on rank 0.

A step is one MSA decode step at 1M context (index scan + block max pool +
TopK + sparse attention + split combine) through the C ABI, batch 1, with
the caches resident in HBM.  Metric: microseconds per decode step per layer
(lower is better).  Also reported: the dominant kernel (the index-key scan)
against the HBM roofline, the dense GQA decode over the same cache, an
end-to-end number with host<->device copies, and the CPU oracle timed on
this host.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun each rank runs its own sequence (weak scaling, no data-path
collective); rank 0 prints the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_sparse_long_12_b200.inputs import WORKLOADS, make_inputs, to_numpy_raw  # noqa: E402

METRIC = "MSA decode us/step/layer @1M ctx; prefill tok/s; % of HBM/tensor roofline"
UNIT = "us/step/layer"
L2_FLUSH_BYTES = 512 << 20
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "decode_index_scan_traffic.json")
# the index scan kernel's own sources: a committed DRAM-traffic capture counts only while they are unchanged
SCAN_SOURCES = ["block_sparse_long_12_b200/csrc/decode_index.cu", "block_sparse_long_12_b200/csrc/scan_args.h",
                "block_sparse_long_12_b200/csrc/msa_device.cuh", "block_sparse_long_12_b200/csrc/tcgen05.cuh"]


def scan_source_hash() -> str:
    h = hashlib.sha256()
    for f in SCAN_SOURCES:
        h.update(open(os.path.join(ROOT, f), "rb").read())
    return h.hexdigest()


def measured_peaks() -> tuple[dict, str]:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        return json.load(open(path)), "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


class ClockSampler:
    """nvidia-smi samples of this GPU's clocks and throttle reasons while running."""
    FIELDS = ("pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        props = torch.cuda.get_device_properties(device_index)
        self.bus = getattr(props, "pci_bus_id", None)
        self.rows = []
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) == 9:
                self.rows.append(parts)

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=2)

    def summary(self) -> dict:
        rows = self.rows
        if self.bus is not None:
            mine = [r for r in rows if r[0].lower().endswith(str(self.bus).lower())]
            rows = mine or rows
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    return world, rank, local


def max_over_ranks(x: float, world: int) -> float:
    """The job's time is the slowest rank's (all ranks run the same steps in the same order)."""
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def rank_seed(w, rank: int) -> int:
    """Weak scaling: every rank decodes its own sequence(s), drawn from a rank-specific seed."""
    return w.seed + 7919 * rank


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def timed_steps(fn, steps, flush, stream):
    """Per-step CUDA events on the launching stream; L2 flushed between steps (outside the events)."""
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        flush()
        ev[i][0].record(stream)
        fn()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) * 1e3 for a, b in ev]  # microseconds


def oracle_decode_seconds(w, x, repeats: int) -> tuple[float, int]:
    """Wall seconds of one oracle decode step (all sequences of the batch) and the threads it used."""
    import oracle
    oracle.build()
    p = oracle.Params(w.batch, w.n_q_heads, w.n_kv_heads, w.n_idx_k_heads, w.head_dim, w.idx_dim, w.block_size,
                      w.top_k, 1, 0, w.max_seq_len, w.dtype, w.softmax_scale)
    rows = [(b, 0) for b in range(w.batch)]
    ts = []
    for _ in range(repeats):
        t0 = time.perf_counter()
        oracle.msa_rows(p, x["seq_lens"], x["q"], x["q_idx"], x["k"], x["v"], x["k_idx"], rows)
        ts.append(time.perf_counter() - t0)
    threads = min(os.cpu_count() or 1, int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1)),
                  len(rows) * w.n_kv_heads)
    return statistics.median(ts), threads


def run_reference(args, world, rank):
    """The oracle, as it stands, on this host's cores, on the same workload and metric.

    Each step runs the oracle on a sample of the workload -- the first g of
    the KV groups (index scan, TopK and attention of those groups), chosen
    so that warm-up plus timed steps take about a minute -- and the step time
    is scaled to all groups."""
    if rank != 0:
        return
    import oracle
    oracle.build()
    w = WORKLOADS[args.workload]
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = make_inputs(w, device=dev)
    x = {n: to_numpy_raw(inp[n]) for n in ("q", "q_idx", "k", "v", "k_idx", "seq_lens")}
    del inp
    r = w.n_q_heads // w.n_kv_heads
    rows = [(b, 0) for b in range(w.batch)]

    def sample(groups):
        hik = groups if w.n_idx_k_heads == w.n_kv_heads else 1
        xs = {"q": np.ascontiguousarray(x["q"][:, :, :groups * r]), "q_idx": np.ascontiguousarray(x["q_idx"][:, :, :groups]),
              "k": np.ascontiguousarray(x["k"][:, :groups]), "v": np.ascontiguousarray(x["v"][:, :groups]),
              "k_idx": np.ascontiguousarray(x["k_idx"][:, :hik]), "seq_lens": x["seq_lens"]}
        p = oracle.Params(w.batch, groups * r, groups, hik, w.head_dim, w.idx_dim, w.block_size, w.top_k, 1, 0,
                          w.max_seq_len, w.dtype, w.softmax_scale)
        return p, xs

    p1, x1 = sample(1)
    t0 = time.perf_counter()
    oracle.msa_rows(p1, x1["seq_lens"], x1["q"], x1["q_idx"], x1["k"], x1["v"], x1["k_idx"], rows)
    per_group = time.perf_counter() - t0
    groups = int(max(1, min(w.n_kv_heads, 60.0 / max(per_group * (args.steps + args.warmup), 1e-9))))
    p, xs = sample(groups)
    for _ in range(args.warmup):
        oracle.msa_rows(p, xs["seq_lens"], xs["q"], xs["q_idx"], xs["k"], xs["v"], xs["k_idx"], rows)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.msa_rows(p, xs["seq_lens"], xs["q"], xs["q_idx"], xs["k"], xs["v"], xs["k_idx"], rows)
    sec = (time.perf_counter() - t0) / args.steps * (w.n_kv_heads / groups)
    threads = min(os.cpu_count() or 1, len(rows) * groups)
    us = sec * 1e6
    sample_txt = (f"{groups} of {w.n_kv_heads} KV groups of {w.name} (batch {w.batch}) per step, fp64 C oracle "
                  f"with OpenMP, time scaled to all groups")
    line = {"impl": "reference", "metric": METRIC, "value": round(us, 1), "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(us / 1e3, 3), "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w, args.gpus),
            "cpu_baseline": {"value": round(us, 1), "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": sample_txt},
            "e2e": {"value": round(us, 1), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def workload_config(w, n):
    return {"workload": w.name, "batch_per_gpu": w.batch, "context": w.max_seq_len, "n_q_heads": w.n_q_heads,
            "n_kv_heads": w.n_kv_heads, "n_idx_k_heads": w.n_idx_k_heads, "head_dim": w.head_dim,
            "idx_dim": w.idx_dim, "block_size": w.block_size, "top_k": w.top_k,
            "l2": (f"inputs larger than L2 (the {w.max_seq_len}-token index-key stream of every step), and a "
                   f"{L2_FLUSH_BYTES >> 20} MiB read pass between timed steps (outside the step events) so that "
                   "no selected K/V tile survives in L2 from the previous step"),
            "parallelism": "replicas" if n == 1 else f"weak-scaling replicas x{n}, no collective"}


def run_ours(args, world, rank, local):
    from block_sparse_long_12_b200 import _lib, api
    torch.cuda.set_device(local)
    w = WORKLOADS[args.workload]
    dev = torch.device("cuda", local)
    inp = make_inputs(w, device=dev, seed=rank_seed(w, rank))
    q, q_idx, k, v, k_idx, lens = (inp[n] for n in ("q", "q_idx", "k", "v", "k_idx", "seq_lens"))
    stream = torch.cuda.current_stream()
    p = api.params_from(q, q_idx, k, k_idx, block_size=w.block_size, top_k=w.top_k, seq_lens=lens)
    ws = api.workspace(p, _lib.MSA_ENTRY_DECODE_FUSED, dev)
    o = torch.empty_like(q)
    ids = torch.empty(w.batch, 1, w.n_kv_heads, w.top_k, dtype=torch.int32, device=dev)
    lse = torch.empty(w.batch, 1, w.n_q_heads, dtype=torch.float32, device=dev)
    flush_buf = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=dev)

    def flush():
        # reads (not writes) so that the next step does not start by writing back dirty lines
        torch.amax(flush_buf)

    def step():
        _lib.msa_decode_fused(p, q, q_idx, k, v, k_idx, o, ids, lse, ws, stream)

    for _ in range(max(args.warmup, 3)):
        flush()
        step()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        barrier(world)
        torch.cuda.synchronize()
        per_step = timed_steps(step, args.steps, flush, stream)
        torch.cuda.synchronize()
        barrier(world)
    step_us = max_over_ranks(sum(per_step) / len(per_step), world)
    assert _lib.msa_get_device_status(ws) == 0, "device status word reports a timeout"

    # per-kernel durations inside the same step (stage events; separate pass)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    for e in evs:
        e.record(stream)
    torch.cuda.synchronize()
    _lib.msa_set_stage_events(evs)
    stage = [[], []]  # index scan; TopK merge + sparse attention + split merge
    try:
        for _ in range(args.steps):
            flush()
            step()
            torch.cuda.synchronize()
            for i in range(2):
                stage[i].append(evs[i].elapsed_time(evs[i + 1]) * 1e3)
    finally:
        _lib.msa_set_stage_events(None)
    scan_us = max_over_ranks(statistics.mean(stage[0]), world)
    attn_us = max_over_ranks(statistics.mean(stage[1]), world)

    # dense GQA decode over the same cache (the sparse-vs-dense ratio)
    pd = api.params_from(q, q_idx, k, k_idx, block_size=w.block_size, top_k=w.top_k, seq_lens=lens,
                         flags=_lib.MSA_DENSE)
    wsd = api.workspace(pd, _lib.MSA_ENTRY_ATTN_DECODE, dev)
    od = torch.empty_like(q)

    def dense():
        _lib.msa_sparse_attn_decode(pd, q, k, v, None, od, None, wsd, stream)

    dense_steps = max(3, min(args.steps, 50))
    for _ in range(3):
        dense()
    dense_us = max_over_ranks(statistics.mean(timed_steps(dense, dense_steps, flush, stream)), world)

    # end to end through the C ABI: pinned host inputs -> device, decode, result -> pinned host
    h_q = torch.empty(q.shape, dtype=q.dtype, pin_memory=True).copy_(q)
    h_qi = torch.empty(q_idx.shape, dtype=q_idx.dtype, pin_memory=True).copy_(q_idx)
    pos = lens.long() - 1
    new_k = torch.empty(w.batch, w.n_kv_heads, 1, w.head_dim, dtype=k.dtype, pin_memory=True)
    new_v = torch.empty_like(new_k).pin_memory()
    new_ki = torch.empty(w.batch, w.n_idx_k_heads, 1, w.idx_dim, dtype=k_idx.dtype, pin_memory=True)
    for b in range(w.batch):
        new_k[b].copy_(k[b, :, pos[b]:pos[b] + 1])
        new_v[b].copy_(v[b, :, pos[b]:pos[b] + 1])
        new_ki[b].copy_(k_idx[b, :, pos[b]:pos[b] + 1])
    h_o = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
    h_ids = torch.empty(ids.shape, dtype=ids.dtype, pin_memory=True)
    pos_host = pos.tolist()

    def e2e_step():
        q.copy_(h_q, non_blocking=True)
        q_idx.copy_(h_qi, non_blocking=True)
        for b in range(w.batch):  # append the new token's K, V and index key at its position
            pb = pos_host[b]
            k[b, :, pb:pb + 1].copy_(new_k[b], non_blocking=True)
            v[b, :, pb:pb + 1].copy_(new_v[b], non_blocking=True)
            k_idx[b, :, pb:pb + 1].copy_(new_ki[b], non_blocking=True)
        step()
        h_o.copy_(o, non_blocking=True)
        h_ids.copy_(ids, non_blocking=True)

    e2e_n = max(3, min(args.steps, 200))
    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(e2e_n)]
    for i in range(e2e_n):
        flush()
        e2e_ev[i][0].record(stream)
        e2e_step()
        e2e_ev[i][1].record(stream)
        e2e_ev[i][1].synchronize()  # the host reads the step's result before the next step
    e2e_us = max_over_ranks(statistics.mean(a.elapsed_time(b) * 1e3 for a, b in e2e_ev), world)
    h2d = sum(t.numel() * t.element_size() for t in (h_q, h_qi, new_k, new_v, new_ki))
    d2h = h_o.numel() * h_o.element_size() + h_ids.numel() * h_ids.element_size()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        x = {n: to_numpy_raw(inp[n]) for n in ("q", "q_idx", "k", "v", "k_idx", "seq_lens")}
        sec, threads = oracle_decode_seconds(w, x, repeats=2)
        cpu = {"value": round(sec * 1e6, 1), "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": f"one full decode step of {w.name} (batch {w.batch}), fp64 C oracle, median of 2"}
        del x

    lens_host = lens.tolist()
    del inp, q, q_idx, k, v, k_idx, ws, wsd, o, od
    torch.cuda.empty_cache()
    shared = None if args.no_shared_index else run_shared_index(args, world, rank, local, stream, flush)
    large_k = None if args.no_large_k else run_shared_index(args, world, rank, local, stream, flush,
                                                            name="decode_ctx1m_large_k")
    prefill = None
    if not args.no_prefill:
        del flush_buf
        torch.cuda.empty_cache()
        prefill = run_prefill(world, rank, local, stream)

    if rank != 0:
        return
    peaks, peak_kind = measured_peaks()
    es = 2 if w.dtype == "bf16" else 4
    scan_bytes = sum(lens_host) * w.n_idx_k_heads * w.idx_dim * es  # every index key read once
    achieved = scan_bytes / (scan_us * 1e-6) / 1e9
    traffic = None
    if os.path.exists(TRAFFIC_FILE):
        rec = json.load(open(TRAFFIC_FILE))
        if rec.get("source_sha256") == scan_source_hash() and rec.get("workload") == w.name:
            traffic = rec.get("dram_bytes_per_launch")
    clocks = clk.summary()

    line = {
        "metric": METRIC, "value": round(step_us, 2), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(step_us / 1e3, 5), "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": workload_config(w, world),
        "roofline": {"bound": "hbm", "kernel": "decode index scan", "achieved": round(achieved, 1),
                     "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                     "peak_kind": peak_kind, "algorithmic_bytes": scan_bytes, "kernel_us": round(scan_us, 2),
                     "traffic": traffic},
        "stages_us": {"index_scan": round(scan_us, 2), "topk_merge_and_sparse_attention": round(attn_us, 2)},
        "step_roofline_frac": round((scan_bytes + w.batch * w.n_kv_heads * w.top_k * w.block_size * w.head_dim * es * 2)
                                    / (step_us * 1e-6) / 1e9 / peaks["hbm_gbs"], 4),
        "dense_gqa_us": round(dense_us, 2), "sparse_vs_dense_speedup": round(dense_us / step_us, 2),
        "e2e": {"value": round(e2e_us, 2), "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": 2 * args.steps,
        "shared_index_head": shared,
        "large_k": large_k,
        "prefill": prefill,
        "clocks": clocks,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)


def run_shared_index(args, world, rank, local, stream, flush, name="decode_ctx1m_shared_idx"):
    """The 1M decode step with one index-K head shared by the 8 groups: the index stream is 1/8
    as long, so the step is no longer dominated by the scan.  Same timing as the main step.
    With name="decode_ctx1m_large_k": the large-k regime (64-token blocks, k 1024 of 16,384; the
    middle stage is then the radix select, the last the attention over 268 MB of K/V)."""
    from block_sparse_long_12_b200 import _lib, api
    w = WORKLOADS[name]
    dev = torch.device("cuda", local)
    inp = make_inputs(w, device=dev, seed=rank_seed(w, rank))
    q, q_idx, k, v, k_idx, lens = (inp[n] for n in ("q", "q_idx", "k", "v", "k_idx", "seq_lens"))
    p = api.params_from(q, q_idx, k, k_idx, block_size=w.block_size, top_k=w.top_k, seq_lens=lens)
    ws = api.workspace(p, _lib.MSA_ENTRY_DECODE_FUSED, dev)
    o = torch.empty_like(q)
    ids = torch.empty(w.batch, 1, w.n_kv_heads, w.top_k, dtype=torch.int32, device=dev)

    def step():
        _lib.msa_decode_fused(p, q, q_idx, k, v, k_idx, o, ids, None, ws, stream)

    for _ in range(max(args.warmup, 3)):
        flush()
        step()
    torch.cuda.synchronize()
    n = max(3, min(args.steps, 500))
    barrier(world)
    step_us = max_over_ranks(statistics.mean(timed_steps(step, n, flush, stream)), world)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    for e in evs:
        e.record(stream)
    torch.cuda.synchronize()
    _lib.msa_set_stage_events(evs)
    stage = [[], []]
    try:
        for _ in range(n):
            flush()
            step()
            torch.cuda.synchronize()
            for i in range(2):
                stage[i].append(evs[i].elapsed_time(evs[i + 1]) * 1e3)
    finally:
        _lib.msa_set_stage_events(None)
    assert _lib.msa_get_device_status(ws) == 0
    scan_us = max_over_ranks(statistics.mean(stage[0]), world)
    attn_us = max_over_ranks(statistics.mean(stage[1]), world)
    peaks, kind = measured_peaks()
    idx_bytes = sum(lens.tolist()) * w.n_idx_k_heads * w.idx_dim * 2
    kv_bytes = w.batch * w.n_kv_heads * w.top_k * w.block_size * w.head_dim * 2 * 2
    del inp, q, q_idx, k, v, k_idx, ws, o
    torch.cuda.empty_cache()
    stages = ({"index_scan": round(scan_us, 2), "topk_merge_and_sparse_attention": round(attn_us, 2)}
              if w.top_k <= 32 else
              {"index_scan": round(scan_us, 2), "radix_select_and_sparse_attention": round(attn_us, 2)})
    return {"workload": w.name, "value": round(step_us, 2), "unit": UNIT, "n_idx_k_heads": w.n_idx_k_heads,
            "block_size": w.block_size, "top_k": w.top_k, "stages_us": stages,
            "algorithmic_bytes": idx_bytes + kv_bytes,
            "step_roofline_frac": round((idx_bytes + kv_bytes) / (step_us * 1e-6) / 1e9 / peaks["hbm_gbs"], 4),
            "scan_gbs": round(idx_bytes / (scan_us * 1e-6) / 1e9, 1), "peak_kind": kind}


def run_prefill(world, rank, local, stream):
    """The 1M-token causal prefill in 8192-token chunks: Step 1 (tensor-core index scores, block max
    pool, TopK) then Step 2 (tensor-core sparse attention) for every chunk.  Returns tok/s and the
    index kernel's tensor-core roofline fraction (max over ranks)."""
    from block_sparse_long_12_b200 import _lib, api
    w = WORKLOADS["prefill_causal_1m"]
    dev = torch.device("cuda", local)
    inp = make_inputs(w, device=dev, seed=rank_seed(w, rank))
    T, C = w.max_seq_len, w.chunk
    n_chunks = T // C
    ids = torch.empty(1, T, w.n_kv_heads, w.top_k, dtype=torch.int32, device=dev)
    o = torch.empty_like(inp["q"])
    chunks = []
    for c in range(n_chunks):
        p = api.make_params(batch=1, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads, n_idx_k_heads=w.n_idx_k_heads,
                            head_dim=w.head_dim, idx_dim=w.idx_dim, block_size=w.block_size, top_k=w.top_k,
                            max_seq_len=T, dtype=_lib.MSA_BF16, q_len=C, q_start=c * C)
        chunks.append((p, inp["q"][:, c * C:(c + 1) * C], inp["q_idx"][:, c * C:(c + 1) * C],
                       ids[:, c * C:(c + 1) * C], o[:, c * C:(c + 1) * C]))
    ws = api.workspace([c[0] for c in chunks], _lib.MSA_ENTRY_PREFILL_INDEX_TOPK, dev)

    def index_pass():
        for (p, q, qi, idc, oc) in chunks:
            _lib.msa_prefill_index_topk(p, qi, inp["k_idx"], idc, None, ws, stream)

    def attn_pass():
        for (p, q, qi, idc, oc) in chunks:
            _lib.msa_sparse_attn_prefill(p, q, inp["k"], inp["v"], idc, oc, None, ws, stream)

    index_pass()
    attn_pass()
    torch.cuda.synchronize()
    ti, ta = [], []
    for _ in range(3):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        e[0].record(stream)
        index_pass()
        e[1].record(stream)
        attn_pass()
        e[2].record(stream)
        torch.cuda.synchronize()
        ti.append(e[0].elapsed_time(e[1]) / 1e3)
        ta.append(e[1].elapsed_time(e[2]) / 1e3)
    assert _lib.msa_get_device_status(ws) == 0
    # issued attention work: every 16-token x 8-head tile walks the union of its tokens' lists
    tq = 128 // (w.n_q_heads // w.n_kv_heads)
    u_sum = 0
    for c0 in range(0, T, 65536):
        blk = ids[0, c0:c0 + 65536].reshape(-1, tq, w.n_kv_heads, w.top_k).permute(0, 2, 1, 3)
        blk = blk.reshape(-1, tq * w.top_k).sort(dim=-1).values
        distinct = (blk[:, 1:] != blk[:, :-1]) & (blk[:, 1:] >= 0)
        u_sum += int(distinct.sum()) + int((blk[:, 0] >= 0).sum())
    att_issued = 4.0 * 128 * w.block_size * w.head_dim * u_sum
    t_idx = max_over_ranks(statistics.median(ti), world)
    t_att = max_over_ranks(statistics.median(ta), world)
    peaks, kind = measured_peaks()
    # algorithmic FLOPs: every visible (row, key) pair of every group scores d_i MACs; attention
    # touches top_k blocks of block_size keys per (row, head) for Q.K and P.V
    pairs = T * (T + 1) // 2
    idx_flops = 2.0 * w.idx_dim * w.n_kv_heads * pairs
    att_flops = 4.0 * w.head_dim * w.n_q_heads * w.top_k * w.block_size * T
    total = t_idx + t_att
    return {"workload": w.name, "tokens": T, "chunk": C, "tok_per_s": round(T * world / total, 1),
            "seconds": round(total, 4), "index_s": round(t_idx, 4), "attention_s": round(t_att, 4),
            "index_tflops": round(idx_flops / t_idx / 1e12, 1),
            "index_frac_of_bf16_peak": round(idx_flops / t_idx / 1e12 / peaks["bf16_tflops_sustained"], 4),
            "attention_useful_tflops": round(att_flops / t_att / 1e12, 1),
            "attention_issued_tflops": round(att_issued / t_att / 1e12, 1),
            "attention_mean_union_blocks": round(u_sum / (T // tq * w.n_kv_heads), 2),
            "overall_frac_of_bf16_peak": round((idx_flops + att_flops) / total / 1e12 / peaks["bf16_tflops_sustained"], 4),
            "peak": peaks["bf16_tflops_sustained"], "peak_kind": f"{kind} sustained (long step)",
            "gpu_launches": 2 * n_chunks * 3}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="decode_ctx1m", choices=["decode_ctx1m", "decode_b4_ctx1m",
                                                                    "decode_b8_ctx128k_ragged"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-shared-index", action="store_true", help="skip the shared index-K head decode step")
    ap.add_argument("--no-large-k", action="store_true", help="skip the large-k (k 1024 of 16,384 blocks) decode step")
    args = ap.parse_args()
    world, rank, local = dist_setup()
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
