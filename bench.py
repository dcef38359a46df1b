"""Benchmark of the MSA hot path on B200: one JSON line on rank 0.

A step is one MSA decode step at 1M context (index scan + block max pool +
TopK + sparse attention + split combine) through the C ABI, batch 1, with
the caches resident in HBM.  Metric: microseconds per decode step per layer
(lower is better).  Also reported, each with its roofline fraction and the
CPU oracle timed on this host:
  * every other workload: tiny fp32 decode, 16K causal prefill, ragged
    batch-8 128K decode, batch-4 1M decode, 128K prefill with k 128 of 2,048
    blocks (``configs``);
  * the 1M decode with one shared index-K head, the large-k regime, and
    MXFP8 index keys;
  * the 1M-token chunked causal prefill (tok/s, tensor-core fraction);
  * the dense GQA decode over the same cache, and an end-to-end number with
    host<->device copies inside the timed region.

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
SPEC_HBM_GBS = 8000.0  # the B200's nominal HBM3e bandwidth (DGX figure), for context beside the measured copy
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
    """nvidia-smi samples of this GPU's clocks and throttle reasons, time-stamped, for the whole run;
    `window()` marks the spans (timed regions) whose samples the summary uses."""
    FIELDS = ("pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        props = torch.cuda.get_device_properties(device_index)
        self.bus = getattr(props, "pci_bus_id", None)
        self.dom = getattr(props, "pci_domain_id", None)
        self.rows = []      # (monotonic time, fields)
        self.windows = []   # (t0, t1)
        self.proc = None
        self.error = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError as e:
            self.proc, self.error = None, f"nvidia-smi did not start: {e}"
        return self

    def _mine(self, bus_field: str) -> bool:
        # "00000000:1B:00.0": domain, bus (hex), device.function
        if self.bus is None:
            return True
        try:
            dom, bus = bus_field.split(":")[:2]
            return int(bus, 16) == int(self.bus) and (self.dom is None or int(dom, 16) == int(self.dom))
        except ValueError:
            return False

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) == 9 and self._mine(parts[0]):
                self.rows.append((time.monotonic(), parts))

    def wait_first(self, timeout=8.0):
        t0 = time.monotonic()
        while self.proc is not None and not self.rows and time.monotonic() - t0 < timeout:
            time.sleep(0.05)
        if self.proc is not None and not self.rows and self.error is None:
            self.error = f"no sample from nvidia-smi within {timeout:.0f} s"

    class _Win:
        def __init__(self, s):
            self.s = s

        def __enter__(self):
            self.t0 = time.monotonic()

        def __exit__(self, *a):
            self.s.windows.append((self.t0, time.monotonic()))

    def window(self):
        return ClockSampler._Win(self)

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=2)
            if not self.rows and self.error is None:
                err = (self.proc.stderr.read() or "").strip()[:200]
                self.error = f"nvidia-smi gave no row for this GPU (bus {self.bus}){': ' + err if err else ''}"

    def summary(self, windows=None) -> dict:
        wins = self.windows if windows is None else windows
        rows = [r for (t, r) in self.rows if any(a <= t <= b for a, b in wins)]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "why_empty": self.error or "no sample fell inside the timed windows"}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        pw = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "power_w_max": max(pw) if pw else None, "reasons": reasons, "samples": len(rows)}


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


def read_stream_gbs(dev, gib: int = 4) -> float:
    """A read-only HBM reference measured here: the faster of torch's max and sum over a float32
    buffer of `gib` GiB (32 times L2), best of 5 each after a warm-up, CUDA events.  The driver's copy
    peak moves every byte twice (read and write), so a kernel that only reads can exceed it; this is
    the read-only counterpart."""
    x = torch.ones(gib << 28, dtype=torch.float32, device=dev)
    best = float("inf")
    for op in (torch.amax, torch.sum):
        op(x)
        for _ in range(5):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            op(x)
            b.record()
            b.synchronize()
            best = min(best, a.elapsed_time(b) * 1e-3)
    n = x.numel() * 4
    del x
    torch.cuda.empty_cache()
    return n / best / 1e9


READ_GBS = None  # set once per run by run_ours


def hbm_frac(nbytes: float, us: float, peaks: dict) -> dict:
    gbs = nbytes / (us * 1e-6) / 1e9
    d = {"achieved_gbs": round(gbs, 1), "frac_of_measured_copy": round(gbs / peaks["hbm_gbs"], 4),
         "frac_of_spec_8tbs": round(gbs / SPEC_HBM_GBS, 4)}
    if READ_GBS:
        d["frac_of_read_stream"] = round(gbs / READ_GBS, 4)
    return d


# ----------------------------------------------------------------------------- oracle timing (CPU legs)
def oracle_params(w, q_len=1, q_start=0, prefill=False):
    import oracle
    return oracle.Params(w.batch, w.n_q_heads, w.n_kv_heads, w.n_idx_k_heads, w.head_dim, w.idx_dim, w.block_size,
                         w.top_k, q_len, q_start, w.max_seq_len, w.dtype, w.softmax_scale, prefill=prefill)


def time_oracle(fn, repeats: int, warmup: int = 1) -> float:
    for _ in range(warmup):
        fn()
    ts = []
    for _ in range(repeats):
        t0 = time.perf_counter()
        fn()
        ts.append(time.perf_counter() - t0)
    return statistics.median(ts)


def oracle_decode(w, x, repeats=5, threads=None) -> dict:
    """The oracle's decode step (every sequence and group of the batch), median of `repeats` after a warm-up."""
    import oracle
    oracle.build()
    n = oracle.set_threads(threads)
    p = oracle_params(w)
    rows = [(b, 0) for b in range(w.batch)]

    def run():
        oracle.msa_rows(p, x["seq_lens"], x["q"], x["q_idx"], x["k"], x["v"], x["k_idx"], rows)
    sec = time_oracle(run, repeats)
    oracle.set_threads(None)
    return {"value": round(sec * 1e6, 1), "unit": UNIT, "cores": min(n, w.batch * w.n_kv_heads), "kind": "oracle",
            "sample": f"one full decode step of {w.name} (batch {w.batch}), fp64 C oracle, median of {repeats} "
                      f"after a warm-up"}


def oracle_prefill_rows(w, inp, positions, repeats=3) -> dict:
    """The oracle's Steps 1 and 2 for query rows at the given absolute positions (prefill), us per row."""
    import oracle
    oracle.build()
    n = oracle.set_threads(None)
    x = {k_: to_numpy_raw(inp[k_]) for k_ in ("k", "v", "k_idx")}
    pos = torch.tensor(sorted(positions), device=inp["q"].device)
    # the rows' q / q_idx placed at their positions of a compact chunk starting at the first row
    c0 = int(pos[0])
    span = int(pos[-1]) - c0 + 1
    q = np.zeros((1, span, w.n_q_heads, w.head_dim), np.uint16)
    qi = np.zeros((1, span, w.n_kv_heads, w.idx_dim), np.uint16)
    q[0, (pos - c0).cpu().numpy()] = to_numpy_raw(inp["q"][0, pos])
    qi[0, (pos - c0).cpu().numpy()] = to_numpy_raw(inp["q_idx"][0, pos])
    p = oracle_params(w, q_len=span, q_start=c0, prefill=True)
    rows = [(0, int(t) - c0) for t in pos.tolist()]

    def run():
        oracle.msa_rows(p, None, q, qi, x["k"], x["v"], x["k_idx"], rows)
    sec = time_oracle(run, repeats, warmup=0)
    return {"us_per_row": round(sec / len(rows) * 1e6, 1), "rows": len(rows), "cores": n,
            "sample": f"{len(rows)} query rows spread over positions {c0}..{int(pos[-1])}, fp64 C oracle "
                      f"(Steps 1 and 2, all groups), median of {repeats}"}


# ----------------------------------------------------------------------------- reference arm
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


# ----------------------------------------------------------------------------- decode timing
def decode_bytes(w, lens_host) -> tuple[int, int]:
    es = 2 if w.dtype == "bf16" else 4
    # every index key read once: idx_dim elements, or MXFP8 codes plus one scale byte per 32
    row = w.idx_dim + w.idx_dim // 32 if w.idx_format == "mxfp8" else w.idx_dim * es
    idx = sum(lens_host) * w.n_idx_k_heads * row
    kv = 0
    for L in lens_host:  # the selected blocks' K and V (the visible part of each)
        nb = -(-L // w.block_size)
        kv += w.n_kv_heads * min(w.top_k, nb) * w.block_size * w.head_dim * es * 2
    return idx, kv


def time_decode(w, rank, world, local, stream, flush, steps, warmup, clk=None, stage=True, oracle_leg=False):
    """Steady-state fused decode steps of workload w: step time, stage times, bytes, roofline."""
    from block_sparse_long_12_b200 import _lib, api
    dev = torch.device("cuda", local)
    inp = make_inputs(w, device=dev, seed=rank_seed(w, rank))
    q, q_idx, k, v, k_idx, lens = (inp[n] for n in ("q", "q_idx", "k", "v", "k_idx", "seq_lens"))
    k_scale = None
    if w.idx_format == "mxfp8":  # the index-key cache as MXFP8, quantised once before timing
        k_idx, k_scale = api.quantize_index_k(k_idx)
        inp["k_idx"], inp["k_idx_scale"] = k_idx, k_scale
        torch.cuda.synchronize()
    p = api.params_from(q, q_idx, k, k_idx, block_size=w.block_size, top_k=w.top_k, seq_lens=lens,
                        k_idx_scale=k_scale)
    ws = api.workspace(p, _lib.MSA_ENTRY_DECODE_FUSED, dev)
    o = torch.empty_like(q)
    ids = torch.empty(w.batch, 1, w.n_kv_heads, w.top_k, dtype=torch.int32, device=dev)
    lse = torch.empty(w.batch, 1, w.n_q_heads, dtype=torch.float32, device=dev)

    def step():
        _lib.msa_decode_fused(p, q, q_idx, k, v, k_idx, o, ids, lse, ws, stream)

    for _ in range(max(warmup, 3)):
        flush()
        step()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    if clk is not None:
        with clk.window():
            per_step = timed_steps(step, steps, flush, stream)
    else:
        per_step = timed_steps(step, steps, flush, stream)
    torch.cuda.synchronize()
    barrier(world)
    step_us = max_over_ranks(sum(per_step) / len(per_step), world)
    assert _lib.msa_get_device_status(ws) == 0, "device status word reports a timeout"
    out = {"step_us": step_us, "per_step": per_step, "inp": inp, "step": step, "p": p, "ws": ws, "o": o,
           "ids": ids, "lse": lse, "lens_host": lens.tolist()}
    if stage:
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        for e in evs:
            e.record(stream)
        torch.cuda.synchronize()
        _lib.msa_set_stage_events(evs)
        st = [[], []]
        try:
            for _ in range(min(steps, 200)):
                flush()
                step()
                torch.cuda.synchronize()
                for i in range(2):
                    st[i].append(evs[i].elapsed_time(evs[i + 1]) * 1e3)
        finally:
            _lib.msa_set_stage_events(None)
        out["scan_us"] = max_over_ranks(statistics.mean(st[0]), world)
        out["attn_us"] = max_over_ranks(statistics.mean(st[1]), world)
    return out


def decode_summary(w, r, peaks, peak_kind, cpu=None) -> dict:
    idx_b, kv_b = decode_bytes(w, r["lens_host"])
    d = {"workload": w.name, "value": round(r["step_us"], 2), "unit": UNIT, "batch": w.batch,
         "context": (min(r["lens_host"]), max(r["lens_host"])) if min(r["lens_host"]) != max(r["lens_host"])
         else r["lens_host"][0],
         "n_idx_k_heads": w.n_idx_k_heads, "block_size": w.block_size, "top_k": w.top_k, "dtype": w.dtype,
         "index_keys": w.idx_format,
         "algorithmic_bytes": idx_b + kv_b, "step_roofline": hbm_frac(idx_b + kv_b, r["step_us"], peaks),
         "peak_kind": peak_kind}
    if "scan_us" in r:
        stage2 = "topk_merge_and_sparse_attention" if w.top_k <= 32 else "radix_select_and_sparse_attention"
        d["stages_us"] = {"index_scan": round(r["scan_us"], 2), stage2: round(r["attn_us"], 2)}
        d["scan_roofline"] = hbm_frac(idx_b, r["scan_us"], peaks)
    if cpu is not None:
        d["oracle"] = cpu
    return d


def run_ours(args, world, rank, local):
    from block_sparse_long_12_b200 import _lib, api
    torch.cuda.set_device(local)
    w = WORKLOADS[args.workload]
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    flush_buf = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=dev)
    peaks, peak_kind = measured_peaks()

    def flush():
        # reads (not writes) so that the next step does not start by writing back dirty lines
        torch.amax(flush_buf)

    global READ_GBS
    READ_GBS = read_stream_gbs(dev)
    clk = ClockSampler(local).start()
    clk.wait_first()

    r = time_decode(w, rank, world, local, stream, flush, args.steps, args.warmup, clk=clk)
    step_us, scan_us, attn_us = r["step_us"], r["scan_us"], r["attn_us"]
    inp, step, p = r["inp"], r["step"], r["p"]
    q, q_idx, k, v, k_idx, lens = (inp[n] for n in ("q", "q_idx", "k", "v", "k_idx", "seq_lens"))
    o, ids = r["o"], r["ids"]
    # clocks: if the timed region was too short for the sampler (100 ms period), keep the same step
    # running back to back for a moment, inside a marked window, so that the record shows its clocks
    if clk.summary()["samples"] < 3:
        with clk.window():
            t_end = time.monotonic() + 1.5
            while time.monotonic() < t_end:
                for _ in range(200):
                    step()
                torch.cuda.synchronize()
        clocks_window = "timed region + 1.5 s of the same decode step back to back"
    else:
        clocks_window = "timed region"

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

    # end to end through the C ABI: every step brings the new token (q, q_idx and its K, V and index
    # key) from pinned host memory in one copy, appends it to the caches (msa_decode_append), decodes,
    # and takes the output and the block ids back in one copy; the host reads them before the next step
    es = q.element_size()

    def seg(n):  # 16-byte aligned segment lengths
        return (n + 15) // 16 * 16
    sizes_in = [q.numel() * es, q_idx.numel() * es, w.batch * w.n_kv_heads * w.head_dim * es,
                w.batch * w.n_kv_heads * w.head_dim * es, w.batch * w.n_idx_k_heads * w.idx_dim * es]
    offs_in = [sum(seg(n) for n in sizes_in[:i]) for i in range(len(sizes_in))]
    h_in = torch.empty(offs_in[-1] + seg(sizes_in[-1]), dtype=torch.uint8, pin_memory=True)
    d_in = torch.empty_like(h_in, device=dev)

    def view(buf, i, shape, dtype):
        return buf[offs_in[i]:offs_in[i] + sizes_in[i]].view(dtype).view(shape)
    pos = lens.long() - 1
    new_k = torch.stack([k[b, :, pos[b]] for b in range(w.batch)])
    new_v = torch.stack([v[b, :, pos[b]] for b in range(w.batch)])
    new_ki = torch.stack([k_idx[b, :, pos[b]] for b in range(w.batch)])
    for i, t in enumerate((q, q_idx, new_k, new_v, new_ki)):
        view(h_in, i, t.shape, t.dtype).copy_(t)
    dq, dqi = view(d_in, 0, q.shape, q.dtype), view(d_in, 1, q_idx.shape, q_idx.dtype)
    dk, dv, dki = (view(d_in, i, t.shape, t.dtype) for i, t in ((2, new_k), (3, new_v), (4, new_ki)))
    o_bytes, id_bytes = o.numel() * es, ids.numel() * 4
    d_out = torch.empty(seg(o_bytes) + id_bytes, dtype=torch.uint8, device=dev)
    h_out = torch.empty_like(d_out, device="cpu").pin_memory()
    do = d_out[:o_bytes].view(o.dtype).view(o.shape)
    dids = d_out[seg(o_bytes):].view(torch.int32).view(ids.shape)

    def e2e_step():
        d_in.copy_(h_in, non_blocking=True)
        _lib.msa_decode_append(p, dk, dv, dki, k, v, k_idx, stream)
        _lib.msa_decode_fused(p, dq, dqi, k, v, k_idx, do, dids, None, r["ws"], stream)
        h_out.copy_(d_out, non_blocking=True)

    e2e_n = max(3, min(args.steps, 200))
    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    assert torch.equal(dids, ids), "the end-to-end step selected other blocks"
    e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(e2e_n)]
    for i in range(e2e_n):
        flush()
        e2e_ev[i][0].record(stream)
        e2e_step()
        e2e_ev[i][1].record(stream)
        e2e_ev[i][1].synchronize()  # the host reads the step's result before the next step
    e2e_stream_us = max_over_ranks(statistics.mean(a.elapsed_time(b) * 1e3 for a, b in e2e_ev), world)

    # the same step captured once as a CUDA graph (copies and kernels as its nodes, the programmatic
    # launch edge kept) and replayed each step, as a serving loop would run it
    graph = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream(device=dev)
    cap.wait_stream(stream)
    torch.cuda.synchronize()
    with torch.cuda.graph(graph, stream=cap):
        s_cap = torch.cuda.current_stream()
        d_in.copy_(h_in, non_blocking=True)
        _lib.msa_decode_append(p, dk, dv, dki, k, v, k_idx, s_cap)
        _lib.msa_decode_fused(p, dq, dqi, k, v, k_idx, do, dids, None, r["ws"], s_cap)
        h_out.copy_(d_out, non_blocking=True)
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    h_ids = h_out[seg(o_bytes):].view(torch.int32).view(ids.shape)
    assert torch.equal(h_ids, ids.cpu()), "the graph-replayed step selected other blocks"
    g_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(e2e_n)]
    for i in range(e2e_n):
        flush()
        g_ev[i][0].record(stream)
        graph.replay()
        g_ev[i][1].record(stream)
        g_ev[i][1].synchronize()  # the host reads the step's result before the next step
    e2e_graph_us = max_over_ranks(statistics.mean(a.elapsed_time(b) * 1e3 for a, b in g_ev), world)
    del graph
    e2e_us = min(e2e_stream_us, e2e_graph_us)
    h2d = h_in.numel()
    d2h = h_out.numel()

    cpu = cpu1 = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        x = {n: to_numpy_raw(inp[n]) for n in ("q", "q_idx", "k", "v", "k_idx", "seq_lens")}
        cpu = oracle_decode(w, x, repeats=5)
        cpu1 = oracle_decode(w, x, repeats=3, threads=1)
        del x

    lens_host = r["lens_host"]
    del r, inp, q, q_idx, k, v, k_idx, o, od, wsd
    torch.cuda.empty_cache()

    # the other workloads, each with its own oracle time
    configs = {}
    if not args.no_configs:
        for name in ("decode_fp32_ctx4k", "decode_b8_ctx128k_ragged", "decode_b4_ctx1m"):
            if name == w.name:
                continue
            wc = WORKLOADS[name]
            rc = time_decode(wc, rank, world, local, stream, flush, max(3, min(args.steps, 500)), args.warmup)
            oc = None
            if rank == 0 and world == 1 and not args.no_cpu_baseline:
                xc = {n: to_numpy_raw(rc["inp"][n]) for n in ("q", "q_idx", "k", "v", "k_idx", "seq_lens")}
                oc = oracle_decode(wc, xc, repeats=3)
                del xc
            configs[name] = decode_summary(wc, rc, peaks, peak_kind, oc)
            del rc
            torch.cuda.empty_cache()
        configs["prefill_causal_16k"] = run_prefill(WORKLOADS["prefill_causal_16k"], world, rank, local, stream,
                                                    peaks, peak_kind, oracle_rows=0 if args.no_cpu_baseline else 256)
        torch.cuda.empty_cache()
        configs["prefill_ctx128k_large_k"] = run_prefill(WORKLOADS["prefill_ctx128k_large_k"], world, rank, local,
                                                         stream, peaks, peak_kind,
                                                         oracle_rows=0 if args.no_cpu_baseline else 32)
        torch.cuda.empty_cache()

    shared = None if args.no_shared_index else run_extra_decode("decode_ctx1m_shared_idx", args, world, rank, local,
                                                                stream, flush, peaks, peak_kind)
    large_k = None if args.no_large_k else run_extra_decode("decode_ctx1m_large_k", args, world, rank, local, stream,
                                                            flush, peaks, peak_kind)
    mxfp8_idx = None if args.no_mxfp8 else run_extra_decode("decode_ctx1m_mxfp8_idx", args, world, rank, local,
                                                            stream, flush, peaks, peak_kind)
    prefill = None
    if not args.no_prefill:
        del flush_buf
        torch.cuda.empty_cache()
        prefill = run_prefill(WORKLOADS["prefill_causal_1m"], world, rank, local, stream, peaks, peak_kind,
                              oracle_rows=0 if args.no_cpu_baseline else 32)
    clk.stop()

    if rank != 0:
        return
    scan_bytes, kv_bytes = decode_bytes(w, lens_host)
    achieved = scan_bytes / (scan_us * 1e-6) / 1e9
    traffic = None
    if os.path.exists(TRAFFIC_FILE):
        rec = json.load(open(TRAFFIC_FILE))
        if rec.get("source_sha256") == scan_source_hash() and rec.get("workload") == w.name:
            traffic = rec.get("dram_bytes_per_launch")
    clocks = clk.summary()
    clocks["window"] = clocks_window
    clocks["whole_run"] = {k_: v_ for k_, v_ in clk.summary([(0.0, float("inf"))]).items() if k_ != "why_empty"}
    if cpu is not None:
        cpu["single_thread_us"] = cpu1["value"]

    line = {
        "metric": METRIC, "value": round(step_us, 2), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(step_us / 1e3, 5), "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": workload_config(w, world),
        "roofline": {"bound": "hbm", "kernel": "decode index scan", "achieved": round(achieved, 1),
                     "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                     "peak_kind": f"{peak_kind} copy (read+write); a read-only stream can exceed it",
                     "frac_of_spec_8tbs": round(achieved / SPEC_HBM_GBS, 4),
                     "read_stream_gbs": round(READ_GBS, 1), "frac_of_read_stream": round(achieved / READ_GBS, 4),
                     "algorithmic_bytes": scan_bytes, "kernel_us": round(scan_us, 2), "traffic": traffic},
        "stages_us": {"index_scan": round(scan_us, 2), "topk_merge_and_sparse_attention": round(attn_us, 2)},
        "step_roofline": hbm_frac(scan_bytes + kv_bytes, step_us, peaks),
        "step_roofline_frac": round((scan_bytes + kv_bytes) / (step_us * 1e-6) / 1e9 / peaks["hbm_gbs"], 4),
        "dense_gqa_us": round(dense_us, 2), "sparse_vs_dense_speedup": round(dense_us / step_us, 2),
        "e2e": {"value": round(e2e_us, 2), "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "stream_us": round(e2e_stream_us, 2), "graph_us": round(e2e_graph_us, 2),
                "how": "one pinned H2D copy of the new token, msa_decode_append, msa_decode_fused, one D2H copy of o "
                       "and ids, the host waiting for each step; value = the faster of launching them on the stream "
                       "and replaying them as one captured CUDA graph"},
        "gpu_launches": 2 * args.steps,
        "e2e_launches_per_step": 3,
        "configs": configs,
        "shared_index_head": shared,
        "large_k": large_k,
        "mxfp8_index_keys": mxfp8_idx,
        "prefill": prefill,
        "clocks": clocks,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)


def run_extra_decode(name, args, world, rank, local, stream, flush, peaks, peak_kind):
    """The 1M decode step with one index-K head shared by the 8 groups (the index stream is 1/8 as
    long), the large-k regime (64-token blocks, k 1024 of 16,384; the middle stage is then the
    radix select, the last the attention over 268 MB of K/V), or MXFP8 index keys (66 bytes per key
    row instead of 128).  Same timing as the main step."""
    w = WORKLOADS[name]
    r = time_decode(w, rank, world, local, stream, flush, max(3, min(args.steps, 500)), args.warmup)
    d = decode_summary(w, r, peaks, peak_kind)
    del r
    torch.cuda.empty_cache()
    return d


def run_prefill(w, world, rank, local, stream, peaks, peak_kind, oracle_rows=0):
    """Causal prefill of workload w in w.chunk-token chunks (the whole sequence when 0): Step 1
    (tensor-core index scores, block max pool, TopK) then Step 2 (sparse attention) for every chunk.
    Returns tok/s and the tensor-core roofline fractions (max over ranks), and the oracle's time per
    row on `oracle_rows` rows spread over the sequence."""
    from block_sparse_long_12_b200 import _lib, api
    dev = torch.device("cuda", local)
    inp = make_inputs(w, device=dev, seed=rank_seed(w, rank))
    T = w.max_seq_len
    C = w.chunk or T
    n_chunks = -(-T // C)
    ids = torch.empty(1, T, w.n_kv_heads, w.top_k, dtype=torch.int32, device=dev)
    o = torch.empty_like(inp["q"])
    chunks = []
    for c in range(n_chunks):
        n = min(C, T - c * C)
        p = api.make_params(batch=1, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads, n_idx_k_heads=w.n_idx_k_heads,
                            head_dim=w.head_dim, idx_dim=w.idx_dim, block_size=w.block_size, top_k=w.top_k,
                            max_seq_len=T, dtype=_lib.MSA_BF16, q_len=n, q_start=c * C)
        chunks.append((p, inp["q"][:, c * C:c * C + n], inp["q_idx"][:, c * C:c * C + n],
                       ids[:, c * C:c * C + n], o[:, c * C:c * C + n]))
    ws_i = api.workspace([c[0] for c in chunks], _lib.MSA_ENTRY_PREFILL_INDEX_TOPK, dev)
    ws_a = api.workspace([c[0] for c in chunks], _lib.MSA_ENTRY_ATTN_PREFILL, dev)

    def index_pass():
        for (p, q, qi, idc, oc) in chunks:
            _lib.msa_prefill_index_topk(p, qi, inp["k_idx"], idc, None, ws_i, stream)

    def attn_pass():
        for (p, q, qi, idc, oc) in chunks:
            _lib.msa_sparse_attn_prefill(p, q, inp["k"], inp["v"], idc, oc, None, ws_a, stream)

    for _ in range(3 if n_chunks == 1 else 1):
        index_pass()
        attn_pass()
    torch.cuda.synchronize()
    ti, ta = [], []
    reps = 20 if n_chunks == 1 else 3
    for _ in range(reps):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        e[0].record(stream)
        index_pass()
        e[1].record(stream)
        attn_pass()
        e[2].record(stream)
        torch.cuda.synchronize()
        ti.append(e[0].elapsed_time(e[1]) / 1e3)
        ta.append(e[1].elapsed_time(e[2]) / 1e3)
    assert _lib.msa_get_device_status(ws_i) == 0 and _lib.msa_get_device_status(ws_a) == 0
    t_idx = max_over_ranks(statistics.median(ti), world)
    t_att = max_over_ranks(statistics.median(ta), world)
    # algorithmic FLOPs: every visible (row, key) pair of every group scores d_i MACs; attention
    # touches the selected blocks' visible keys per (row, head) for Q.K and P.V
    pairs = T * (T + 1) // 2
    idx_flops = 2.0 * w.idx_dim * w.n_kv_heads * pairs
    nb = torch.arange(T, device=dev) // w.block_size + 1
    keys = (torch.clamp(nb, max=w.top_k) * w.block_size).double().sum().item()  # upper bound per row: k full blocks
    att_flops = 4.0 * w.head_dim * w.n_q_heads * keys
    total = t_idx + t_att
    sus, burst = peaks["bf16_tflops_sustained"], peaks["bf16_tflops"]
    d = {"workload": w.name, "tokens": T, "chunk": C, "tok_per_s": round(T * world / total, 1),
         "seconds": round(total, 5), "index_s": round(t_idx, 5), "attention_s": round(t_att, 5),
         "index_tflops": round(idx_flops / t_idx / 1e12, 1),
         "index_frac_of_bf16_peak": round(idx_flops / t_idx / 1e12 / sus, 4),
         "attention_useful_tflops": round(att_flops / t_att / 1e12, 1),
         "attention_frac_of_bf16_peak": round(att_flops / t_att / 1e12 / sus, 4),
         "overall_frac_of_bf16_peak": round((idx_flops + att_flops) / total / 1e12 / sus, 4),
         "overall_frac_of_bf16_burst_peak": round((idx_flops + att_flops) / total / 1e12 / burst, 4),
         "algorithmic_flops": idx_flops + att_flops,
         "peak": sus, "peak_kind": f"{peak_kind} sustained (long step); burst {burst}",
         "gpu_launches": None}
    if oracle_rows and rank == 0 and world == 1:
        rng = np.random.default_rng(w.seed)
        positions = sorted(set(rng.choice(T, oracle_rows, replace=False).tolist()))
        orc = oracle_prefill_rows(w, inp, positions)
        orc["extrapolated_full_sequence_s"] = round(orc["us_per_row"] * T / 1e6, 1)
        orc["extrapolation"] = ("us_per_row x all rows; rows late in the sequence cost more (Step 1 is linear in "
                                "the position), so the sample spreads over the whole sequence")
        d["oracle"] = orc
    del inp, ids, o, chunks, ws_i, ws_a
    torch.cuda.empty_cache()
    return d


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
    ap.add_argument("--no-configs", action="store_true", help="skip the other workloads' sub-lines")
    ap.add_argument("--no-shared-index", action="store_true", help="skip the shared index-K head decode step")
    ap.add_argument("--no-large-k", action="store_true", help="skip the large-k (k 1024 of 16,384 blocks) decode step")
    ap.add_argument("--no-mxfp8", action="store_true", help="skip the decode step with MXFP8 index keys")
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
