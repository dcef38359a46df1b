"""MSA oracle: plain fp64 CPU statement of MiniMax Sparse Attention.

TEST INFRASTRUCTURE ONLY.  Imported by ``tests/``, by ``__graft_entry__.smoke()``
and by the CPU-baseline leg of ``bench.py``; the product package never imports
it and shares no code with it.

Two independent formulations live here:

* ``msa_oracle.c`` (built into ``liboracle_msa.so``), plain loops in fp64,
  the oracle proper, wrapped below through ctypes;
* ``numpy_twin.py``, a vectorised NumPy restatement written differently
  (rank counting instead of sorting, masks instead of gathers), used only to
  cross-check the C code;
* ``mxfp8.py``, the MXFP8 storage of index keys (E4M3 elements, one E8M0 scale
  per 32): its quantiser and its exact decoding to float32, after which Step 1
  runs through the C oracle like every other workload.

Method source: "MiniMax wird duenn: M3-Attention anhand eines einzigen
Diagramms entschluesselt" (atlascloud.ai), section 1, Step 1 (index branch:
index query . index key, block max pool, TopK per group) and Step 2 (sparse
branch: every head of the group attends over the group's selected blocks of
the real K/V), with Figure 1.

Inputs are NumPy arrays holding the exact bits the GPU sees: ``float32`` for
the fp32 workload, ``uint16`` bf16 bit patterns otherwise.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "msa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle_msa.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (fp64, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", _SRC, "-o", _LIB_PATH, "-lm"]
        subprocess.check_call(cmd)
    return _LIB_PATH


class _Params(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int), ("n_q_heads", ctypes.c_int), ("n_kv_heads", ctypes.c_int),
        ("n_idx_k_heads", ctypes.c_int), ("head_dim", ctypes.c_int), ("idx_dim", ctypes.c_int),
        ("block_size", ctypes.c_int), ("top_k", ctypes.c_int), ("q_len", ctypes.c_int),
        ("q_start", ctypes.c_int), ("max_seq_len", ctypes.c_int), ("dtype", ctypes.c_int),
        ("dense", ctypes.c_int), ("prefill", ctypes.c_int), ("force_sink_local", ctypes.c_int),
        ("softmax_scale", ctypes.c_double),
    ]


@dataclass
class Params:
    """Shape and mode of one MSA call (see the C header comment for layouts)."""
    batch: int
    n_q_heads: int
    n_kv_heads: int
    n_idx_k_heads: int
    head_dim: int
    idx_dim: int
    block_size: int
    top_k: int
    q_len: int
    q_start: int
    max_seq_len: int
    dtype: str  # "f32" or "bf16"
    softmax_scale: float
    prefill: bool = False
    dense: bool = False
    force_sink_local: bool = False  # block 0 and the query's own block always selected

    def c(self) -> _Params:
        return _Params(self.batch, self.n_q_heads, self.n_kv_heads, self.n_idx_k_heads,
                       self.head_dim, self.idx_dim, self.block_size, self.top_k, self.q_len,
                       self.q_start, self.max_seq_len, 0 if self.dtype == "f32" else 1,
                       int(self.dense), int(self.prefill), int(self.force_sink_local),
                       float(self.softmax_scale))


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.POINTER(_Params)
        vp, ip, dp = ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p
        lib.oracle_token_scores.argtypes = [P, vp, vp, ip, ip, ip, ip, dp]
        lib.oracle_block_scores.argtypes = [P, dp, ip, dp]
        lib.oracle_block_scores.restype = ctypes.c_int
        lib.oracle_topk.argtypes = [P, dp, ip, vp, dp, dp, dp]
        lib.oracle_attention_row.argtypes = [P, vp, vp, vp, ip, ip, ip, ip, vp, ip, dp, dp, dp]
        lib.oracle_attention_row.restype = ctypes.c_int
        lib.oracle_msa_rows.argtypes = [P, vp, vp, vp, vp, vp, vp, ip, vp, vp, vp, dp, dp, dp, dp, dp, ip]
        _lib = lib
    return _lib


def _raw(x: np.ndarray, p: Params) -> np.ndarray:
    want = np.float32 if p.dtype == "f32" else np.uint16
    if x.dtype != want:
        raise TypeError(f"oracle expects {np.dtype(want).name} storage for dtype {p.dtype}, got {x.dtype}")
    return np.ascontiguousarray(x)


def _ptr(x: np.ndarray):
    return ctypes.c_void_p(x.ctypes.data)


def token_scores(p: Params, q_idx, k_idx, b: int, t: int, g: int, pos: int) -> np.ndarray:
    """Index-branch token scores s_j, j = 0..pos, for (b, t, group g)."""
    q_idx, k_idx = _raw(q_idx, p), _raw(k_idx, p)
    out = np.empty(pos + 1, np.float64)
    _load().oracle_token_scores(ctypes.byref(p.c()), _ptr(q_idx), _ptr(k_idx), b, t, g, pos, _ptr(out))
    return out


def block_scores(p: Params, s: np.ndarray, pos: int) -> np.ndarray:
    """Block max pool of token scores over causally visible tokens."""
    s = np.ascontiguousarray(s, np.float64)
    out = np.empty(pos // p.block_size + 1, np.float64)
    _load().oracle_block_scores(ctypes.byref(p.c()), _ptr(s), pos, _ptr(out))
    return out


def topk(p: Params, S: np.ndarray):
    """TopK over block scores: (ids int32[k], scores f64[k], kth, kth_next)."""
    S = np.ascontiguousarray(S, np.float64)
    ids = np.empty(p.top_k, np.int32)
    sc = np.empty(p.top_k, np.float64)
    kth = np.empty(1, np.float64)
    kn = np.empty(1, np.float64)
    _load().oracle_topk(ctypes.byref(p.c()), _ptr(S), len(S), _ptr(ids), _ptr(sc), _ptr(kth), _ptr(kn))
    return ids, sc, float(kth[0]), float(kn[0])


def attention_row(p: Params, q, k, v, b: int, t: int, h: int, pos: int, ids):
    """Sparse-branch attention of one query head: (o f64[D], lse, w f64[pos+1], n_keys)."""
    q, k, v = _raw(q, p), _raw(k, p), _raw(v, p)
    ids = np.ascontiguousarray(ids, np.int32)
    o = np.empty(p.head_dim, np.float64)
    lse = np.empty(1, np.float64)
    w = np.empty(pos + 1, np.float64)
    n = _load().oracle_attention_row(ctypes.byref(p.c()), _ptr(q), _ptr(k), _ptr(v), b, t, h, pos,
                                     _ptr(ids), len(ids), _ptr(o), _ptr(lse), _ptr(w))
    return o, float(lse[0]), w, n


def msa_rows(p: Params, seq_lens, q, q_idx, k, v, k_idx, rows, ids_in=None, attention: bool = True) -> dict:
    """Steps 1 and 2 for the (b, t) query rows listed in ``rows`` (shape [n, 2]).

    Returns a dict with ``ids`` int32[n, G, k], ``top_scores`` f64[n, G, k],
    ``kth``/``kth_next`` f64[n, G] (k-th and (k+1)-th block scores of the full
    ranking, NaN where absent), ``o`` f64[n, Hq, D] and ``lse`` f64[n, Hq].
    With ``ids_in`` the given selection drives Step 2 instead; with
    ``attention=False`` only Step 1 runs (``o``/``lse`` stay NaN).
    """
    q, q_idx, k, v, k_idx = (_raw(x, p) for x in (q, q_idx, k, v, k_idx))
    rows = np.ascontiguousarray(np.asarray(rows, np.int32).reshape(-1, 2))
    n = rows.shape[0]
    G, K = p.n_kv_heads, p.top_k
    sl = np.ascontiguousarray(np.asarray(seq_lens if seq_lens is not None else [0] * p.batch, np.int32))
    ids = np.empty((n, G, K), np.int32)
    ts = np.full((n, G, K), -np.inf)
    kth = np.empty((n, G), np.float64)
    kn = np.empty((n, G), np.float64)
    o = np.full((n, p.n_q_heads, p.head_dim), np.nan)
    lse = np.full((n, p.n_q_heads), np.nan)
    idin = None if ids_in is None else np.ascontiguousarray(np.asarray(ids_in, np.int32).reshape(n, G, K))
    _load().oracle_msa_rows(ctypes.byref(p.c()), _ptr(sl), _ptr(q), _ptr(q_idx), _ptr(k), _ptr(v),
                            _ptr(k_idx), n, _ptr(rows), None if idin is None else _ptr(idin),
                            _ptr(ids), _ptr(ts), _ptr(kth), _ptr(kn), _ptr(o), _ptr(lse), int(attention))
    return {"ids": ids, "top_scores": ts, "kth": kth, "kth_next": kn, "o": o, "lse": lse}


def set_threads(n: int | None) -> int:
    """Threads the oracle's OpenMP loops use from now on (None: all cores); returns the count set."""
    n = int(n) if n else (os.cpu_count() or 1)
    _load()
    ctypes.CDLL("libgomp.so.1").omp_set_num_threads(n)
    return n


def to_f64(x: np.ndarray) -> np.ndarray:
    """Exact widening of stored f32 / bf16-bit arrays to float64."""
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return x.astype(np.float64)
