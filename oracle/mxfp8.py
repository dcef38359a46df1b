"""MXFP8 storage of index keys for the oracle.  TEST INFRASTRUCTURE ONLY (imported by ``tests/`` and
``bench.py``'s CPU legs; the product package never imports it).

Reading: the pages name MXFP8 as the format of the official quantised checkpoints (docs.clore.ai
"MiniMax M3", the deployment table's "MXFP8 offiziell" row and the pre-quantised checkpoint list)
and say nothing more about it.  The plainest reading of MXFP8 is the microscaling format: blocks of
32 consecutive elements share one power-of-two scale stored as an 8-bit exponent (E8M0: value
2^(E - 127), 255 reserved for NaN), and every element is an FP8 E4M3 number (1 sign bit, 4
exponent bits with bias 7, 3 mantissa bits; exponent field 0 gives the subnormals m/8 * 2^-6; no
infinities; S.1111.111 is NaN; the largest finite magnitude is 1.75 * 2^8 = 448).  Here it is the
storage of the index keys k_idx only (one scale per 32 index dimensions of a token's row), a
bandwidth lever for the decode index scan; the index query and Step 2 stay bf16.

Quantisation of one block V (the conversion rule of the microscaling format): the shared exponent
is floor(log2 max|V_i|) - 8 (8 = the exponent of E4M3's largest normal), clamped to E8M0's range
[-127, 127]; every V_i / 2^shared is rounded to the nearest E4M3 value, ties to the even mantissa,
magnitudes beyond 448 saturating to 448 (the ratio stays below 2^9 = 512).  An all-zero block
takes the smallest scale (byte 0) and zero codes.

Decoding is exact in float32 for every code this quantiser writes from bf16 inputs, so the oracle
runs Step 1 in fp64 on the decoded keys (``decode``) through the same C oracle as every other
workload.
"""
from __future__ import annotations

import math

import numpy as np

BLOCK = 32          # elements per shared scale
E4M3_EMAX = 8       # exponent of the largest normal E4M3 number
E4M3_MAX = 448.0


def e4m3_value(code: int) -> float:
    """The real number an E4M3 code denotes, from its bit fields."""
    sign = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return math.nan
    if e == 0:
        return sign * (m / 8.0) * 2.0 ** -6
    return sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)


E4M3_TABLE = np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)
# the non-negative finite magnitudes in code order (codes 0..126): strictly increasing
_POS = E4M3_TABLE[:127]


def e8m0_value(byte: int) -> float:
    return math.nan if byte == 255 else 2.0 ** (byte - 127)


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """Round each value to the nearest E4M3 number, ties to the even code (the even mantissa),
    magnitudes of 448 and beyond saturating to 448; the sign is kept, also for zero.  uint8 codes."""
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), E4M3_MAX)
    hi = np.clip(np.searchsorted(_POS, a, side="left"), 0, 126)   # first magnitude >= a
    lo = np.clip(hi - 1, 0, 126)
    d_lo, d_hi = a - _POS[lo], _POS[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    mag = np.where(pick_hi, hi, lo).astype(np.uint8)
    return np.where(np.signbit(x), mag | np.uint8(0x80), mag).astype(np.uint8)


def quantize(v: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """MXFP8 quantisation of rows of values (last axis a multiple of 32): (codes uint8 [..., n],
    scale bytes uint8 [..., n / 32])."""
    v = np.asarray(v, dtype=np.float64)
    n = v.shape[-1]
    assert n % BLOCK == 0
    blocks = v.reshape(v.shape[:-1] + (n // BLOCK, BLOCK))
    amax = np.max(np.abs(blocks), axis=-1)
    _, e = np.frexp(amax)  # amax = f * 2^e with f in [1/2, 1): floor(log2 amax) = e - 1
    shared = np.where(amax > 0, np.clip(e - 1 - E4M3_EMAX, -127, 127), -127).astype(np.int64)
    codes = e4m3_encode(blocks * np.ldexp(1.0, -shared)[..., None])
    return codes.reshape(v.shape), (shared + 127).astype(np.uint8)


def decode(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """The values an MXFP8 row stands for, as float32 (exact for scales of the quantiser above)."""
    codes = np.asarray(codes, dtype=np.uint8)
    n = codes.shape[-1]
    vals = E4M3_TABLE[codes].reshape(codes.shape[:-1] + (n // BLOCK, BLOCK))
    sb = np.asarray(scales).astype(np.int64)
    sc = np.where(sb == 255, np.nan, np.ldexp(1.0, sb - 127))
    out = (vals * sc[..., None]).reshape(codes.shape)
    assert np.array_equal(out.astype(np.float32).astype(np.float64), out, equal_nan=True), "not exact in float32"
    return out.astype(np.float32)
