"""The FMA-pipe 2^x of the prefill softmax, restated in float32 NumPy with the constants read from
its source: it must stay within 1e-4 relative of 2^x wherever P is not negligible, and 2^-125 must
stand for everything below (the kernels store P in bf16, whose unit round-off is 2^-9)."""
from __future__ import annotations

import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "block_sparse_long_12_b200", "csrc", "prefill_attn.cu")


def coefficients():
    body = open(SRC).read().split("float exp2_poly(float x) {", 1)[1].split("}", 1)[0]
    c = [float(v) for v in re.findall(r"([0-9]+\.[0-9]*)f", body)]
    # clamp, shift constant (twice), then the cubic from the highest power down
    assert c[0] == 125.0 and c[1] == c[2] == 12582912.0, c
    return np.float32(c[3]), np.float32(c[4]), np.float32(c[5]), np.float32(c[6])


def exp2_poly(x: np.ndarray) -> np.ndarray:
    c3, c2, c1, c0 = coefficients()
    f32 = np.float32
    x = np.maximum(x.astype(f32), f32(-125.0))
    t = (x + f32(12582912.0)).astype(f32)
    f = (x - (t - f32(12582912.0))).astype(f32)
    p = (f * c3 + c2).astype(f32)  # the kernel fuses these multiply-adds; the bound below has room for it
    p = (p * f + c1).astype(f32)
    p = (p * f + c0).astype(f32)
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.astype(np.uint32).view(np.float32)


def test_relative_error_against_exp2():
    x = np.linspace(-124.0, 0.0, 2_000_001, dtype=np.float32)
    got = exp2_poly(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(got / want - 1.0)) < 1e-4


def test_exact_integers_and_the_floor():
    x = np.arange(-124, 1, dtype=np.float32)
    assert np.max(np.abs(exp2_poly(x) / np.exp2(x.astype(np.float64)) - 1.0)) < 1e-4
    low = exp2_poly(np.array([-125.0, -300.0, -np.inf], np.float32))
    assert np.allclose(low, 2.0 ** -125, rtol=1e-4)
