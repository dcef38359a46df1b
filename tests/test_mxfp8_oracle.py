"""Pins of the oracle's MXFP8 index-key storage (oracle/mxfp8.py) against what the format fixes:
E4M3 values from their bit fields checked against torch's float8_e4m3fn (a library decoding), the
encoder's round-to-nearest-even against torch's conversion, hand-worked blocks of the shared-scale
rule, and exactness of the decoded keys in float32.  Reading of the pages: MXFP8, named by
docs.clore.ai "MiniMax M3" as the official checkpoints' format, taken as the microscaling format
(32 E4M3 elements per E8M0 power-of-two scale)."""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

from oracle import mxfp8


def test_e4m3_table_equals_torch_float8_e4m3fn():
    lib = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(lib, mxfp8.E4M3_TABLE, equal_nan=True)


@pytest.mark.parametrize("code,value", [
    (0x00, 0.0), (0x01, 2.0 ** -9), (0x07, 7 * 2.0 ** -9), (0x08, 2.0 ** -6), (0x38, 1.0), (0x3C, 1.5),
    (0x40, 2.0), (0x70, 128.0), (0x78, 256.0), (0x7E, 448.0), (0xB8, -1.0), (0xFE, -448.0),
])
def test_e4m3_values_of_the_format(code, value):
    assert mxfp8.E4M3_TABLE[code] == value
    assert mxfp8.e4m3_encode(np.array([value]))[0] == code


def test_e4m3_nan_and_signed_zero():
    assert math.isnan(mxfp8.E4M3_TABLE[0x7F]) and math.isnan(mxfp8.E4M3_TABLE[0xFF])
    assert mxfp8.E4M3_TABLE[0x80] == 0.0 and math.copysign(1.0, mxfp8.E4M3_TABLE[0x80]) < 0
    assert mxfp8.e4m3_encode(np.array([-0.0, -1e-9]))[0] == 0x80
    pos = mxfp8.E4M3_TABLE[:127]
    assert (np.diff(pos) > 0).all(), "magnitudes must increase with the code"


def test_e4m3_encode_equals_torch_round_to_nearest_even():
    rng = np.random.default_rng(3)
    x = rng.standard_normal(100_000) * rng.choice([1e-3, 0.05, 1.0, 30.0, 200.0], 100_000)
    x = np.clip(x, -448.0, 448.0)
    # every midpoint between consecutive magnitudes: ties go to the even code
    pos = mxfp8.E4M3_TABLE[:127]
    mids = (pos[:-1] + pos[1:]) / 2
    x = np.concatenate([x, mids, -mids, pos, -pos])
    ours = mxfp8.e4m3_encode(x)
    lib = torch.tensor(x, dtype=torch.float64).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, lib)
    assert (ours[100_000:100_000 + len(mids)] % 2 == 0).all()


def test_e4m3_encode_saturates():
    assert list(mxfp8.e4m3_encode(np.array([448.0, 460.0, 500.0, 1e30, -1e30]))) == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE]


def test_block_scale_hand_worked():
    # max |v| = 3: floor(log2 3) = 1, shared exponent 1 - 8 = -7 (byte 120); v * 2^7
    v = np.zeros((1, 32))
    v[0, 0], v[0, 1], v[0, 2] = 1.0, -3.0, 0.7
    codes, scales = mxfp8.quantize(v)
    assert scales.tolist() == [[120]]
    assert codes[0, 0] == 0x70                      # 128 = 1.0 * 2^7
    assert codes[0, 1] == 0xFC                      # -384 = -1.5 * 2^8
    assert mxfp8.E4M3_TABLE[codes[0, 2]] == 88.0    # 0.7 * 128 = 89.6 -> 88 (1.375 * 2^6)
    assert (codes[0, 3:] == 0).all()
    # a block maximum just below a power of two saturates: 1.99 -> shared -8, 509.4 -> 448
    c, s = mxfp8.quantize(np.full((1, 32), 1.99))
    assert s.tolist() == [[119]] and (c == 0x7E).all()
    assert (mxfp8.decode(c, s) == np.float32(1.75)).all()
    # all zeros: the smallest scale, zero codes
    c, s = mxfp8.quantize(np.zeros((2, 64)))
    assert (s == 0).all() and (c == 0).all()


def test_quantize_error_bound_and_exact_decode():
    rng = np.random.default_rng(5)
    v = rng.standard_normal((2000, 64)) * rng.choice([1e-4, 1.0, 1e4], (2000, 1))
    v = torch.tensor(v).to(torch.bfloat16).double().numpy()  # the stored index keys are bf16
    codes, scales = mxfp8.quantize(v)
    d = mxfp8.decode(codes, scales).astype(np.float64)
    X = np.ldexp(1.0, scales.astype(np.int64) - 127)
    Xe = np.repeat(X, 32, axis=-1)
    sat = np.abs(v) > 448.0 * Xe
    normal = (np.abs(v) >= 2.0 ** -6 * Xe) & ~sat
    # normal range: half a unit in the last of 3 mantissa bits; below it: half of 2^-9 X; beyond
    # 448 X (a block maximum in [448, 512) X): saturated to 448 X
    assert (np.abs(d - v)[normal] <= 2.0 ** -4 * np.abs(v)[normal] * (1 + 1e-12)).all()
    small = np.abs(v) < 2.0 ** -6 * Xe
    assert (np.abs(d - v)[small] <= 2.0 ** -10 * Xe[small] * (1 + 1e-12)).all()
    assert (np.abs(d)[sat] == 448.0 * Xe[sat]).all() and sat.any()
    # every block's largest element maps to a magnitude in [256, 448] of its scale
    mags = (codes & 0x7F).reshape(2000, 2, 32).max(axis=-1)
    assert ((mags >= 0x78) & (mags <= 0x7E)).all()
