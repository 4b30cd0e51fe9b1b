"""Pins for oracle/formats.py: the E2M1 and E4M3 definitions and their rounding.

Checked against (a) the published format tables in tests/golden (OCP MX / OCP
FP8 definitions, ties-to-even rule), (b) two independent library routines
(ml_dtypes, torch float8), exhaustively over every code.
"""
import math
import os

import ml_dtypes
import numpy as np
import pytest
import torch

from oracle import formats

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e2m1_e4m3_points.txt")


def _golden(section):
    rows = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.split()
            if parts[0] == section:
                rows.append(parts[1:])
    assert rows, section
    return rows


def _same(a, b):
    if math.isnan(a) or math.isnan(b):
        return math.isnan(a) and math.isnan(b)
    return a == b and math.copysign(1, a) == math.copysign(1, b)


def test_e2m1_table_golden():
    for code, val in _golden("e2m1_value"):
        assert _same(formats.e2m1_value(int(code, 16)), float(val)), code


def test_e2m1_table_vs_ml_dtypes_exhaustive():
    lib = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    for c in range(16):
        assert _same(formats.E2M1_TABLE[c], lib[c]), c


def test_e2m1_round_golden():
    for v, code in _golden("e2m1_round"):
        got = int(formats.e2m1_encode(np.float32(float(v))))
        assert got == int(code, 16), (v, hex(got), code)


def test_e2m1_round_vs_ml_dtypes_dense():
    # every float32 on a fine grid over [-8, 8] plus all midpoints and their neighbours
    grid = np.linspace(-8, 8, 40001, dtype=np.float32)
    mids = (formats.E2M1_MAGNITUDES[1:] + formats.E2M1_MAGNITUDES[:-1]) / 2
    mids = np.concatenate([mids, -mids]).astype(np.float32)
    near = np.concatenate([np.nextafter(mids, np.float32(np.inf)), np.nextafter(mids, np.float32(-np.inf))])
    v = np.concatenate([grid, mids, near, np.float32([0.0, -0.0])])
    ours = formats.e2m1_encode(v)
    lib = v.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    np.testing.assert_array_equal(ours, lib)


def test_e4m3_table_golden():
    for code, val in _golden("e4m3_value"):
        assert _same(formats.e4m3_value(int(code, 16)), float(val)), code


def test_e4m3_table_vs_libraries_exhaustive():
    codes = np.arange(256, dtype=np.uint8)
    ml = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    th = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).double().numpy()
    for c in range(256):
        assert _same(formats.E4M3_TABLE[c], ml[c]), c
        assert _same(formats.E4M3_TABLE[c], th[c]), c
    assert formats.E4M3_TABLE[0x7E] == formats.E4M3_MAX == 448.0
    assert formats.E4M3_TABLE[0x01] == formats.E4M3_MIN_SUBNORMAL


def test_e4m3_round_golden():
    for v, code in _golden("e4m3_round"):
        got = int(formats.e4m3_encode_nonneg(np.float32(float(v))))
        assert got == int(code, 16), (v, hex(got), code)


def test_e4m3_round_vs_libraries():
    rng = np.random.default_rng(7)
    pos = formats.E4M3_TABLE[:0x7F]
    mids = (pos[1:] + pos[:-1]) / 2
    v = np.concatenate([
        pos, mids,
        np.nextafter(mids.astype(np.float32), np.float32(np.inf)).astype(np.float64),
        np.nextafter(mids.astype(np.float32), np.float32(0)).astype(np.float64),
        np.exp(rng.uniform(np.log(1e-5), np.log(460.0), 200000)),
    ]).astype(np.float32)
    v = v[v < 464]                                     # both libraries saturate/NaN above
    ours = formats.e4m3_encode_nonneg(v)
    ml = v.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    th = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(ours, ml)
    np.testing.assert_array_equal(ours, th)


def test_e4m3_saturates():
    v = np.float32([448, 463.9, 464, 480, 1e6, 3e38])
    assert np.all(formats.e4m3_encode_nonneg(v) == 0x7E)


def test_bf16_round_vs_torch():
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.standard_normal(100000) * 10.0 ** rng.integers(-20, 20, 100000),
                        [0.0, 1.0, -1.0, 1.00390625, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8]])
    x32 = x.astype(np.float32)                          # float32 inputs: torch rounds them once
    ours = formats.bf16_round(x32.astype(np.float64))
    th = torch.from_numpy(x32).to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(ours, th)


def test_bf16_round_keeps_sign_of_zero():
    # IEEE rounding: -0 stays -0, a negative value below half the smallest
    # bfloat16 subnormal (2^-133) rounds to -0; torch's conversion agrees
    x32 = np.float32([-0.0, 0.0, -1e-45, 1e-45, -3e-41, -2.0 ** -134])
    ours = formats.bf16_round(x32.astype(np.float64))
    th = torch.from_numpy(x32).to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(ours, th)
    np.testing.assert_array_equal(np.signbit(ours), np.signbit(th))
    assert np.signbit(ours[0]) and not np.signbit(ours[1]) and np.signbit(ours[2])


def test_bf16_round_ties_even():
    # 1 + 2^-8 lies halfway between 1 and 1 + 2^-7: ties to even -> 1
    assert formats.bf16_round(np.array([1.0 + 2 ** -8]))[0] == 1.0
    assert formats.bf16_round(np.array([1.0 + 3 * 2 ** -8]))[0] == 1.0 + 2 ** -6
    # a value that float32 would round first (double rounding) is rounded once here
    v = 1.0 + 2 ** -8 + 2 ** -30
    assert formats.bf16_round(np.array([v]))[0] == 1.0 + 2 ** -7
