"""Pins for the oracle's number formats (OCP E4M3, bf16).

The e4m3 codec is pinned to the named points of the OCP FP8 specification
(tests/golden/e4m3_spec_points.txt) and, exhaustively, to torch's
float8_e4m3fn conversion, an independent library implementation.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _spec_points():
    pts = []
    with open(os.path.join(GOLD, "e4m3_spec_points.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                c, v = line.split()
                pts.append((int(c, 16), float(v)))
    return pts


def test_e4m3_spec_points():
    for code, val in _spec_points():
        got = oracle.e4m3_decode(code)
        if math.isnan(val):
            assert math.isnan(got)
        else:
            assert got == val and math.copysign(1, got) == math.copysign(1, val), hex(code)
            assert oracle.e4m3_encode(val) == code, hex(code)


def test_e4m3_decode_all_codes_vs_torch():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float32).numpy()
    for c in range(256):
        got = oracle.e4m3_decode(c)
        if np.isnan(ref[c]):
            assert math.isnan(got)
        else:
            assert got == float(ref[c]), c


def test_e4m3_encode_roundtrip_and_midpoints_vs_torch():
    finite = [c for c in range(256) if (c & 0x7F) != 0x7F]
    for c in finite:
        assert oracle.e4m3_encode(oracle.e4m3_decode(c)) == c
    # every midpoint between adjacent non-negative codes (ties to even) and
    # points a quarter-step either side of it
    vals = []
    for c in range(0, 0x7E):
        a, b = oracle.e4m3_decode(c), oracle.e4m3_decode(c + 1)
        m = 0.5 * (a + b)
        vals += [m, m - 0.25 * (b - a), m + 0.25 * (b - a)]
    vals = np.array(vals, dtype=np.float32)
    vals = np.concatenate([vals, -vals])
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    for v, r in zip(vals, ref):
        assert oracle.e4m3_encode(float(v)) == int(r), float(v)


def test_e4m3_encode_random_vs_torch():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal(20000) * np.exp(rng.uniform(-9, 6, 20000))).astype(np.float32)
    x = np.clip(x, -448, 448)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(float(v)) for v in x], dtype=np.uint8)
    # torch keeps the sign of values that round to zero; so does the oracle
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("v", [448.0, 449.0, 463.99, 464.0, 1e6, 3.4e38, float("inf")])
def test_e4m3_saturates(v):
    assert oracle.e4m3_encode(v) == 0x7E
    assert oracle.e4m3_encode(-v) == 0xFE


def test_bf16_decode_vs_torch():
    rng = np.random.default_rng(2)
    bits = rng.integers(0, 1 << 16, size=5000).astype(np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float32).numpy()
    for b, r in zip(bits, ref):
        g = oracle.bf16_decode(int(b))
        if np.isnan(r):
            assert math.isnan(g)
        else:
            assert g == float(r)
