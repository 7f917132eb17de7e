"""Pins for the oracle's number formats (CPU only).

The E4M3 / E2M1 / E8M0 codecs are fixed by the OCP FP8 and MX format
definitions; the IndexerQuantCache page (计算公式, 参数说明) names the formats and
the round(x / scale) rule.  Each codec is checked against something other than
itself: torch's own float8 types (a library routine), hand-derived golden points
(tests/golden), and the defining properties of nearest rounding.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle


def _points(path):
    rows = []
    with open(path) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            rows.append(line.split())
    return rows


def test_e4m3_decode_matches_torch_for_every_code():
    # torch.float8_e4m3fn is the OCP E4M3 "fn" type: an independent decoder.
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    ours = np.array([oracle.e4m3_value(c) for c in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(ours))
    assert np.array_equal(ref[~nan], ours[~nan])
    assert np.array_equal(np.signbit(ref[~nan]), np.signbit(ours[~nan]))
    assert nan.sum() == 2  # 0x7F and 0xFF only


def test_e4m3_encode_matches_torch_cast_in_range():
    # torch's float32 -> float8_e4m3fn cast rounds to nearest-even; it maps
    # overflow to NaN, so only |v| <= 448 is compared.
    g = torch.Generator().manual_seed(11)
    parts = [
        torch.randn(20000, generator=g) * 50,
        torch.randn(20000, generator=g) * 0.01,   # subnormal range
        torch.rand(20000, generator=g) * 448,
    ]
    # exact midpoints between neighbouring codes (ties) and the codes themselves
    vals = torch.arange(0, 0x7E, dtype=torch.uint8).view(torch.float8_e4m3fn).float()
    mids = (vals[:-1] + vals[1:]) / 2
    parts += [vals, mids, -mids, -vals]
    v = torch.cat(parts).clamp(-448, 448)
    ref = v.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = np.array([oracle.e4m3_encode(float(x)) for x in v.numpy()], np.uint8)
    assert np.array_equal(ref, ours)


def test_e4m3_golden_points(golden_dir):
    for kind, value, code in _points(os.path.join(golden_dir, "e4m3_points.txt")):
        value, code = float(value), int(code, 16)
        if kind == "dec":
            got = oracle.e4m3_value(code)
            assert got == value and math.copysign(1, got) == math.copysign(1, value), (code, got)
        else:
            assert oracle.e4m3_encode(value) == code, (value, hex(oracle.e4m3_encode(value)))


def test_e2m1_golden_points(golden_dir):
    for kind, value, code in _points(os.path.join(golden_dir, "e2m1_points.txt")):
        value, code = float(value), int(code, 16)
        if kind == "dec":
            got = oracle.e2m1_value(code)
            assert got == value and math.copysign(1, got) == math.copysign(1, value), (code, got)
        else:
            assert oracle.e2m1_encode(value) == code, (value, oracle.e2m1_encode(value))


def test_e2m1_encode_is_nearest_grid_point():
    # Defining property of round-to-nearest: no grid value is strictly closer;
    # at an exact tie the chosen code is even.  Grid from the torch float4 type
    # decode would also work; the magnitudes are listed by the MX spec.
    grid = {c: oracle.e2m1_value(c) for c in range(16)}
    rng = np.random.default_rng(5)
    xs = np.concatenate([rng.uniform(-7, 7, 4000), np.arange(-6.5, 6.51, 0.25)]).astype(np.float32)
    for x in xs:
        c = oracle.e2m1_encode(float(x))
        if abs(x) >= 6:
            assert c & 7 == 7
            continue
        d = abs(grid[c] - x)
        for c2, v2 in grid.items():
            assert abs(v2 - x) >= d
            if abs(v2 - x) == d and abs(v2) != abs(grid[c]):
                assert c % 2 == 0
        assert (c >> 3) == (1 if np.signbit(x) else 0)


def test_e8m0_decode_matches_torch_for_every_code():
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e8m0fnu).double().numpy()
    ours = np.array([oracle.e8m0_value(c) for c in range(256)])
    assert np.isnan(ref[255]) and np.isnan(ours[255])
    assert np.array_equal(ref[:255], ours[:255])


def test_e8m0_ceil_golden(golden_dir):
    for s, e in _points(os.path.join(golden_dir, "e8m0_ceil_points.txt")):
        assert oracle.e8m0_ceil(float(np.float32(s))) == int(e), (s, e)


def test_e8m0_ceil_is_smallest_power_of_two_not_below():
    rng = np.random.default_rng(7)
    s = np.concatenate([
        np.exp2(rng.uniform(-126, 126, 3000)),
        np.exp2(np.arange(-126, 127, dtype=np.float64)),
    ]).astype(np.float32)
    for x in s:
        e = oracle.e8m0_ceil(float(x))
        val = oracle.e8m0_value(e)
        assert val >= float(x)
        assert val / 2 < float(x)


def test_e5m2_decode_matches_torch_for_every_code():
    # torch.float8_e5m2 is the OCP E5M2 type: an independent decoder.
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e5m2).double().numpy()
    ours = np.array([oracle.e5m2_value(c) for c in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(ours))
    assert np.array_equal(ref[~nan], ours[~nan])
    assert np.array_equal(np.signbit(ref[~nan]), np.signbit(ours[~nan]))
    assert nan.sum() == 6 and np.isinf(ours).sum() == 2


def test_e5m2_encode_matches_torch_cast_in_range():
    # torch's float32 -> float8_e5m2 cast rounds to nearest-even; it maps
    # overflow to infinity, so only |v| <= 57344 is compared.
    g = torch.Generator().manual_seed(13)
    parts = [
        torch.randn(20000, generator=g) * 2000,
        torch.randn(20000, generator=g) * 1e-4,   # subnormal range
        torch.rand(20000, generator=g) * 57344,
    ]
    vals = torch.arange(0, 0x7C, dtype=torch.uint8).view(torch.float8_e5m2).float()
    mids = (vals[:-1] + vals[1:]) / 2
    parts += [vals, mids, -mids, -vals]
    v = torch.cat(parts).clamp(-57344, 57344)
    ref = v.to(torch.float8_e5m2).view(torch.uint8).numpy()
    ours = np.array([oracle.e5m2_encode(float(x)) for x in v.numpy()], np.uint8)
    assert np.array_equal(ref, ours)


def test_e5m2_golden_points(golden_dir):
    for kind, value, code in _points(os.path.join(golden_dir, "e5m2_points.txt")):
        value, code = float(value), int(code, 16)
        if kind == "dec":
            got = oracle.e5m2_value(code)
            assert got == value and math.copysign(1, got) == math.copysign(1, value), (code, got)
        else:
            assert oracle.e5m2_encode(value) == code, (value, hex(oracle.e5m2_encode(value)))


def test_e8m0_floor_golden(golden_dir):
    for s, e in _points(os.path.join(golden_dir, "e8m0_floor_points.txt")):
        assert oracle.e8m0_floor(float(np.float32(s))) == int(e), (s, e)


def test_e8m0_floor_is_largest_power_of_two_not_above():
    rng = np.random.default_rng(9)
    s = np.concatenate([
        np.exp2(rng.uniform(-126, 126, 3000)),
        np.exp2(np.arange(-126, 127, dtype=np.float64)),
    ]).astype(np.float32)
    for x in s:
        e = oracle.e8m0_floor(float(x))
        val = oracle.e8m0_value(e)
        assert val <= float(x)
        assert val * 2 > float(x)
