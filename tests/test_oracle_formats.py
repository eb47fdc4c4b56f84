"""Pins for the oracle's element codecs and the pages' KV-size example.

Every codec is checked against a library implementation of the same format
(numpy float16, torch bfloat16 and float8_e4m3fn) or against the format's
fixed points (largest finite value, subnormal spacing, ties to even)."""

import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def same_or_both_nan(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    both_nan = np.isnan(a) & np.isnan(b)
    return np.all(both_nan | (a == b)) and np.all(np.signbit(a[~both_nan]) == np.signbit(b[~both_nan]))


def test_f16_all_codes_match_numpy():
    codes = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.decode(codes, oracle.F16)
    ref = codes.view(np.float16).astype(np.float64)
    assert same_or_both_nan(ours, ref)


def test_bf16_all_codes_match_torch():
    codes = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.decode(codes, oracle.BF16)
    ref = torch.from_numpy(codes.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    assert same_or_both_nan(ours, ref)


def test_e4m3_all_codes_match_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.decode(codes, oracle.E4M3)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert same_or_both_nan(ours, ref)
    assert np.nanmax(ours) == 448.0 and np.nanmin(ours) == -448.0
    assert np.isnan(ours[0x7F]) and np.isnan(ours[0xFF])
    assert np.sum(np.isnan(ours)) == 2  # no infinities, one NaN code per sign
    assert ours[1] == 2.0 ** -9  # smallest subnormal


def test_e4m3_encode_roundtrips_every_finite_code():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    vals = oracle.decode(codes, oracle.E4M3).astype(np.float32)
    back = oracle.e4m3_encode(vals)
    assert np.array_equal(back, codes)


def _finite_grid():
    codes = np.arange(0, 0x7F, dtype=np.uint8)  # non-negative finite codes, ascending
    return oracle.decode(codes, oracle.E4M3)


def test_e4m3_encode_ties_to_even_at_every_midpoint():
    grid = _finite_grid()
    for i in range(len(grid) - 1):
        lo, hi = grid[i], grid[i + 1]
        mid = np.float32((lo + hi) / 2)
        assert float(mid) == (lo + hi) / 2  # midpoints are exact in fp32
        want = i if i % 2 == 0 else i + 1  # even mantissa = even code
        got = oracle.e4m3_encode(np.array([mid, -mid], dtype=np.float32))
        assert got[0] == want, (lo, hi)
        assert got[1] == (want | 0x80)
        # just off the midpoint rounds to the nearer neighbour
        above = np.nextafter(mid, np.float32(np.inf))
        below = np.nextafter(mid, np.float32(0))
        assert oracle.e4m3_encode(np.array([above]))[0] == i + 1
        assert oracle.e4m3_encode(np.array([below]))[0] == i


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(451)
    x = np.concatenate([
        rng.standard_normal(200000).astype(np.float32) * np.float32(60.0),
        (rng.standard_normal(50000) * 2.0 ** -7).astype(np.float32),  # subnormal range
        rng.uniform(-463.9, 463.9, 50000).astype(np.float32),
    ])
    x = x[np.abs(x) < 464.0]
    ours = oracle.e4m3_encode(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    # torch's cast and ours agree bit for bit below the saturation threshold
    assert np.array_equal(ours, ref)


def test_e4m3_encode_saturates_and_keeps_nan():
    x = np.array([448.0, 460.0, 464.0, 464.0001, 480.0, 1e6, np.inf, -500.0, -np.inf, np.nan],
                 dtype=np.float32)
    got = oracle.e4m3_encode(x)
    assert list(got[:9]) == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE]
    assert got[9] == 0x7F


def test_e4m3_encode_underflow_and_signed_zero():
    tiny = np.float32(2.0 ** -10)  # half the smallest subnormal: tie -> even (zero)
    got = oracle.e4m3_encode(np.array([tiny, -tiny, np.float32(3 * 2.0 ** -11), 0.0, -0.0],
                                      dtype=np.float32))
    assert list(got) == [0x00, 0x80, 0x01, 0x00, 0x80]


def test_kv_size_worked_example():
    with open(os.path.join(GOLDEN, "kv_size.txt")) as f:
        row = [ln for ln in f if ln.strip() and not ln.startswith("#")][0].split()
    seq, layers, heads, hd, eb, exact = (int(v) for v in row[:6])
    per_req_gb, reqs, total_gb = float(row[6]), int(row[7]), float(row[8])
    b = oracle.kv_cache_bytes(seq, layers, heads, hd, eb)
    assert b == exact == 2 ** 30
    assert round(b / 1e9, 2) == per_req_gb
    assert round(reqs * b / 1e9) == total_gb
    assert math.isclose(reqs * b / 1e9, 34.36, abs_tol=5e-3)
