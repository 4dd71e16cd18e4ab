"""Pins for the oracle's number formats (e4m3fn codec, bf16 rounding).

The codec is written from the OCP FP8 definition; here it is checked against the OCP
table values (tests/golden/e4m3fn_ocp.txt) and against torch's own float8_e4m3fn and
bfloat16 casts, which share no code with it.
"""
import os

import numpy as np
import pytest
import torch

from oracle import fp8

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e4m3fn_ocp.txt")


def test_decode_matches_ocp_table():
    n = 0
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        code, val = line.split()
        got = fp8.e4m3_decode(np.array([int(code, 16)], np.uint8))[0]
        if val == "nan":
            assert np.isnan(got)
        else:
            assert got == float(val) and np.signbit(got) == val.startswith("-"), code
        n += 1
    assert n >= 10


def test_decode_all_codes_match_torch():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = fp8.e4m3_decode(codes.numpy())
    assert np.array_equal(np.isnan(ref), np.isnan(got))
    ok = ~np.isnan(ref)
    assert np.array_equal(ref[ok], got[ok])
    assert np.array_equal(np.signbit(ref[ok]), np.signbit(got[ok]))


def _all_finite_values():
    v = fp8.E4M3_TABLE[:127]
    return v


def test_encode_roundtrip_every_code():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    vals = fp8.e4m3_decode(codes)
    back = fp8.e4m3_encode(vals)
    # -0.0 encodes to 0x80, +0.0 to 0x00
    assert np.array_equal(back, codes)


def test_encode_ties_and_sweep_match_torch():
    v = _all_finite_values()
    mids = (v[:-1] + v[1:]) / 2          # exact ties between neighbours
    quarter = v[:-1] + (v[1:] - v[:-1]) / 4
    rng = np.random.default_rng(0)
    rand = rng.uniform(-460, 460, 200000)
    small = rng.uniform(-0.03, 0.03, 50000)
    x = np.concatenate([mids, -mids, quarter, -quarter, rand, small, v, -v]).astype(np.float32)
    x = x[np.abs(x) < 464.0]             # beyond 464 torch gives NaN where satfinite saturates
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = fp8.e4m3_encode(x)
    bad = np.nonzero(ref != got)[0]
    assert bad.size == 0, (x[bad[:5]], ref[bad[:5]], got[bad[:5]])


def test_encode_ties_go_to_even_mantissa():
    # 1.0625 is halfway between 1.0 (mantissa 000) and 1.125 (001): goes to 1.0
    assert fp8.e4m3_encode(np.array([1.0625]))[0] == 0x38
    # 1.1875 halfway between 1.125 (001) and 1.25 (010): goes to 1.25
    assert fp8.e4m3_encode(np.array([1.1875]))[0] == 0x3A
    # half of the smallest subnormal rounds to zero, 3/4 of it rounds up
    assert fp8.e4m3_encode(np.array([2.0 ** -10]))[0] == 0x00
    assert fp8.e4m3_encode(np.array([0.75 * 2.0 ** -9]))[0] == 0x01


def test_encode_saturates_and_nan():
    x = np.array([448.0, 463.99, 464.0, 500.0, 1e9, np.inf, -1e9, -np.inf, np.nan])
    got = fp8.e4m3_encode(x)
    assert list(got) == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE, 0x7F]


def test_bf16_round_matches_torch():
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.standard_normal(100000) * 10.0 ** rng.integers(-8, 8, 100000),
        # exact ties: bf16 values plus half an ulp
        (np.arange(1, 1000, dtype=np.float32) * np.float32(2.0 ** -7) + np.float32(1.0)) +
        np.float32(2.0 ** -8),
    ]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = fp8.bf16_round(x.astype(np.float64))
    assert np.array_equal(ref, got)
    bits = fp8.bf16_bits(got)
    assert np.array_equal(fp8.bf16_from_bits(bits), got)
