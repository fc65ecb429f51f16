"""Pins for the oracle's scalar codecs (CPU only).

The E4M3 decoder is pinned to the values printed in the OCP OFP8 specification (golden file) and to
PyTorch's independent float8_e4m3fn implementation for all 256 codes; the encoder to PyTorch's
round-to-nearest-even cast inside the finite range, to brute-force nearest search, to exact ties and
to the saturation reading; the 16-bit decoders to numpy / PyTorch for every bit pattern.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
ALL_CODES = np.arange(256, dtype=np.uint8)
FINITE_CODES = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)


def torch_e4m3_decode(codes):
    return torch.from_numpy(np.asarray(codes, np.uint8).copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_e4m3_decode_matches_spec_table():
    spec = json.load(open(os.path.join(GOLDEN, "e4m3_ocp_values.json")))
    for row in spec["values"]:
        code = int(row["code"], 16)
        got = oracle.e4m3_to_double([code])[0]
        if row["value"] == "nan":
            assert math.isnan(got), row
        else:
            assert got == row["value"], row
            assert math.copysign(1.0, got) == math.copysign(1.0, row["value"]), row


def test_e4m3_decode_matches_torch_for_all_codes():
    ours = oracle.e4m3_to_double(ALL_CODES)
    ref = torch_e4m3_decode(ALL_CODES)
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    fin = ~np.isnan(ref)
    assert np.array_equal(ours[fin], ref[fin])
    assert np.array_equal(np.signbit(ours[fin]), np.signbit(ref[fin]))


def test_e4m3_decode_structure():
    v = oracle.e4m3_to_double(ALL_CODES)
    assert np.isnan(v).sum() == 2                      # only S.1111.111
    pos = v[:0x7F]
    assert np.all(np.diff(pos) > 0)                   # strictly increasing over 0x00..0x7E
    assert np.array_equal(v[0x80:0xFF], -v[0x00:0x7F])  # sign symmetry


def test_e4m3_encode_roundtrips_every_finite_code():
    values = oracle.e4m3_to_double(FINITE_CODES).astype(np.float32)
    assert np.array_equal(oracle.e4m3_from_float(values), FINITE_CODES)


def test_e4m3_encode_matches_torch_cast_in_range():
    rng = np.random.default_rng(7)
    x = np.concatenate([
        rng.standard_normal(200000).astype(np.float32) * 50,
        rng.uniform(-447.9, 447.9, 100000).astype(np.float32),
        (rng.standard_normal(100000) * 1e-2).astype(np.float32),
        (rng.standard_normal(50000) * 1e-4).astype(np.float32),
    ])
    x = x[np.abs(x) < 448]
    ours = oracle.e4m3_from_float(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_e4m3_encode_ties_go_to_even_code():
    pos = oracle.e4m3_to_double(np.arange(0x7F, dtype=np.uint8))
    mids = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)
    assert np.array_equal(mids.astype(np.float64), (pos[:-1] + pos[1:]) / 2)  # exact in float
    got = oracle.e4m3_from_float(mids)
    lower = np.arange(0x7E, dtype=np.uint8)
    expect = np.where(lower % 2 == 0, lower, lower + 1).astype(np.uint8)
    assert np.array_equal(got, expect)
    assert np.array_equal(oracle.e4m3_from_float(-mids), expect | 0x80)


def test_e4m3_encode_is_nearest_by_brute_force():
    rng = np.random.default_rng(11)
    x = (rng.standard_normal(4000) * rng.choice([1e-3, 1e-1, 1, 30, 200], 4000)).astype(np.float32)
    x = x[np.abs(x) < 448]
    codes = oracle.e4m3_from_float(x)
    table = oracle.e4m3_to_double(FINITE_CODES)
    for xi, ci in zip(x.astype(np.float64), codes):
        best = np.min(np.abs(table - xi))
        assert abs(oracle.e4m3_to_double([ci])[0] - xi) == best


def test_e4m3_encode_saturates_and_maps_nan_to_canonical_nan():
    big = np.array([448.0, 449.0, 463.9, 464.0, 480.0, 1e6, 3.0e38, np.inf], np.float32)
    assert np.all(oracle.e4m3_from_float(big) == 0x7E)
    assert np.all(oracle.e4m3_from_float(-big) == 0xFE)
    nan = np.array([np.nan], np.float32)
    assert oracle.e4m3_from_float(nan)[0] == 0x7F
    assert oracle.e4m3_from_float(-nan)[0] == 0x7F   # reading: NaN of either sign -> canonical NaN


def test_e4m3_encode_signed_zero_and_underflow():
    x = np.array([0.0, -0.0, 2.0 ** -10, -(2.0 ** -10), 2.0 ** -11, 1e-30], np.float32)
    assert list(oracle.e4m3_from_float(x)) == [0x00, 0x80, 0x00, 0x80, 0x00, 0x00]


def test_f16_decode_all_patterns_match_numpy():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.f16_to_double(bits)
    ref = bits.view(np.float16).astype(np.float64)
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    fin = ~np.isnan(ref)
    assert np.array_equal(ours[fin], ref[fin])


def test_bf16_decode_all_patterns_match_torch():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.bf16_to_double(bits)
    ref = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    fin = ~np.isnan(ref)
    assert np.array_equal(ours[fin], ref[fin])
