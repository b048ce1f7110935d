"""Pins of the oracle's format codecs against things other than the oracle.

* e4m3 decode of all 256 codes against torch's float8_e4m3fn (a library
  routine), and against a table derived here from the bit fields;
* e4m3 encode against a brute-force nearest-even search over the finite
  e4m3 values, over every bf16 bit pattern and a million random float32
  values, and against torch's float -> float8_e4m3fn cast inside the finite
  range;
* e5m2 decode of all 256 codes and encode of every bf16 pattern, random
  float32 values and tie midpoints, against the bit fields, a brute-force
  nearest-even search and torch's float8_e5m2;
* e2m1 decode/encode against the bit-field definition and a brute-force
  search; page-independent tie cases from tests/golden;
* UE8M0 against a brute-force smallest power of two;
* bf16 rounding against torch's float32 -> bfloat16 cast.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _e4m3_from_fields(code: int) -> float:
    s = -1.0 if code & 0x80 else 1.0
    e, m = (code >> 3) & 0xF, code & 7
    if e == 15 and m == 7:
        return math.nan
    if e == 0:
        return s * m * 2.0 ** -9
    return s * (1 + m / 8) * 2.0 ** (e - 7)


def _e2m1_from_fields(code: int) -> float:
    s = -1.0 if code & 0x8 else 1.0
    e, m = (code >> 1) & 3, code & 1
    if e == 0:
        return s * m * 0.5
    return s * (1 + m / 2) * 2.0 ** (e - 1)


def _brute_nearest_even(v: np.ndarray, mags: np.ndarray, sign_bit: int, max_code: int) -> np.ndarray:
    """Nearest non-negative magnitude code (ties to the even code), saturating, sign from v."""
    a = np.abs(v.astype(np.float64))
    dist = np.abs(a[:, None] - mags[None, :])
    best = dist.min(axis=1, keepdims=True)
    cand = dist == best
    codes = np.arange(len(mags))
    # among tied candidates prefer an even code
    even = cand & (codes[None, :] % 2 == 0)
    pick = np.where(even.any(axis=1), even.argmax(axis=1), cand.argmax(axis=1))
    pick = np.where(a >= mags[max_code], max_code, pick)
    sign = (np.signbit(v)).astype(np.uint8) * sign_bit
    return (pick.astype(np.uint8) | sign).astype(np.uint8)


E4M3_MAGS = np.array([_e4m3_from_fields(c) for c in range(0x7F)], np.float64)  # 0x00..0x7E
E2M1_MAGS = np.array([_e2m1_from_fields(c) for c in range(8)], np.float64)


def test_e4m3_decode_matches_bitfields_and_torch():
    codes = np.arange(256, dtype=np.uint8)
    dec = oracle.e4m3_decode(codes).astype(np.float64)
    ref = np.array([_e4m3_from_fields(int(c)) for c in codes])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(dec), nan)
    assert np.array_equal(dec[~nan], ref[~nan])
    tdec = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(tdec), nan)
    assert np.array_equal(dec[~nan], tdec[~nan])
    assert dec[0x7E] == 448.0 and dec[0xFE] == -448.0 and dec[0x01] == 2.0 ** -9
    assert nan[0x7F] and nan[0xFF] and nan.sum() == 2


def test_e4m3_encode_all_bf16_patterns_brute_force():
    bits = np.arange(65536, dtype=np.uint32)
    v = (bits << 16).view(np.float32)
    v = v[~np.isnan(v)]
    got = oracle.e4m3_encode(v)
    exp = _brute_nearest_even(v, E4M3_MAGS, 0x80, 0x7E)
    assert np.array_equal(got, exp)


def test_e4m3_encode_random_f32_brute_force_and_torch():
    rng = np.random.default_rng(1234)
    n = 1_000_000
    # log-uniform magnitudes over the whole e4m3 range and beyond, random signs
    mag = np.exp2(rng.uniform(-12, 10, n)).astype(np.float32)
    v = np.where(rng.random(n) < 0.5, -mag, mag).astype(np.float32)
    # exact midpoints between neighbouring codes (tie cases) with random signs
    mids = ((E4M3_MAGS[1:] + E4M3_MAGS[:-1]) / 2).astype(np.float32)
    v = np.concatenate([v, mids, -mids])
    got = oracle.e4m3_encode(v)
    exp = np.concatenate([_brute_nearest_even(c, E4M3_MAGS, 0x80, 0x7E)
                          for c in np.array_split(v, 20)])
    assert np.array_equal(got, exp)
    inside = np.abs(v) <= 448.0
    t = torch.from_numpy(v[inside]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got[inside], t)


def test_e4m3_golden_points():
    cases = json.load(open(os.path.join(GOLDEN, "e4m3_points.json")))["cases"]
    x = np.array([c["x"] for c in cases], np.float32)
    exp = np.array([c["code"] for c in cases], np.uint8)
    assert np.array_equal(oracle.e4m3_encode(x), exp), [c["why"] for c in cases]


def test_e4m3_saturates_and_nan():
    v = np.array([np.inf, -np.inf, 3e38, -500.0], np.float32)
    assert list(oracle.e4m3_encode(v)) == [0x7E, 0xFE, 0x7E, 0xFE]
    assert oracle.e4m3_encode(np.array([np.nan], np.float32))[0] & 0x7F == 0x7F


def test_e2m1_decode_and_encode():
    codes = np.arange(16, dtype=np.uint8)
    dec = oracle.e2m1_decode(codes).astype(np.float64)
    ref = np.array([_e2m1_from_fields(int(c)) for c in codes])
    assert np.array_equal(dec, ref)
    assert np.array_equal(np.signbit(dec), np.signbit(ref))
    rng = np.random.default_rng(7)
    v = rng.uniform(-8, 8, 200_000).astype(np.float32)
    mids = ((E2M1_MAGS[1:] + E2M1_MAGS[:-1]) / 2).astype(np.float32)
    v = np.concatenate([v, mids, -mids, E2M1_MAGS.astype(np.float32)])
    assert np.array_equal(oracle.e2m1_encode(v), _brute_nearest_even(v, E2M1_MAGS, 0x8, 7))


def test_e2m1_golden_points():
    cases = json.load(open(os.path.join(GOLDEN, "e2m1_points.json")))["cases"]
    x = np.array([c["x"] for c in cases], np.float32)
    exp = np.array([c["code"] for c in cases], np.uint8)
    assert np.array_equal(oracle.e2m1_encode(x), exp)


def _brute_pow2_ceil(s: float) -> float:
    if not s > 0:
        return 2.0 ** -127
    p = -149
    while 2.0 ** p < s:
        p += 1
    return 2.0 ** min(max(p, -127), 127)


def test_ue8m0_brute_force():
    rng = np.random.default_rng(3)
    s = np.concatenate([
        np.exp2(rng.uniform(-140, 120, 3000)),
        np.exp2(np.arange(-130, 128, dtype=np.float64)),          # exact powers of two
        np.exp2(np.arange(-130, 127, dtype=np.float64)) * 1.0000001,
        [0.0, 1.0 / 448, 1e-45, 2.0 ** -126, 3.4e38],
    ]).astype(np.float32)
    got = oracle.ue8m0_ceil(s)
    exp = np.array([_brute_pow2_ceil(float(x)) for x in s], np.float32)
    assert np.array_equal(got, exp)


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(11)
    v = np.concatenate([
        rng.standard_normal(500_000).astype(np.float32) * np.float32(1000),
        (np.arange(0, 1 << 20, dtype=np.uint32) * 4093).view(np.float32),
    ])
    v = v[~np.isnan(v)]
    got = oracle.bf16_from_f32(v)
    exp = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, exp)


def _e5m2_from_fields(code: int) -> float:
    s = -1.0 if code & 0x80 else 1.0
    e, m = (code >> 2) & 0x1F, code & 3
    if e == 31:
        return math.nan if m else s * math.inf
    if e == 0:
        return s * m * 2.0 ** -16
    return s * (1 + m / 4) * 2.0 ** (e - 15)


E5M2_MAGS = np.array([_e5m2_from_fields(c) for c in range(0x7C)], np.float64)  # 0x00..0x7B finite


def test_e5m2_decode_matches_bitfields_and_torch():
    codes = np.arange(256, dtype=np.uint8)
    dec = oracle.e5m2_decode(codes).astype(np.float64)
    ref = np.array([_e5m2_from_fields(int(c)) for c in codes])
    tdec = torch.from_numpy(codes).view(torch.float8_e5m2).to(torch.float64).numpy()
    for a in (ref, tdec):
        nan = np.isnan(a)
        assert np.array_equal(np.isnan(dec), nan)
        assert np.array_equal(dec[~nan], a[~nan])
    assert dec[0x7B] == 57344.0 and dec[0x01] == 2.0 ** -16 and dec[0x7C] == np.inf


def test_e5m2_encode_brute_force_and_torch():
    bits = np.arange(65536, dtype=np.uint32)
    v = (bits << 16).view(np.float32)
    v = v[~np.isnan(v)]
    rng = np.random.default_rng(9)
    mag = np.exp2(rng.uniform(-20, 18, 300_000)).astype(np.float32)
    mids = ((E5M2_MAGS[1:] + E5M2_MAGS[:-1]) / 2).astype(np.float32)
    v = np.concatenate([v, mag, -mag, mids, -mids])
    got = oracle.e5m2_encode(v)
    exp = np.concatenate([_brute_nearest_even(c, E5M2_MAGS, 0x80, 0x7B) for c in np.array_split(v, 40)])
    assert np.array_equal(got, exp)
    inside = np.abs(v) <= 57344.0
    t = torch.from_numpy(v[inside]).to(torch.float8_e5m2).view(torch.uint8).numpy()
    assert np.array_equal(got[inside], t)
