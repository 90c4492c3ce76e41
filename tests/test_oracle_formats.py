"""Pins for the oracle's number formats (E2M1, E4M3, E8M0, MX scale, bf16).

Each encoder is checked against values the format specifications fix
(tests/golden/*.txt), against round-to-nearest-even at every midpoint, and
against an independent implementation (ml_dtypes / torch casts)."""
import math
import os

import ml_dtypes
import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    rows = []
    for line in open(os.path.join(GOLDEN, name)):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        c, v = line.split()
        rows.append((int(c, 16), float(v)))
    return rows


def test_e2m1_all_codes_match_spec(ora):
    rows = _read_golden("e2m1_codes.txt")
    assert len(rows) == 16
    for code, val in rows:
        got = ora.e2m1_value(code)
        assert got == val and math.copysign(1, got) == math.copysign(1, val), (code, got, val)
        # every code is its own encoding (including -0 -> 0x8)
        assert ora.e2m1_encode(val) == code


def test_e2m1_round_half_even_midpoints(ora):
    # midpoint -> expected code (the even one of the two neighbours)
    mids = {0.25: 0x0, 0.75: 0x2, 1.25: 0x2, 1.75: 0x4, 2.5: 0x4, 3.5: 0x6, 5.0: 0x6}
    for m, code in mids.items():
        assert ora.e2m1_encode(m) == code, m
        assert ora.e2m1_encode(-m) == code | 8, -m
        up, dn = np.nextafter(np.float32(m), np.float32(10)), np.nextafter(np.float32(m), np.float32(0))
        assert ora.e2m1_value(ora.e2m1_encode(float(up))) > m
        assert ora.e2m1_value(ora.e2m1_encode(float(dn))) < m


def test_e2m1_saturates_and_keeps_sign(ora):
    for x in [6.0, 6.5, 7.0, 100.0, 1e30]:
        assert ora.e2m1_encode(x) == 7
        assert ora.e2m1_encode(-x) == 0xF
    assert ora.e2m1_encode(-1e-30) == 0x8
    assert ora.e2m1_encode(1e-30) == 0x0


def test_e2m1_matches_ml_dtypes_sweep(ora):
    """Independent encoder: ml_dtypes.float4_e2m1fn (RNE, saturating)."""
    rng = np.random.default_rng(0)
    xs = np.concatenate([
        rng.uniform(-8, 8, 20000).astype(np.float32),
        np.linspace(-7, 7, 20001, dtype=np.float32),
        (rng.standard_normal(5000) * 1e-3).astype(np.float32),
    ])
    ref = xs.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    got = np.array([ora.e2m1_encode(float(x)) for x in xs], np.uint8)
    assert np.array_equal(got, ref)


def test_e4m3_named_points(ora):
    for code, val in _read_golden("e4m3_points.txt"):
        got = ora.e4m3_value(code)
        if math.isnan(val):
            assert math.isnan(got)
        else:
            assert got == val, (code, got, val)


def test_e4m3_all_256_codes_match_torch(ora):
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        got = ora.e4m3_value(c)
        if math.isnan(ref[c]):
            assert math.isnan(got), c
        else:
            assert got == ref[c], (c, got, ref[c])


def test_e4m3_encode_rne_and_saturation(ora):
    # code round trip
    for c in range(0x7F):
        assert ora.e4m3_encode(ora.e4m3_value(c)) == c
    # every midpoint between neighbouring codes goes to the even code
    for c in range(0x7E):
        mid = (ora.e4m3_value(c) + ora.e4m3_value(c + 1)) / 2
        assert ora.e4m3_encode(mid) == (c if c % 2 == 0 else c + 1), c
    # saturation (satfinite): >= 448 -> 448
    for u in [448.0, 449.0, 464.0, 500.0, 1e10]:
        assert ora.e4m3_encode(u) == 0x7E
    # underflow: below half the smallest subnormal -> 0
    assert ora.e4m3_encode(2.0 ** -10) == 0
    assert ora.e4m3_encode(2.0 ** -10 * 1.0001) == 1


def test_e4m3_encode_matches_torch_sweep(ora):
    rng = np.random.default_rng(1)
    u = np.concatenate([rng.uniform(0, 448, 20000), np.exp(rng.uniform(-12, 6, 20000))]).astype(np.float32)
    u = u[u < 448]
    ref = torch.from_numpy(u).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([ora.e4m3_encode(float(x)) for x in u], np.uint8)
    assert np.array_equal(got, ref)


def test_e8m0_points_and_all_codes(ora):
    for code, val in _read_golden("e8m0_points.txt"):
        got = ora.e8m0_value(code)
        assert (math.isnan(got) and math.isnan(val)) or got == val
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e8m0fnu).to(torch.float64).numpy()
    for c in range(255):
        assert ora.e8m0_value(c) == ref[c]


def test_mx_scale_rule(ora):
    # OCP MX v1.0: X = 2^(floor(log2 amax) - emax_elem), emax_elem = 2 for E2M1
    for e in range(-100, 100):
        for f in [1.0, 1.5, 1.999]:
            amax = f * 2.0 ** e
            code = ora.mx_scale_code(amax)
            assert code == e - 2 + 127
            assert 4.0 <= amax / ora.e8m0_value(code) < 8.0
    assert ora.mx_scale_code(0.0) == 0
    assert ora.mx_scale_code(2.0 ** 200) == 254
    assert ora.mx_scale_code(2.0 ** -200) == 0


def test_bf16_rounding_matches_ml_dtypes(ora):
    rng = np.random.default_rng(2)
    xs = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-30, 30, 20000),
                         rng.standard_normal(2000)]).astype(np.float32)
    ref = xs.astype(ml_dtypes.bfloat16).view(np.uint16)
    got = np.array([ora.f64_to_bf16(float(x)) for x in xs], np.uint16)
    assert np.array_equal(got, ref)
    # ties to even on exact midpoints
    assert ora.f64_to_bf16(1.0 + 2.0 ** -8) == 0x3F80
    assert ora.f64_to_bf16(1.0 + 3 * 2.0 ** -8) == 0x3F82
