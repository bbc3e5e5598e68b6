"""Pins for the oracle's E4M3 encode/decode (CPU only).

The oracle's E4M3 conversion is checked against things other than itself: the closed-form
special values of the format (tests/golden/e4m3_special_values.txt), torch's own
float8_e4m3fn conversion (a library routine), and a brute-force nearest-value search.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e4m3_special_values.txt")


def _golden():
    out = []
    for line in open(GOLDEN):
        line = line.split("#")[0].strip()
        if line:
            c, v = line.split()
            out.append((int(c, 16), float(v)))
    return out


def _finite_table():
    """All finite E4M3 values, decoded by torch (independent of the oracle)."""
    codes = np.arange(256, dtype=np.uint8)
    vals = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    return codes, vals


@pytest.mark.parametrize("code,value", _golden())
def test_special_values(code, value):
    got = oracle.e4m3_decode(code)
    if math.isnan(value):
        assert math.isnan(got)
    else:
        assert got == value and math.copysign(1, got) == math.copysign(1, value)


def test_decode_all_codes_match_torch():
    codes, ref = _finite_table()
    got = np.array([oracle.e4m3_decode(c) for c in codes])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    m = ~np.isnan(ref)
    assert np.array_equal(got[m], ref[m])
    assert np.isnan(got).sum() == 2          # only S.1111.111


def test_encode_decode_round_trip_every_finite_code():
    codes, ref = _finite_table()
    for c, v in zip(codes, ref):
        if not np.isnan(v):
            assert oracle.e4m3_encode(np.float32(v)) == c, hex(c)


def _brute_force_encode(v: float) -> int:
    """Nearest finite E4M3 value by exhaustive search; ties to the even mantissa; saturating."""
    codes, vals = _finite_table()
    if math.isnan(v):
        return 0x7F | (0x80 if math.copysign(1, v) < 0 else 0)
    sign = 0x80 if math.copysign(1, v) < 0 else 0
    a = min(abs(v), 448.0)
    pos = [(c, x) for c, x in zip(codes, vals) if c < 0x80 and not np.isnan(x)]
    best = min(pos, key=lambda cx: (abs(cx[1] - a), cx[0] & 1))
    return int(best[0]) | sign


def test_encode_matches_brute_force_random():
    rng = np.random.default_rng(7)
    xs = np.concatenate([
        rng.standard_normal(3000) * 10.0 ** rng.uniform(-4, 3, 3000),
        rng.uniform(-500, 500, 500),
    ]).astype(np.float32)
    for v in xs:
        assert oracle.e4m3_encode(v) == _brute_force_encode(float(v)), float(v)


def test_encode_matches_torch_cast_in_range():
    rng = np.random.default_rng(8)
    x = (rng.standard_normal(200000) * 60).astype(np.float32)
    x = x[np.abs(x) < 448]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = oracle.e4m3_encode_array(x)
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("v,code", [
    (1.0625, 0x38),      # halfway 1.0 | 1.125  -> even mantissa (1.0)
    (1.1875, 0x3A),      # halfway 1.125 | 1.25 -> even mantissa (1.25)
    (0.0009765625, 0x00),  # halfway 0 | 2^-9 -> 0
    (0.0029296875, 0x02),  # halfway 2^-9 | 2*2^-9 -> even (2)
    (464.0, 0x7E),       # beyond the largest finite: saturates
    (1e30, 0x7E),
    (-1e30, 0xFE),
    (float("inf"), 0x7E),
    (-0.0, 0x80),
    (-1e-9, 0x80),       # rounds to zero, keeps the sign
])
def test_encode_closed_form_cases(v, code):
    assert oracle.e4m3_encode(np.float32(v)) == code


def test_nan_encodes_to_nan():
    c = oracle.e4m3_encode(np.float32("nan"))
    assert c & 0x7F == 0x7F
