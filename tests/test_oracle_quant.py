"""Pins for the oracle's dynamic activation quantization (CPU only).

Recipe 0 ("metrale ... fp8_grouped_tc_w8a8.rs", module doc: E4M3 per (row, 128 group)) and
recipe 1 ("DeepGEMM PR #371", Changes: UE8M0 power-of-two scale per 32 elements).  The pins
are closed forms (the group maximum maps to 448; values on the grid round-trip), an exact
brute-force search for the power-of-two exponent, and the rounding bound.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle


def _dec(codes):
    return np.array([oracle.e4m3_decode(c) for c in np.asarray(codes).ravel()])


def test_recipe0_group_max_maps_to_448():
    rng = np.random.default_rng(1)
    x = rng.standard_normal(1024).astype(np.float32)
    q, s = oracle.quant_row(x, 0)
    assert s.shape == (8,) and s.dtype == np.float32
    for g in range(8):
        blk = x[128 * g:128 * (g + 1)]
        i = int(np.argmax(np.abs(blk)))
        assert s[g] == np.float32(np.abs(blk).max()) / np.float32(448.0)
        assert q[128 * g + i] == (0xFE if blk[i] < 0 else 0x7E)


def test_recipe0_grid_values_round_trip():
    rng = np.random.default_rng(2)
    s = np.float32(0.0390625)          # 1.25 * 2^-5: 448*s and v*s are exact in fp32
    finite = [c for c in range(0x7F) if c != 0x7F]
    codes = rng.choice(finite, 128).astype(np.uint8)
    codes[5] = 0x7E                    # make 448 the group maximum
    signs = rng.integers(0, 2, 128).astype(np.uint8) << 7
    codes = codes | signs
    x = (_dec(codes) * float(s)).astype(np.float32)
    q, sc = oracle.quant_row(x, 0)
    assert sc[0] == s
    nz = _dec(codes) != 0
    assert np.array_equal(q[nz], codes[nz])


def test_zero_group_gives_unit_scale_and_zero_codes():
    q, s = oracle.quant_row(np.zeros(256, np.float32), 0)
    assert np.all(s == 1.0) and np.all(q == 0)
    q, s = oracle.quant_row(np.zeros(64, np.float32), 1)
    assert np.all(s == 127) and np.all(q == 0)


def _brute_mx_exponent(amax: float) -> int:
    """Smallest integer e with amax <= 448 * 2^e, by exact rational search."""
    a = Fraction(float(amax))
    e = -127
    while e < 127 and a > Fraction(448) * Fraction(2) ** e:
        e += 1
    return e


@pytest.mark.parametrize("amax,e", [(448.0, 0), (449.0, 1), (224.0, -1), (224.5, 0),
                                    (1.0, -8), (896.0, 1), (1e-45, -127)])
def test_mx_exponent_closed_form(amax, e):
    assert oracle.mx_exponent(np.float32(amax)) == e


def test_mx_exponent_matches_exact_search():
    rng = np.random.default_rng(3)
    vals = (10.0 ** rng.uniform(-30, 30, 400)).astype(np.float32)
    edges = np.array([448.0 * 2.0 ** k for k in range(-20, 20)], np.float32)
    vals = np.concatenate([vals, edges, np.nextafter(edges, np.float32(np.inf))])
    for v in vals:
        assert oracle.mx_exponent(v) == _brute_mx_exponent(float(v)), float(v)


def test_mx_never_saturates_and_bounds_error():
    rng = np.random.default_rng(4)
    x = (rng.standard_normal(4096) * 10.0 ** rng.uniform(-3, 3, 4096)).astype(np.float32)
    q, b = oracle.quant_row(x, 1)
    assert b.dtype == np.uint8 and b.shape == (128,)
    deq = _dec(q).reshape(128, 32) * np.exp2(b.astype(np.float64) - 127)[:, None]
    assert np.all(np.abs(_dec(q)) <= 448)
    xs = x.reshape(128, 32).astype(np.float64)
    # Round to nearest with 3 mantissa bits: error <= 2^-4 of the value for normals, or half the
    # subnormal step 2^-10 * scale.
    scale = np.exp2(b.astype(np.float64) - 127)[:, None]
    bound = np.maximum(np.abs(xs) * 2.0 ** -4, 2.0 ** -10 * scale)
    assert np.all(np.abs(deq - xs) <= bound * (1 + 1e-12))


def test_recipe0_error_bound():
    rng = np.random.default_rng(5)
    x = rng.standard_normal(2048).astype(np.float32)
    q, s = oracle.quant_row(x, 0)
    deq = _dec(q).reshape(16, 128) * s.astype(np.float64)[:, None]
    xs = x.reshape(16, 128).astype(np.float64)
    s64 = s.astype(np.float64)[:, None]
    # x/s is rounded once to fp32 before the E4M3 rounding; allow that relative 2^-24.
    bound = np.maximum(np.abs(xs) * 2.0 ** -4, 2.0 ** -10 * s64) + np.abs(xs) * 2.0 ** -23
    assert np.all(np.abs(deq - xs) <= bound)


def test_quantize_tokens_matches_row_quantizer():
    rng = np.random.default_rng(6)
    import torch
    xb = torch.from_numpy(rng.standard_normal((5, 384)).astype(np.float32)).to(torch.bfloat16)
    bits = xb.view(torch.int16).numpy().view(np.uint16)
    for recipe in (0, 1):
        q, s = oracle.quantize_tokens(bits, recipe)
        for t in range(5):
            q1, s1 = oracle.quant_row(xb[t].float().numpy(), recipe)
            assert np.array_equal(q[t], q1) and np.array_equal(s[t], s1)
