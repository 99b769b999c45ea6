"""Pins for the oracle's number-format conversions (CPU only).

The E2M1 and E4M3 conversions are checked against two independent
implementations (ml_dtypes, torch) and against hand tables in tests/golden.
The pages (bayesiansapien wiki "The four-part mechanism study"; nefut
abstract) name NVFP4 with 16-element block scales; the rounding rules are the
oracle's readings R1 and R2.
"""
import os

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _table(name):
    rows = []
    with open(os.path.join(GOLD, name)) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                parts = line.split()
                rows.append((float(parts[0]), int(parts[1], 16)))
    return rows


def _ref_e2m1(v):
    return np.asarray(v, np.float32).astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF


def test_e2m1_hand_table():
    for v, code in _table("e2m1_ties.txt"):
        got = int(oracle.e2m1_encode(np.float32(v)))
        assert got == code, (v, got, code)


def test_e2m1_decode_all_codes():
    codes = np.arange(16, dtype=np.uint8)
    ref = codes.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    np.testing.assert_array_equal(oracle.e2m1_decode(codes), ref)


@pytest.mark.parametrize("exp", range(-4, 4))
def test_e2m1_exhaustive_binade(exp):
    """Every float32 in [2^exp, 2^(exp+1)) and its negative: 2 x 2^23 values per binade."""
    mant = np.arange(1 << 23, dtype=np.uint32)
    bits = ((exp + 127) << 23) | mant
    v = bits.view(np.float32)
    for s in (v, -v):
        np.testing.assert_array_equal(oracle.e2m1_encode(s), _ref_e2m1(s))


def test_e2m1_wide_random_and_specials():
    rng = np.random.default_rng(1)
    bits = rng.integers(0, 1 << 32, size=2_000_000, dtype=np.uint64).astype(np.uint32)
    v = bits.view(np.float32)
    v = v[np.isfinite(v)]
    specials = np.array([0.0, -0.0, 1e-45, -1e-45, 1e-38, 3.4e38, -3.4e38], np.float32)
    for s in (v, specials):
        np.testing.assert_array_equal(oracle.e2m1_encode(s), _ref_e2m1(s))


def test_e4m3_hand_table():
    for v, code in _table("e4m3_table.txt"):
        got = int(oracle.e4m3_encode(np.float32(v)))
        assert got == code, (v, hex(got), hex(code))


def test_e4m3_decode_all_codes():
    codes = np.arange(127, dtype=np.uint8)
    ref = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    np.testing.assert_array_equal(oracle.e4m3_decode(codes), ref)


def _e4m3_probe_values():
    """Every rounding decision of E4M3 on [2^-20, 2^9]: all top-8 mantissa bits x sticky patterns."""
    top = np.arange(256, dtype=np.uint32) << 15
    low = np.array([0, 1, 0x3FFF, 0x4000, 0x4001, 0x7FFF], dtype=np.uint32)
    mant = (top[:, None] | low[None, :]).ravel()
    out = []
    for e in range(-20, 9):
        out.append((((e + 127) << 23) | mant).view(np.float32))
    # two binades exhaustively: a subnormal-scale one and a normal one
    allm = np.arange(1 << 23, dtype=np.uint32)
    for e in (-8, 0):
        out.append((((e + 127) << 23) | allm).view(np.float32))
    out.append(np.array([0.0, 448.0, 447.99997, 464.0], np.float32))
    return np.concatenate(out)


def test_e4m3_vs_ml_dtypes():
    v = _e4m3_probe_values()
    c = np.minimum(v, np.float32(448.0))           # satfinite: clamp first
    ref = c.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    np.testing.assert_array_equal(oracle.e4m3_encode(v), ref)


def test_e4m3_vs_torch():
    v = _e4m3_probe_values()
    c = torch.from_numpy(np.minimum(v, np.float32(448.0)))
    ref = c.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(oracle.e4m3_encode(v), ref)


def test_e4m3_saturates_above_448():
    v = np.array([448.0, 449.0, 464.0, 465.0, 1e6, 3e38], np.float32)
    assert np.all(oracle.e4m3_encode(v) == 0x7E)


def test_global_scale_is_fp32_division():
    for amax in (1.0, 6.0, 2688.0, 123.456, 1e-3, 7.5e4):
        gs = oracle.global_scale(amax)
        assert gs.dtype == np.float32
        # correctly rounded: the exact quotient lies within half an ulp of gs
        exact = float(np.float32(amax)) / 2688.0
        ulp = float(np.spacing(gs))
        assert abs(float(gs) - exact) <= 0.5 * ulp
    assert oracle.global_scale(2688.0) == np.float32(1.0)


def test_global_scale_of_an_all_zero_tensor_is_one():
    """Reading R3: an all-zero tensor (amax = 0) gets gs = 1, not 0.  Any
    positive gs encodes zeros the same way; 0 would make the block-scale
    divisor 6 gs zero and the block reciprocal infinite.  The scale must be a
    usable one: positive, finite, and the zero tensor must quantise to zero
    codes and zero scales and dequantise to exact zeros."""
    gs = oracle.global_scale(0.0)
    assert gs.dtype == np.float32 and gs == np.float32(1.0)
    assert oracle.global_scale(np.float32(-0.0)) == np.float32(1.0)
    x = np.zeros((3, 64), np.float32)
    with np.errstate(all="raise"):
        q, s = oracle.quantize(x, gs)
        xh = oracle.dequantize(q, s, gs)
    assert not q.any() and not s.any()
    assert np.array_equal(xh, np.zeros_like(xh))
    # the smallest positive amax already takes the division branch
    tiny = np.float32(np.finfo(np.float32).smallest_subnormal)
    assert oracle.global_scale(tiny) == np.float32(tiny / np.float32(2688.0))
