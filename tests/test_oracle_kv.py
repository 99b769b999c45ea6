"""Pins for the CPU oracle of the FP8 (E4M3) KV cache (no GPU).

kv_quantize is checked against an independent library conversion
(ml_dtypes.float8_e4m3fn, round to nearest even) on every finite bf16 value
under several per-tensor scales, with saturation and signed zeros by hand;
kv_scale against IEEE fp32 division; kv_dequantize as the exact inverse on
the grid.  The recipe is the pages' "ship calibrated FP8 KV-cache scales"
(nefut abstract; aimodeling, "What engineers should actually take away").
"""
import ml_dtypes
import numpy as np
import pytest

from oracle.kv import kv_dequantize, kv_quantize, kv_scale


def all_finite_bf16():
    bits = np.arange(1 << 16, dtype=np.uint32)
    f = (bits << 16).view(np.float32)
    return f[np.isfinite(f)]


@pytest.mark.parametrize("amax", [1.0, 448.0, 3.7, 1e-3, 6.5e4])
def test_every_bf16_value_matches_the_library_conversion(amax):
    x = all_finite_bf16()
    s = kv_scale(amax)
    codes = kv_quantize(x, s)
    with np.errstate(over="ignore"):
        v = (x * np.float32(np.float32(1) / s)).astype(np.float32)
    inside = np.abs(v) <= 448.0                         # the library gives NaN past the range
    lib = v[inside].astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    np.testing.assert_array_equal(codes[inside], lib)
    # saturation past the calibrated range (the largest finite magnitude, sign kept)
    big = ~inside
    np.testing.assert_array_equal(codes[big], np.where(v[big] < 0, 0xFE, 0x7E).astype(np.uint8))


def test_scale_is_an_fp32_division_by_448():
    for a in (1.0, 123.456, 6e4, 3.1e-3):
        assert kv_scale(a) == np.float32(np.float32(a) / np.float32(448.0))
    assert kv_scale(0.0) == np.float32(1.0)


def test_signed_zeros_and_the_calibrated_maximum():
    s = kv_scale(448.0)                                    # scale 1
    x = np.array([0.0, -0.0, 1e-30, -1e-30, 448.0, -448.0, 464.0, 1e6], np.float32)
    assert list(kv_quantize(x, s)) == [0x00, 0x80, 0x00, 0x80, 0x7E, 0xFE, 0x7E, 0x7E]


def test_dequantize_inverts_on_the_grid():
    """Every code's own value (times the scale) encodes back to the code."""
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)   # not NaN
    s = kv_scale(17.0)
    xh = kv_dequantize(codes, s).astype(np.float32)
    back = kv_quantize(xh, s)
    # +0 and -0 keep their sign; everything else is the same code
    np.testing.assert_array_equal(back, codes)


def test_relative_error_is_within_half_an_e4m3_step():
    rng = np.random.default_rng(0)
    x = rng.standard_normal(100000).astype(np.float32)
    s = kv_scale(np.abs(x).max())
    xh = kv_dequantize(kv_quantize(x, s), s)
    normal = np.abs(x) >= 2.0 ** -6 * s                    # above E4M3's subnormal range
    rel = np.abs(xh[normal] - x[normal]) / np.abs(x[normal])
    assert rel.max() <= 2.0 ** -4 * (1 + 1e-6)            # 3 mantissa bits: half step = 2^-4
