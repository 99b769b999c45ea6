"""CPU oracle for the FP8 KV cache -- TEST INFRASTRUCTURE ONLY.

The pages' second recommendation: ship calibrated FP8 KV-cache scales, which
cost no speed ("quantize everything, ship KV scales": nefut abstract;
bayesiansapien wiki, "Two practical repairs"; aimodeling, "What engineers
should actually take away").  They give no arithmetic; the readings here
follow the NVFP4 quantiser's (oracle.nvfp4):
  scale     = fp32(amax_calib) / fp32(448)  (one per tensor, from a
              calibration batch; 1 when amax is 0) -- 448 is the largest
              finite E4M3 value;
  r         = fp32(1 / scale)               (one reciprocal per tensor);
  code      = sign | E4M3_RNE_satfinite(|fp32(x * r)|)  (the sign bit is
              kept for values that round to zero; live values beyond the
              calibration range saturate at 448);
  x_hat     = e4m3(code) * scale            (exact in float64).

Pinning status: kv_quantize -- ml_dtypes.float8_e4m3fn on every finite bf16
input under several scales, saturation and signed zeros by hand; kv_scale --
IEEE fp32 division; kv_dequantize -- exact inverse on the grid.
"""
from __future__ import annotations

import numpy as np

from .nvfp4 import E4M3_MAX, e4m3_decode, e4m3_encode


def kv_scale(amax) -> np.float32:
    a = np.float32(amax)
    if not a > 0:
        return np.float32(1.0)
    return np.float32(a / np.float32(E4M3_MAX))


def kv_quantize(x, scale) -> np.ndarray:
    """float32-valued x (bf16 inputs), per-tensor scale -> signed E4M3 codes (uint8)."""
    x = np.asarray(x, dtype=np.float32)
    r = np.float32(np.float32(1.0) / np.float32(scale))
    with np.errstate(over="ignore"):                    # past fp32 range: saturates below
        v = (x * r).astype(np.float32)                  # one fp32 multiply, RN
    mag = e4m3_encode(np.abs(v).astype(np.float64))
    sign = np.signbit(v).astype(np.uint8) << 7
    return (mag | sign).astype(np.uint8)


def kv_dequantize(codes, scale) -> np.ndarray:
    codes = np.asarray(codes, dtype=np.uint8)
    val = e4m3_decode(codes & 0x7F)
    return np.where(codes & 0x80, -val, val) * np.float64(np.float32(scale))
