"""Test-side helpers: read the GPU's buffers back into the oracle's logical
layout, move seeded inputs to the device, and the parity tolerances.

Nothing here computes NVFP4 arithmetic; the mapping functions are pinned in
tests/test_layout_helpers.py against a brute-force reading of the layout
stated in include/nvfp4.h.
"""
from __future__ import annotations

import os

import numpy as np
import torch

import workloads

# NVFP4_TEST_LAUNCH_OVERLAP=1 runs the whole suite with launch overlap on;
# tests that switch it restore this default.
LAUNCH_OVERLAP_DEFAULT = os.environ.get("NVFP4_TEST_LAUNCH_OVERLAP") == "1"


# ------------------------------------------------------------------ layouts
def sf_logical(buf: np.ndarray, rows: int, K: int) -> np.ndarray:
    """Atom-layout scale bytes -> logical [rows, K/16] (row r, block j)."""
    kb = K // 16
    r = np.arange(rows)[:, None]
    j = np.arange(kb)[None, :]
    off = ((r // 128) * (kb // 4) + j // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + j % 4
    return np.asarray(buf, np.uint8)[off]


def sf_padding_rows(buf: np.ndarray, rows: int, K: int) -> np.ndarray:
    """Scale bytes of the padding rows [rows, ceil128(rows)) (must all be 0)."""
    padded = (rows + 127) // 128 * 128
    if padded == rows:
        return np.zeros((0,), np.uint8)
    kb = K // 16
    r = np.arange(rows, padded)[:, None]
    j = np.arange(kb)[None, :]
    off = ((r // 128) * (kb // 4) + j // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + j % 4
    return np.asarray(buf, np.uint8)[off]


def unpack_codes(packed: np.ndarray) -> np.ndarray:
    """[R, K/2] bytes -> [R, K] codes (low nibble = even element)."""
    p = np.asarray(packed, np.uint8)
    out = np.empty((p.shape[0], p.shape[1] * 2), np.uint8)
    out[:, 0::2] = p & 0xF
    out[:, 1::2] = p >> 4
    return out


# ------------------------------------------------------------ device moves
def bf16_dev(bits: np.ndarray, device="cuda", ld: int | None = None) -> torch.Tensor:
    """bf16 bit patterns (uint16 numpy) -> bf16 CUDA tensor, optionally with a wider row stride."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    if ld is not None and ld != bits.shape[1]:
        big = torch.zeros((bits.shape[0], ld), dtype=torch.bfloat16)
        big[:, :bits.shape[1]] = t
        return big.to(device)[:, :bits.shape[1]]
    return t.to(device)


def f32(bits: np.ndarray) -> np.ndarray:
    return workloads.bf16_bits_to_f32(bits)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """float -> nearest bf16 value (as float32), ties to even."""
    return workloads.bf16_bits_to_f32(workloads.f32_to_bf16_bits(np.asarray(x, np.float32)))


# --------------------------------------------------------------- tolerances
def check_gemm_fp32(y: np.ndarray, ref: np.ndarray, what: str = ""):
    """The stated GEMM bar: max |y - ref| <= 1e-3 rms(ref), rel. Frobenius <= 1e-5."""
    y = np.asarray(y, np.float64)
    ref = np.asarray(ref, np.float64)
    rms = np.sqrt(np.mean(ref ** 2))
    err = np.abs(y - ref)
    fro = np.linalg.norm(y - ref) / max(np.linalg.norm(ref), 1e-300)
    assert np.all(np.isfinite(y)), f"{what}: non-finite outputs"
    assert err.max() <= 1e-3 * rms, f"{what}: max err {err.max():.3e} > 1e-3 rms {rms:.3e}"
    assert fro <= 1e-5, f"{what}: rel Frobenius {fro:.3e} > 1e-5"
    return float(err.max() / rms), float(fro)


def check_bf16_out(y_bf16: np.ndarray, y_fp32: np.ndarray, ref: np.ndarray, what: str = ""):
    """bf16 output = bf16_RNE(fp32 epilogue value) exactly, and within half a bf16
    ulp of the reference plus the fp32 bar."""
    yb = np.asarray(y_bf16, np.float32)
    np.testing.assert_array_equal(yb, bf16_round(y_fp32), err_msg=f"{what}: bf16 != RNE(fp32)")
    ref = np.asarray(ref, np.float64)
    rms = np.sqrt(np.mean(ref ** 2))
    bound = np.abs(ref) * 2.0 ** -8 + 1e-3 * rms
    assert np.all(np.abs(yb - ref) <= bound), f"{what}: bf16 output outside bound"
