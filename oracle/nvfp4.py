"""NVFP4 W4A4 linear layer, written out as plainly as possible (CPU, numpy).

TEST INFRASTRUCTURE ONLY (see the package docstring).

Source: the paper "Why Gated DeltaNet Survives 4-Bit Quantization: NVFP4 W4A4
for the Recurrent Half of a Hybrid 27B LLM", as summarised on five web pages.
What the pages fix:
  * every linear layer is NVFP4 W4A4: 4-bit weights AND 4-bit activations
    (nefut abstract, "Minima: NVFP4 W4A4, quantizing all 496 linear layers");
  * NVFP4 scales every 16 consecutive elements with one block scale, which
    confines an outlier to its own block (bayesiansapien wiki, "The four-part
    mechanism study", part 1; aimodeling news, "Why the recurrent half
    survives");
  * fused serving kernels that merge several per-module-calibrated projections
    into one GEMM mis-scale the per-module global scales; the repair applies
    each module's own scale (wiki, "Two practical repairs"; aimodeling,
    "What engineers should actually take away");
  * the GDN gates are a sigmoid (write strength) and a softplus/exponential
    (decay) parameterisation (wiki, mechanism study part 2).
What the pages leave open, and the reading taken here (plainest one consistent
with them):
  R1 value grid: E2M1 magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6}, sign bit on top;
     conversion rounds to nearest, ties to the even code, saturates at 6, and
     keeps the sign of results that round to zero.
  R2 block scale: unsigned E4M3 (bias 7, max 448, subnormals down to 2^-9),
     s = E4M3_RNE_satfinite(fp32(amax_block / fp32(6 * gs))).
  R3 global scale: gs = fp32(amax) / fp32(448 * 6), one per tensor (per module
     for weights), computed once from a calibration batch for activations;
     a tensor whose amax is 0 gets gs = 1 (any positive gs quantises it to
     all-zero codes and scales, and 0 would divide by zero).
  R4 element code: q = E2M1(fp32(x * r)) with r = fp32(1 / fp32(s_dec * gs)),
     using the DECODED (rounded) block scale; an all-zero scale gives code 0.
  R5 dequantised value: e2m1(q) * s_dec * gs, exact in float64.
  R6 GEMM: y = Xhat @ What^T in float64; each fused module uses its own
     weight global scale (this IS the repaired result).
  R7 gates: beta = 1 / (1 + exp(-y)); g = -exp(A_log[h]) * softplus(y + dt_bias[h]),
     h = column - module offset, softplus(z) = max(z, 0) + log1p(exp(-|z|)).
Quantizer steps run in float32 (the precision the kernel decides codes in,
since the pages fix none); everything after dequantisation is float64.
"""
from __future__ import annotations

import numpy as np

F32 = np.float32

# R1: the E2M1 grid, indexed by the 3-bit magnitude code.
E2M1_VALUES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)
# Midpoints between neighbouring grid values, and the code a tie resolves to
# (the even one of the two neighbours).
_E2M1_MID = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], dtype=np.float32)
_E2M1_TIE_CODE = np.array([0, 2, 2, 4, 4, 6, 6], dtype=np.uint8)

E2M1_MAX = 6.0
E4M3_MAX = 448.0
GS_DIVISOR = F32(448.0 * 6.0)   # 2688, exact in float32


# ---------------------------------------------------------------- E2M1 (R1)
def e2m1_encode(v) -> np.ndarray:
    """float32 -> 4-bit E2M1 code (uint8 in 0..15), RNE, saturating at 6.

    Code = sign << 3 | magnitude index.  For each midpoint m_i between grid
    values g_i and g_{i+1}: |v| > m_i moves past it; |v| == m_i resolves to the
    even code of the pair.
    """
    v = np.asarray(v, dtype=np.float32)
    a = np.abs(v)
    mag = np.zeros(v.shape, dtype=np.uint8)
    for i in range(len(_E2M1_MID)):
        above = a > _E2M1_MID[i]
        tie = a == _E2M1_MID[i]
        mag = np.where(above, np.uint8(i + 1), mag)
        mag = np.where(tie, _E2M1_TIE_CODE[i], mag)
    sign = np.signbit(v).astype(np.uint8)
    return (sign << 3) | mag


def e2m1_decode(code) -> np.ndarray:
    code = np.asarray(code, dtype=np.uint8)
    mag = E2M1_VALUES[code & 7]
    return np.where(code & 8, -mag, mag)


# ---------------------------------------------------------------- E4M3 (R2)
def e4m3_decode(code) -> np.ndarray:
    """Unsigned E4M3 (fn) code -> float64 value. Exponent bias 7; field 0 is subnormal."""
    code = np.asarray(code, dtype=np.int64)
    e = (code >> 3) & 0xF
    m = code & 7
    normal = np.ldexp(1.0 + m / 8.0, (e - 7).astype(np.int64))
    sub = np.ldexp(m / 8.0, -6)
    return np.where(e == 0, sub, normal)


_E4M3_CODES = np.arange(0, 127, dtype=np.int64)        # 0x00..0x7E: all finite, non-negative
_E4M3_TABLE = e4m3_decode(_E4M3_CODES)                  # strictly increasing


def e4m3_encode(t) -> np.ndarray:
    """Non-negative float32 -> E4M3 code, round to nearest even, saturating at 448.

    The value is clamped to 448, then rounded on the E4M3 grid: the grid step
    at binade 2^E (E >= -6) is 2^(E-3); below 2^-6 the step is 2^-9.  The
    rounded value is looked up in the table of all 127 finite codes.
    """
    t = np.minimum(np.asarray(t, dtype=np.float64), E4M3_MAX)
    if np.any(t < 0) or np.any(~np.isfinite(t)):
        raise ValueError("e4m3_encode expects finite non-negative input")
    _, ex = np.frexp(t)                                  # t = f * 2^ex, f in [0.5, 1)
    E = np.maximum(ex - 1, -6)
    step = np.ldexp(1.0, (E - 3).astype(np.int64))
    r = np.rint(t / step) * step                         # np.rint: ties to even
    idx = np.searchsorted(_E4M3_TABLE, r)
    if not np.all(_E4M3_TABLE[np.minimum(idx, 126)] == r):
        raise AssertionError("rounded value not on the E4M3 grid")
    return idx.astype(np.uint8)


# ------------------------------------------------------------ global scale (R3)
def global_scale(amax) -> np.float32:
    """gs = fp32(amax) / fp32(2688); 1 for an all-zero tensor (reading R3)."""
    if F32(amax) == 0:
        return F32(1.0)
    return F32(F32(amax) / GS_DIVISOR)


# ------------------------------------------------------------- quantize (R2, R4)
def quantize(x, gs, block: int = 16):
    """Quantise rows of x (float32 values, here bf16 inputs) under global scale gs.

    Returns (codes uint8 [R, K] one code per element, scales uint8 [R, K/16]
    E4M3 codes, in logical order: scales[r, j] covers x[r, 16j:16j+16]).
    Steps per 16-element block b of a row:
      amax_b = max |x| (exact)
      c      = fp32(6 * gs)
      s      = E4M3(fp32(amax_b / c))
      s_dec  = decoded s
      if s_dec == 0: all codes 0
      else  p = fp32(s_dec * gs); r = fp32(1 / p); q_k = E2M1(fp32(x_k * r))
    """
    x = np.asarray(x, dtype=np.float32)
    R, K = x.shape
    if K % block:
        raise ValueError("K must be a multiple of the block size")
    gs = F32(gs)
    xb = x.reshape(R, K // block, block)
    amax_b = np.max(np.abs(xb), axis=2)                         # float32, exact
    c = F32(F32(6.0) * gs)
    s = e4m3_encode(np.divide(amax_b, c, dtype=np.float32))
    s_dec = e4m3_decode(s).astype(np.float32)                   # exact in float32
    p = np.multiply(s_dec, gs, dtype=np.float32)
    with np.errstate(divide="ignore"):
        r = np.divide(F32(1.0), p, dtype=np.float32)
    r = np.where(s_dec == 0, F32(0.0), r).astype(np.float32)
    y = np.multiply(xb, r[:, :, None], dtype=np.float32)
    q = e2m1_encode(y)
    q = np.where((s_dec == 0)[:, :, None], np.uint8(0), q)
    return q.reshape(R, K).astype(np.uint8), s.astype(np.uint8)


def pack_codes(codes) -> np.ndarray:
    """[R, K] codes -> [R, K/2] bytes; element 2i in the low nibble, 2i+1 in the high."""
    codes = np.asarray(codes, dtype=np.uint8)
    return (codes[:, 0::2] & 0xF) | ((codes[:, 1::2] & 0xF) << 4)


# ------------------------------------------------------------- dequantize (R5)
def dequantize(codes, scales, gs, block: int = 16) -> np.ndarray:
    """float64 xhat[r, k] = e2m1(codes[r, k]) * s_dec[r, k // 16] * gs (exact)."""
    vals = e2m1_decode(codes)
    sd = np.repeat(e4m3_decode(scales), block, axis=1)
    return vals * sd * float(F32(gs))


# ---------------------------------------------------------------- GEMM (R6)
def linear64(xhat, what) -> np.ndarray:
    """y = xhat @ what^T in float64 (both operands K-major: [M, K] and [N, K])."""
    return np.asarray(xhat, np.float64) @ np.asarray(what, np.float64).T


def sigmoid64(y) -> np.ndarray:
    """beta = 1 / (1 + exp(-y)), evaluated without overflow."""
    y = np.asarray(y, dtype=np.float64)
    e = np.exp(-np.abs(y))
    return np.where(y >= 0, 1.0 / (1.0 + e), e / (1.0 + e))


def gdn_decay64(y, a_log, dt_bias) -> np.ndarray:
    """g = -exp(A_log) * softplus(y + dt_bias), per column head (R7)."""
    z = np.asarray(y, dtype=np.float64) + np.asarray(dt_bias, dtype=np.float64)
    softplus = np.maximum(z, 0.0) + np.log1p(np.exp(-np.abs(z)))
    return -np.exp(np.asarray(a_log, dtype=np.float64)) * softplus


def fused_linear64(x_codes, x_scales, w_codes, w_scales, segments) -> np.ndarray:
    """Fused multi-module projection with each module's own global scales.

    segments: list of dicts {n_offset, width, w_gs, a_gs, op, a_log, dt_bias};
    op in {"none", "sigmoid", "gdn_decay"}.  Columns [n_offset, n_offset+width)
    of y come from the module's weight rows, dequantised with that module's
    w_gs and the activation dequantised with that module's a_gs.
    """
    M = x_codes.shape[0]
    N = sum(s["width"] for s in segments)
    y = np.empty((M, N), dtype=np.float64)
    for s in segments:
        n0, n1 = s["n_offset"], s["n_offset"] + s["width"]
        xhat = dequantize(x_codes, x_scales, s["a_gs"])
        what = dequantize(w_codes[n0:n1], w_scales[n0:n1], s["w_gs"])
        ys = linear64(xhat, what)
        op = s.get("op", "none")
        if op == "sigmoid":
            ys = sigmoid64(ys)
        elif op == "gdn_decay":
            ys = gdn_decay64(ys, np.asarray(s["a_log"])[None, :], np.asarray(s["dt_bias"])[None, :])
        elif op != "none":
            raise ValueError(op)
        y[:, n0:n1] = ys
    return y


def fused_linear64_shared_scale(x_codes, x_scales, w_codes, w_scales, segments) -> np.ndarray:
    """The mis-scaled fused GEMM the pages describe: one global scale for all modules.

    A fused kernel that ignores per-module calibration applies the first
    module's (a_gs, w_gs) to every column.  Used only to show the repair.
    """
    shared = [dict(s, w_gs=segments[0]["w_gs"], a_gs=segments[0]["a_gs"], op="none")
              for s in segments]
    return fused_linear64(x_codes, x_scales, w_codes, w_scales, shared)


# ------------------------------------------------- MLP pair glue (workload 4)
def _bf16_rne(x32) -> np.ndarray:
    """float32 values -> nearest bf16 values (ties to even), as float32."""
    u = np.asarray(x32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return u.astype(np.uint32).view(np.float32)


def silu_mul_bf16(gate, up) -> np.ndarray:
    """h = bf16_RNE(fp32(silu(g) * u)) with g = bf16(fp32(gate)), u = bf16(fp32(up)).

    Reading R8: the gate_up projection is itself a W4A4 linear layer and, like
    every layer here, emits bf16, so SiLU(gate) * up reads bf16 gate and up
    values (each the RNE bf16 of the fp32 value); the product is evaluated in
    float64, rounded to fp32 and then to bf16, which is the down projection's
    activation input.  Returns float32 values.
    """
    g = _bf16_rne(np.asarray(gate, dtype=np.float64).astype(np.float32)).astype(np.float64)
    u = _bf16_rne(np.asarray(up, dtype=np.float64).astype(np.float32)).astype(np.float64)
    return _bf16_rne((g * sigmoid64(g) * u).astype(np.float32))
