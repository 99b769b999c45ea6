"""Pins for the oracle's GEMM, fused segments and gates (CPU only).

* float64 GEMM on dequantised operands vs exact rational brute force, with
  operand values taken from ml_dtypes (independent of the oracle's decoders);
* every E2M1 x E2M1 product, and every pair of positive E4M3 scales, is exact;
* the global-scale mismatch of fused kernels (bayesiansapien wiki, "Two
  practical repairs"; aimodeling "What engineers should actually take away"):
  without the repair module s comes out scaled by exactly
  (a_gs_0 w_gs_0) / (a_gs_s w_gs_s);
* gate contraction (wiki mechanism study part 2): |dbeta| <= |dy| / 4 and
  |dg| <= exp(A_log) |dy|, plus closed values and limits.
"""
from fractions import Fraction

import ml_dtypes
import numpy as np
import pytest

import oracle


def _rand_quant(rng, R, K):
    codes = rng.integers(0, 16, size=(R, K)).astype(np.uint8)
    scales = rng.integers(0, 127, size=(R, K // 16)).astype(np.uint8)
    return codes, scales


def _exact_value(code, scale, gs):
    v = Fraction(float(np.uint8(code).view(ml_dtypes.float4_e2m1fn)))
    s = Fraction(float(np.uint8(scale).view(ml_dtypes.float8_e4m3fn)))
    return v * s * Fraction(float(gs))


def test_linear64_matches_exact_bruteforce():
    rng = np.random.default_rng(11)
    M, N, K = 3, 5, 48
    xa, xs = _rand_quant(rng, M, K)
    wa, ws = _rand_quant(rng, N, K)
    agsv, wgsv = np.float32(0.0123), np.float32(0.000731)
    y = oracle.linear64(oracle.dequantize(xa, xs, agsv), oracle.dequantize(wa, ws, wgsv))
    assert y.shape == (M, N)
    for m in range(M):
        for n in range(N):
            exact = sum(_exact_value(xa[m, k], xs[m, k // 16], agsv) *
                        _exact_value(wa[n, k], ws[n, k // 16], wgsv) for k in range(K))
            # every product is exact in float64; the sum of 48 terms rounds at most
            # K times, each by <= 2^-53 of the running magnitude
            bound = 48 * 2.0 ** -52 * float(sum(abs(_exact_value(xa[m, k], xs[m, k // 16], agsv) *
                                                    _exact_value(wa[n, k], ws[n, k // 16], wgsv))
                                                for k in range(K)))
            assert abs(y[m, n] - float(exact)) <= bound


def test_all_e2m1_pairs_exact():
    """Single non-zero k: y = e2m1(a) * e2m1(b) * s_a * s_b * gs_a * gs_b, exact."""
    K = 64
    for ca in range(16):
        for cb in range(16):
            xa = np.zeros((1, K), np.uint8)
            wa = np.zeros((1, K), np.uint8)
            xa[0, 37], wa[0, 37] = ca, cb
            xs = np.full((1, K // 16), 0x38, np.uint8)    # 1.0
            ws = np.full((1, K // 16), 0x41, np.uint8)    # 2.25
            y = oracle.linear64(oracle.dequantize(xa, xs, 0.5), oracle.dequantize(wa, ws, 0.25))
            ref = (float(np.uint8(ca).view(ml_dtypes.float4_e2m1fn)) *
                   float(np.uint8(cb).view(ml_dtypes.float4_e2m1fn)) * 2.25 * 0.5 * 0.25)
            assert y[0, 0] == ref


def test_all_e4m3_scale_pairs_exact_in_fp32():
    s = np.arange(1, 127, dtype=np.uint8)
    v = oracle.e4m3_decode(s)
    prod = np.outer(v, v)
    assert np.all(prod.astype(np.float32).astype(np.float64) == prod)


def test_block_index_mapping():
    """Scale j applies to elements 16j..16j+15 only (a transposed or shifted block index fails)."""
    K = 64
    codes = np.full((1, K), 2, np.uint8)                 # value 1.0 everywhere
    scales = np.array([[0x38, 0x40, 0x48, 0x50]], np.uint8)   # 1, 2, 4, 8
    xhat = oracle.dequantize(codes, scales, 1.0)
    np.testing.assert_array_equal(xhat[0], np.repeat([1.0, 2.0, 4.0, 8.0], 16))


def _segments(rng, widths, ops=None):
    segs, off = [], 0
    for i, w in enumerate(widths):
        segs.append(dict(n_offset=off, width=w, w_gs=np.float32(rng.uniform(1e-4, 1e-2)),
                         a_gs=np.float32(0.01), op=(ops[i] if ops else "none"),
                         a_log=rng.uniform(-1, 1.5, w).astype(np.float32),
                         dt_bias=rng.normal(0, 0.5, w).astype(np.float32)))
        off += w
    return segs


def test_mismatch_ratio_is_closed_form():
    rng = np.random.default_rng(5)
    M, K = 4, 64
    widths = [32, 16, 48]
    xa, xs = _rand_quant(rng, M, K)
    wa, ws = _rand_quant(rng, sum(widths), K)
    segs = _segments(rng, widths)
    y = oracle.fused_linear64(xa, xs, wa, ws, segs)
    ybug = oracle.fused_linear64_shared_scale(xa, xs, wa, ws, segs)
    for s in segs:
        sl = slice(s["n_offset"], s["n_offset"] + s["width"])
        ratio = (float(segs[0]["a_gs"]) * float(segs[0]["w_gs"])) / (float(s["a_gs"]) * float(s["w_gs"]))
        # float64 sums of differently scaled terms round differently: bound by the magnitude
        tol = 1e-13 * np.abs(y[:, sl] * ratio).max()
        np.testing.assert_allclose(ybug[:, sl], y[:, sl] * ratio, rtol=1e-13, atol=tol)
        # and a wrong ratio (e.g. the repair applied twice) is far outside that
        assert np.abs(ybug[:, sl] - y[:, sl]).max() > 1e3 * tol or abs(ratio - 1) < 1e-12


def test_fused_equals_independent_per_module_products():
    rng = np.random.default_rng(6)
    M, K = 3, 32
    widths = [16, 16]
    xa, xs = _rand_quant(rng, M, K)
    wa, ws = _rand_quant(rng, 32, K)
    segs = _segments(rng, widths)
    y = oracle.fused_linear64(xa, xs, wa, ws, segs)
    for s in segs:
        for m in range(M):
            for j in range(s["width"]):
                n = s["n_offset"] + j
                exact = sum(_exact_value(xa[m, k], xs[m, k // 16], s["a_gs"]) *
                            _exact_value(wa[n, k], ws[n, k // 16], s["w_gs"]) for k in range(K))
                assert abs(y[m, n] - float(exact)) <= 1e-12 * (abs(float(exact)) + 1e-30)


def test_sigmoid_closed_values_and_bound():
    assert oracle.sigmoid64(0.0) == 0.5
    assert abs(oracle.sigmoid64(np.log(3.0)) - 0.75) < 1e-15
    assert oracle.sigmoid64(-800.0) == 0.0 and oracle.sigmoid64(800.0) == 1.0
    rng = np.random.default_rng(2)
    y1 = rng.normal(0, 4, 100000)
    y2 = y1 + rng.normal(0, 0.3, y1.shape)
    assert np.all(np.abs(oracle.sigmoid64(y1) - oracle.sigmoid64(y2)) <= 0.25 * np.abs(y1 - y2) + 1e-15)


def test_gdn_decay_closed_values_limits_and_bound():
    A = np.array([-1.0, 0.0, 0.7, 1.5])
    dt = np.array([0.3, -0.2, 0.0, 0.5])
    # z = y + dt = 0 -> softplus = ln 2
    np.testing.assert_allclose(oracle.gdn_decay64(-dt, A, dt), -np.exp(A) * np.log(2.0), rtol=1e-15)
    # large z: softplus(z) -> z
    np.testing.assert_allclose(oracle.gdn_decay64(50.0, A, dt), -np.exp(A) * (50.0 + dt), rtol=1e-15)
    # very negative z: g -> 0 from below
    g = oracle.gdn_decay64(-60.0, A, dt)
    assert np.all(g < 0) and np.all(g > -1e-20)
    rng = np.random.default_rng(4)
    for a, d in zip(A, dt):
        y1 = rng.normal(0, 4, 100000)
        y2 = y1 + rng.normal(0, 0.3, y1.shape)
        dg = np.abs(oracle.gdn_decay64(y1, a, d) - oracle.gdn_decay64(y2, a, d))
        assert np.all(dg <= np.exp(a) * np.abs(y1 - y2) * (1 + 1e-12) + 1e-15)


@pytest.mark.parametrize("op", ["sigmoid", "gdn_decay"])
def test_gates_contract_relative_error(op):
    """Gate outputs carry a smaller relative error than their pre-activations.

    The pages report ~11% GEMM error shrinking to ~2% after the gates on real
    activations; on synthetic pre-activations the ratio must at least be < 1.
    """
    rng = np.random.default_rng(9)
    y = rng.normal(0, 2.0, 200000)
    y_noisy = y * (1 + rng.normal(0, 0.11, y.shape))
    if op == "sigmoid":
        out, out_n = oracle.sigmoid64(y), oracle.sigmoid64(y_noisy)
    else:
        out, out_n = oracle.gdn_decay64(y, 0.5, 0.2), oracle.gdn_decay64(y_noisy, 0.5, 0.2)
    rel_in = np.linalg.norm(y_noisy - y) / np.linalg.norm(y)
    rel_out = np.linalg.norm(out_n - out) / np.linalg.norm(out)
    assert rel_out < rel_in


# ------------------------------------------------- MLP glue (SiLU(gate) * up)
def test_silu_mul_bf16_rounding_matches_ml_dtypes():
    """The bf16 rounding steps against an independent RNE: ml_dtypes' bfloat16
    casts of the float32 gate / up inputs and of the float32 products (random,
    ties at every exponent, and values whose low 16 bits are exactly 0x8000)."""
    rng = np.random.default_rng(21)
    g = rng.standard_normal(20000) * 4
    u = rng.standard_normal(20000) * 3
    h = oracle.silu_mul_bf16(g, u)
    gb = g.astype(np.float32).astype(ml_dtypes.bfloat16).astype(np.float64)
    ub = u.astype(np.float32).astype(ml_dtypes.bfloat16).astype(np.float64)
    prod32 = (gb * (1.0 / (1.0 + np.exp(-gb))) * ub).astype(np.float32)
    want = prod32.astype(ml_dtypes.bfloat16).astype(np.float32)
    # the oracle's product is float64 rounded once to float32, as here; allow
    # the rare case where the two float64 evaluations land on different float32s
    diff = h != want
    assert diff.mean() < 1e-3
    ulp = np.abs(want[diff]) * 2.0 ** -7
    assert np.all(np.abs(h[diff] - want[diff]) <= ulp)
    # exact ties: silu(48) = 48 exactly in float64 (sigmoid(48) rounds to 1),
    # and 48 * (1 + k/128) for odd k (u exact in bf16) has nine significant
    # bits: a float32 value halfway between two bf16 values, rounded to even
    k = np.array([1, 3, 5, 7, 9, 17, -1, -33], np.float64)
    up = 1.0 + k / 128.0
    prod = (48.0 * up).astype(np.float32)
    assert np.all((prod.view(np.uint32) & 0xFFFF) == 0x8000)
    got = oracle.silu_mul_bf16(np.full(len(k), 48.0), up)
    np.testing.assert_array_equal(got, prod.astype(ml_dtypes.bfloat16).astype(np.float32))


def test_silu_mul_bf16_reads_bf16_gate_and_up():
    """Reading R8: gate and up are the gate_up layer's bf16 outputs, so the
    oracle rounds them to bf16 before SiLU * up: inputs that round to the same
    bf16 values give the same h, and h differs from the product of the
    unrounded values where the rounding of the inputs moves it."""
    one_plus = np.float64(1.0 + 2.0 ** -10)          # not a bf16 value: rounds to 1
    assert oracle.silu_mul_bf16(np.array([one_plus]), np.array([1.0]))[0] == \
        oracle.silu_mul_bf16(np.array([1.0]), np.array([1.0]))[0]
    rng = np.random.default_rng(5)
    g = rng.standard_normal(4096) * 3
    u = rng.standard_normal(4096) * 2
    gb = g.astype(np.float32).astype(ml_dtypes.bfloat16).astype(np.float64)
    ub = u.astype(np.float32).astype(ml_dtypes.bfloat16).astype(np.float64)
    np.testing.assert_array_equal(oracle.silu_mul_bf16(g, u), oracle.silu_mul_bf16(gb, ub))
    unrounded = (g / (1.0 + np.exp(-g)) * u).astype(np.float32).astype(ml_dtypes.bfloat16)
    assert np.mean(oracle.silu_mul_bf16(g, u) != unrounded.astype(np.float32)) > 0.05


def test_silu_mul_bf16_closed_values_and_limits():
    up = np.array([3.0, -2.0, 0.5], np.float64)
    # silu(0) = 0
    np.testing.assert_array_equal(oracle.silu_mul_bf16(np.zeros(3), up), np.zeros(3, np.float32))
    # silu(g) -> g for large g, -> 0 for very negative g
    big = oracle.silu_mul_bf16(np.full(3, 40.0), up)
    np.testing.assert_allclose(big, (40.0 * up).astype(np.float32), rtol=2.0 ** -8)
    neg = oracle.silu_mul_bf16(np.full(3, -60.0), up)
    assert np.all(np.abs(neg) < 1e-20)
    # silu(1) * 1 = 1 / (1 + e^-1), to bf16 precision
    one = oracle.silu_mul_bf16(np.array([1.0]), np.array([1.0]))
    assert abs(float(one[0]) - 1.0 / (1.0 + np.exp(-1.0))) <= 2.0 ** -9
    # the output holds bf16 values only
    h = oracle.silu_mul_bf16(np.linspace(-8, 8, 999), np.linspace(3, -3, 999))
    assert np.all((h.view(np.uint32) & 0xFFFF) == 0)
