"""Pins for the oracle's block quantiser (CPU only).

* hand-derived blocks (tests/golden/quant_blocks.txt);
* exact round trip of inputs already on the NVFP4 grid;
* outlier locality: one outlier changes only its own 16-element block's scale
  byte and 16 codes (the pages' first mechanism: bayesiansapien wiki "The
  four-part mechanism study" part 1; aimodeling "Why the recurrent half
  survives");
* zero blocks, saturation under a static global scale, nibble packing.
"""
import os

import ml_dtypes
import numpy as np

import oracle
import workloads

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _golden_blocks():
    gs, blocks = None, []
    with open(os.path.join(GOLD, "quant_blocks.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            if line.startswith("gs "):
                gs = np.float32(float(line.split()[1]))
                continue
            head, vals = line.split("|")
            name, sc, codes = head.split()
            x = np.array([float(t) for t in vals.split()], np.float32)
            blocks.append((name, int(sc, 16), [int(ch, 16) for ch in codes], x))
    return gs, blocks


def test_golden_blocks():
    gs, blocks = _golden_blocks()
    for name, sc, codes, x in blocks:
        assert len(x) == 16 and len(codes) == 16
        q, s = oracle.quantize(x[None, :], gs)
        assert int(s[0, 0]) == sc, (name, hex(int(s[0, 0])), hex(sc))
        assert list(q[0]) == codes, (name, list(q[0]), codes)


def test_round_trip_on_grid():
    """x = e2m1 * s * gs with a +-6 in every block reproduces codes and scales exactly."""
    rng = np.random.default_rng(7)
    gs = np.float32(2.0 ** -6)
    R, K = 64, 512
    codes = rng.integers(0, 16, size=(R, K)).astype(np.uint8)
    codes[:, ::16] = rng.choice([7, 15], size=(R, K // 16))        # one |q| = 6 per block
    scales = rng.integers(1, 127, size=(R, K // 16)).astype(np.uint8)  # any finite non-zero E4M3
    # values from the independent library's decoders
    vals = codes.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    sdec = np.repeat(scales.view(ml_dtypes.float8_e4m3fn).astype(np.float64), 16, axis=1)
    x = (vals * sdec * float(gs)).astype(np.float32)
    assert np.all(workloads.bf16_bits_to_f32(workloads.f32_to_bf16_bits(x)) == x)  # bf16-exact
    q, s = oracle.quantize(x, gs)
    np.testing.assert_array_equal(s, scales)
    # -0 and +0 both decode to zero; compare values, then the sign of non-zeros
    np.testing.assert_array_equal(oracle.e2m1_decode(q), vals)
    nz = (codes & 7) != 0
    np.testing.assert_array_equal(q[nz], codes[nz])
    xhat = oracle.dequantize(q, s, gs)
    np.testing.assert_array_equal(xhat, x.astype(np.float64))


def test_outlier_changes_only_its_block():
    rng = np.random.default_rng(3)
    R, K = 32, 1024
    x = workloads.bf16_bits_to_f32(workloads.f32_to_bf16_bits(rng.standard_normal((R, K)).astype(np.float32)))
    gs = oracle.global_scale(np.float32(np.abs(x).max() * 200))    # fixed gs, leaves headroom
    q0, s0 = oracle.quantize(x, gs)
    for factor in (50.0, 100.0):
        for _ in range(20):
            r, c = int(rng.integers(R)), int(rng.integers(K))
            x1 = x.copy()
            blk = x[r, (c // 16) * 16:(c // 16) * 16 + 16]
            x1[r, c] = np.float32(np.abs(blk).max() * factor)   # an outlier of its block
            q1, s1 = oracle.quantize(x1, gs)
            ds = np.argwhere(s1 != s0)
            dq = np.argwhere(q1 != q0)
            assert all((a, b) == (r, c // 16) for a, b in ds)
            assert all(a == r and b // 16 == c // 16 for a, b in dq)
            assert len(ds) == 1        # the block's scale does move


def test_zero_block_gives_zero_codes():
    x = np.zeros((3, 64), np.float32)
    x[1, 20] = -0.0
    q, s = oracle.quantize(x, np.float32(0.01))
    assert np.all(q == 0) and np.all(s == 0)


def test_static_scale_saturates():
    gs = oracle.global_scale(np.float32(10.0))
    x = np.zeros((1, 16), np.float32)
    x[0, :4] = [1e4, -1e4, 5e3, 1.0]
    q, s = oracle.quantize(x, gs)
    assert s[0, 0] == 0x7E
    assert list(q[0, :3]) == [7, 15, 7]


def test_pack_codes_low_nibble_first():
    codes = np.array([[1, 2, 3, 4, 15, 0]], np.uint8)
    packed = oracle.pack_codes(codes)
    assert list(packed[0]) == [0x21, 0x43, 0x0F]


def test_workload_calibration_scales():
    """Global scales of the tiny workload are finite, positive and from fp32(amax)/2688."""
    w = workloads.WORKLOADS[1]
    xc = workloads.bf16_bits_to_f32(workloads.activations(w, calib=True))
    gs = oracle.global_scale(np.abs(xc).max())
    assert np.isfinite(gs) and gs > 0
    assert gs == np.float32(np.float32(np.abs(xc).max()) / np.float32(2688.0))


def test_global_scale_by_a_power_of_two_leaves_the_values_unchanged():
    """A global scale 4x larger quarters every block scale exactly (E4M3 is a
    binary float format) and leaves the block reciprocal, hence every code and
    every dequantised value, unchanged -- as long as no block scale leaves the
    normal E4M3 range.  So the global scale sets only the block scales' range:
    one shared scale for all modules of a fused weight (the pages' pre-
    harmonised checkpoint: aimodeling, "What engineers should actually take
    away") costs no precision beyond where a block scale rounds."""
    rng = np.random.default_rng(11)
    x = rng.normal(0, 1, (64, 256)).astype(np.float32)
    gs = oracle.global_scale(np.abs(x).max())
    q1, s1 = oracle.quantize(x, gs)
    q4, s4 = oracle.quantize(x, np.float32(gs * 4))
    d1, d4 = oracle.e4m3_decode(s1), oracle.e4m3_decode(s4)
    assert d1.min() / 4 >= 2.0 ** -6                  # quartered scales stay normal E4M3
    np.testing.assert_array_equal(d4 * 4, d1)
    np.testing.assert_array_equal(q4, q1)
    np.testing.assert_array_equal(oracle.dequantize(q4, s4, np.float32(gs * 4)),
                                  oracle.dequantize(q1, s1, gs))


def test_shared_global_scale_across_modules_costs_no_precision():
    """Modules with the GDN in-projection's spread of weight stds (log-uniform
    over 0.25..4 of 1/sqrt(K)), each quantised under its own global scale or
    under the largest one: the relative errors agree within 2%."""
    rng = np.random.default_rng(12)
    K = 512
    stds = np.array([0.25, 0.5, 1.0, 2.0, 4.0]) / np.sqrt(K)
    mods = [rng.normal(0, s, (64, K)).astype(np.float32) for s in stds]
    gs_shared = oracle.global_scale(max(np.abs(m).max() for m in mods))
    for m in mods:
        gs = oracle.global_scale(np.abs(m).max())
        own = np.linalg.norm(oracle.dequantize(*oracle.quantize(m, gs), gs) - m)
        shared = np.linalg.norm(oracle.dequantize(*oracle.quantize(m, gs_shared), gs_shared) - m)
        assert abs(shared / own - 1.0) < 0.02
