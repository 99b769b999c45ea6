"""GPU parity: conversions, amax, activation and weight quantisers vs the oracle.

Codes and block scales must match the oracle bit for bit (the conversions
decide integers, so both sides round in fp32 with the same steps).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
import nvfp4_w4a4_quantized_quantizer_b200 as nv
from tests import _helpers as H
from tests.test_oracle_formats import _e4m3_probe_values

pytestmark = pytest.mark.gpu


# ----------------------------------------------------------- conversions
@pytest.mark.parametrize("exp", [-3, -2, -1, 0, 1, 2])
def test_e2m1_conversion_exhaustive_binade(exp):
    mant = np.arange(1 << 23, dtype=np.uint32)
    v = (((exp + 127) << 23) | mant).view(np.float32)
    v = np.concatenate([v, -v])
    got = nv.nvfp4_test_e2m1(torch.from_numpy(v).cuda()).cpu().numpy()
    np.testing.assert_array_equal(got, oracle.e2m1_encode(v))


def test_e2m1_conversion_wide_random_and_specials():
    rng = np.random.default_rng(21)
    v = rng.integers(0, 1 << 32, size=4_000_000, dtype=np.uint64).astype(np.uint32).view(np.float32)
    v = v[np.isfinite(v)]
    v = np.concatenate([v, np.array([0.0, -0.0, 1e-45, -1e-45, 6.0, -6.0, 3e38], np.float32)])
    got = nv.nvfp4_test_e2m1(torch.from_numpy(v).cuda()).cpu().numpy()
    np.testing.assert_array_equal(got, oracle.e2m1_encode(v))


def test_e4m3_conversion_every_rounding_boundary():
    v = _e4m3_probe_values()
    got = nv.nvfp4_test_e4m3(torch.from_numpy(v).cuda()).cpu().numpy()
    np.testing.assert_array_equal(got, oracle.e4m3_encode(v))


# ------------------------------------------------------------------ amax
def test_amax_exact_with_stride():
    bits = workloads.random_bf16((300, 320), seed=3, std=5.0)
    x = H.bf16_dev(bits, ld=328)
    got = nv.nvfp4_amax(x).item()
    assert got == float(np.abs(H.f32(bits)).max())
    z = torch.zeros((17, 64), dtype=torch.bfloat16, device="cuda")
    assert nv.nvfp4_amax(z).item() == 0.0


# ------------------------------------------------------- activation quant
def _quant_and_check(bits, gs, ld=None):
    M, K = bits.shape
    x = H.bf16_dev(bits, ld=ld)
    code_bytes = M * K // 2
    sbytes = nv.nvfp4_scale_bytes(M, K)
    # canaries after both outputs
    cbuf = torch.full((code_bytes + 64,), 0xAB, dtype=torch.uint8, device="cuda")
    sbuf = torch.full((sbytes + 64,), 0xCD, dtype=torch.uint8, device="cuda")
    codes = cbuf[:code_bytes].view(M, K // 2)
    nv.nvfp4_quantize_act(x, float(gs), codes=codes, scales=sbuf[:sbytes])
    torch.cuda.synchronize()
    c = cbuf.cpu().numpy()
    s = sbuf.cpu().numpy()
    assert np.all(c[code_bytes:] == 0xAB) and np.all(s[sbytes:] == 0xCD), "wrote past the end"
    q_ref, s_ref = oracle.quantize(H.f32(bits), np.float32(gs))
    np.testing.assert_array_equal(H.unpack_codes(c[:code_bytes].reshape(M, K // 2)), q_ref)
    np.testing.assert_array_equal(H.sf_logical(s[:sbytes], M, K), s_ref)
    assert np.all(H.sf_padding_rows(s[:sbytes], M, K) == 0)
    return q_ref, s_ref


@pytest.mark.parametrize("M,K,ld", [(1, 64, None), (3, 192, None), (100, 320, 336),
                                    (129, 5120, None), (300, 576, 640), (64, 256, None),
                                    # a 64-element last segment; rows 16 (not 32) bytes apart
                                    # mod 32; more units than every warp's staging ring holds
                                    (70, 1088, 1096), (5, 2048, None), (3000, 5120, None)])
def test_quantize_act_matches_oracle(M, K, ld):
    bits = workloads.random_bf16((M, K), seed=M * 7 + K, std=3.0)
    gs = oracle.global_scale(np.abs(H.f32(bits)).max())
    _quant_and_check(bits, gs, ld)


def test_quantize_act_tiny_workload():
    w = workloads.WORKLOADS[1]
    calib = workloads.activations(w, calib=True)
    live = workloads.activations(w)
    a_gs_gpu = nv.nvfp4_global_scale(nv.nvfp4_amax(H.bf16_dev(calib)).item())
    a_gs = oracle.global_scale(np.abs(H.f32(calib)).max())
    assert np.float32(a_gs_gpu) == a_gs
    _quant_and_check(live, a_gs)


def test_quantize_act_saturation_zeros_and_negative_zero():
    bits = workloads.random_bf16((64, 256), seed=5)
    bits[3, :] = 0                           # all-zero row
    bits[4, 0:16] = 0x8000                   # -0.0 block
    bits[5, 17] = workloads.f32_to_bf16_bits(np.array([1e4], np.float32))[0]
    gs = oracle.global_scale(np.float32(4.0))  # static scale well below the live amax
    q, s = _quant_and_check(bits, gs)
    assert s[5, 1] == 0x7E


def test_outlier_changes_only_its_block_on_gpu():
    M, K = 32, 1024
    bits = workloads.random_bf16((M, K), seed=8)
    gs = np.float32(oracle.global_scale(np.abs(H.f32(bits)).max() * 200))
    c0, s0 = nv.nvfp4_quantize_act(H.bf16_dev(bits), float(gs))
    rng = np.random.default_rng(1)
    for factor in (50.0, 100.0):
        r, col = int(rng.integers(M)), int(rng.integers(K))
        b1 = bits.copy()
        blk = H.f32(bits)[r, col // 16 * 16: col // 16 * 16 + 16]
        b1[r, col] = workloads.f32_to_bf16_bits(np.array([np.abs(blk).max() * factor], np.float32))[0]
        c1, s1 = nv.nvfp4_quantize_act(H.bf16_dev(b1), float(gs))
        dq = np.argwhere(H.unpack_codes(c1.cpu().numpy()) != H.unpack_codes(c0.cpu().numpy()))
        ds = np.argwhere(H.sf_logical(s1.cpu().numpy(), M, K) != H.sf_logical(s0.cpu().numpy(), M, K))
        assert len(ds) == 1 and tuple(ds[0]) == (r, col // 16)
        assert all(a == r and b // 16 == col // 16 for a, b in dq)


def test_scale_layout_identity():
    """Block (m, j) is built so that its scale code is a known function of (m, j)."""
    M, K = 200, 320
    gs = np.float32(2.0 ** -6)
    want = (1 + (np.arange(M)[:, None] * 7 + np.arange(K // 16)[None, :] * 3) % 125).astype(np.uint8)
    x = np.zeros((M, K), np.float32)
    # amax = 6 gs s_dec  ->  amax / (6 gs) = s_dec exactly
    x[:, 0::16] = 6.0 * float(gs) * oracle.e4m3_decode(want)
    bits = workloads.f32_to_bf16_bits(x)
    assert np.all(H.f32(bits) == x)
    _, s = nv.nvfp4_quantize_act(H.bf16_dev(bits), float(gs))
    np.testing.assert_array_equal(H.sf_logical(s.cpu().numpy(), M, K), want)


# ----------------------------------------------------------- weight quant
def test_quantize_weight_segmented_matches_oracle():
    K = 320
    widths = [64, 64, 32, 16, 16, 16]
    offs = np.cumsum([0] + widths[:-1]).tolist()
    N = sum(widths)
    rng = np.random.default_rng(2)
    rows = []
    for i, wdt in enumerate(widths):
        std = float(np.exp(rng.uniform(np.log(0.25), np.log(4.0)))) / np.sqrt(K)
        rows.append(workloads.random_bf16((wdt, K), seed=40 + i, std=std))
    bits = np.concatenate(rows)
    codes, scales, gss = nv.nvfp4_quantize_weight(H.bf16_dev(bits), seg_offsets=offs)
    torch.cuda.synchronize()
    wf = H.f32(bits)
    sl = H.sf_logical(scales.cpu().numpy(), N, K)
    cu = H.unpack_codes(codes.cpu().numpy())
    for i, (o, wdt) in enumerate(zip(offs, widths)):
        gs = oracle.global_scale(np.abs(wf[o:o + wdt]).max())
        assert np.float32(gss[i]) == gs
        q, s = oracle.quantize(wf[o:o + wdt], gs)
        np.testing.assert_array_equal(cu[o:o + wdt], q)
        np.testing.assert_array_equal(sl[o:o + wdt], s)
    assert np.all(H.sf_padding_rows(scales.cpu().numpy(), N, K) == 0)
