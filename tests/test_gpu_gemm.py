"""GPU parity: block-scaled FP4 GEMM (every kernel) vs the float64 oracle.

Operands are either built directly in the device layout from random codes
and scales (so the GEMM is checked independently of the quantiser) or come
from the quantisers.  Bar: fp32 output within max |err| <= 1e-3 rms and
relative Frobenius <= 1e-5 of the float64 product of the dequantised
operands; bf16 output = bf16_RNE(fp32 output) exactly.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
import nvfp4_w4a4_quantized_quantizer_b200 as nv
from tests import _helpers as H

pytestmark = pytest.mark.gpu

LARGE, SMALL, AUTO, PAIR, PAIR_NFAST = 1, 2, 0, 3, 4


@pytest.fixture(autouse=True)
def _reset_path():
    yield
    nv.nvfp4_set_gemm_path(AUTO)


def sf_pack(logical: np.ndarray, rows: int, K: int) -> np.ndarray:
    """Logical [rows, K/16] scale codes -> atom-layout bytes (padding rows 0)."""
    padded = (rows + 127) // 128 * 128
    buf = np.zeros(padded * K // 16, np.uint8)
    kb = K // 16
    r = np.arange(rows)[:, None]
    j = np.arange(kb)[None, :]
    off = ((r // 128) * (kb // 4) + j // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + j % 4
    buf[off] = logical
    return buf


def pack(codes: np.ndarray) -> np.ndarray:
    return ((codes[:, 0::2] & 0xF) | ((codes[:, 1::2] & 0xF) << 4)).astype(np.uint8)


def dev_operands(codes, scales, rows, K):
    c = torch.from_numpy(pack(codes)).cuda()
    s = torch.from_numpy(sf_pack(scales, rows, K)).cuda()
    return c, s


def run(path, ac, as_, a_gs, wc, ws, w_gs, M, N, K):
    nv.nvfp4_set_gemm_path(path)
    y32 = nv.nvfp4_linear(ac, as_, a_gs, wc, ws, w_gs, M, N, K, out_dtype=nv.OUT_FP32)
    yb = nv.nvfp4_linear(ac, as_, a_gs, wc, ws, w_gs, M, N, K, out_dtype=nv.OUT_BF16)
    st, info = nv.nvfp4_last_device_error()
    assert st == 0, f"device error word {info:#x}"
    return y32.cpu().numpy(), yb.float().cpu().numpy()


@pytest.mark.parametrize("path,M", [(LARGE, 16), (SMALL, 16), (PAIR, 16), (PAIR_NFAST, 16)])
@pytest.mark.parametrize("p", [0, 1, 14, 15, 16, 31, 63, 64, 127, 128, 200, 255])
def test_all_code_pairs_single_k(path, M, p):
    """Row m holds code m, column n holds code n, both at k = p only; random scales."""
    K, N = 256, 16
    rng = np.random.default_rng(p)
    ac = np.zeros((M, K), np.uint8)
    wc = np.zeros((N, K), np.uint8)
    ac[:, p] = np.arange(16)
    wc[:, p] = np.arange(16)
    as_ = rng.integers(1, 127, size=(M, K // 16)).astype(np.uint8)
    ws = rng.integers(1, 127, size=(N, K // 16)).astype(np.uint8)
    a_gs, w_gs = np.float32(0.5), np.float32(0.25)
    y32, yb = run(path, *dev_operands(ac, as_, M, K), float(a_gs), *dev_operands(wc, ws, N, K),
                  float(w_gs), M, N, K)
    ref = oracle.linear64(oracle.dequantize(ac, as_, a_gs), oracle.dequantize(wc, ws, w_gs))
    # every product is exact; only the final alpha multiply rounds (half an fp32 ulp)
    assert np.all(np.abs(y32 - ref) <= np.abs(ref) * 2.0 ** -23)
    H.check_bf16_out(yb, y32, ref, "pairs")


@pytest.mark.parametrize("path,M,N,K", [
    (LARGE, 128, 256, 256), (LARGE, 256, 512, 512), (LARGE, 200, 272, 320),
    (LARGE, 129, 16, 64), (LARGE, 2048, 2560, 256), (LARGE, 300, 608, 1280),
    (SMALL, 1, 16, 64), (SMALL, 7, 128, 320), (SMALL, 16, 400, 1024), (SMALL, 17, 144, 256),
    (SMALL, 33, 272, 512), (SMALL, 64, 1040, 768),
    # CTA pairs: odd CTA's rows all past M (M <= 128), a ragged last tile
    # whose odd-CTA weight rows lie past N, several tiles per pair
    (PAIR, 100, 272, 320), (PAIR, 256, 256, 256), (PAIR, 300, 608, 1280),
    (PAIR, 129, 16, 64), (PAIR, 2048, 2560, 256), (PAIR, 2304, 5120, 512),
    # tiles walked N fastest (ragged M and N tiles, several tiles per pair)
    (PAIR_NFAST, 300, 608, 1280), (PAIR_NFAST, 2304, 5120, 512), (PAIR_NFAST, 129, 16, 64)])
def test_random_codes_and_scales(path, M, N, K):
    rng = np.random.default_rng(M * 131 + N * 7 + K)
    ac = rng.integers(0, 16, size=(M, K)).astype(np.uint8)
    wc = rng.integers(0, 16, size=(N, K)).astype(np.uint8)
    as_ = rng.integers(0x28, 0x58, size=(M, K // 16)).astype(np.uint8)   # 2^-2 .. 2^4
    ws = rng.integers(0x28, 0x58, size=(N, K // 16)).astype(np.uint8)
    a_gs, w_gs = np.float32(0.0173), np.float32(0.00291)
    y32, yb = run(path, *dev_operands(ac, as_, M, K), float(a_gs), *dev_operands(wc, ws, N, K),
                  float(w_gs), M, N, K)
    ref = oracle.linear64(oracle.dequantize(ac, as_, a_gs), oracle.dequantize(wc, ws, w_gs))
    H.check_gemm_fp32(y32, ref, f"random {M}x{N}x{K}")
    H.check_bf16_out(yb, y32, ref, f"random {M}x{N}x{K}")


def test_cancellation_heavy_accumulation():
    """Alternating large +-6 * 448 products with small ones: fp32 accumulation must hold 1e-5."""
    M, N, K = 128, 256, 5120
    rng = np.random.default_rng(77)
    ac = rng.integers(0, 16, size=(M, K)).astype(np.uint8)
    wc = rng.integers(0, 16, size=(N, K)).astype(np.uint8)
    ac[:, 0::64] = 7
    wc[:, 0::128] = 7
    wc[:, 64::128] = 15
    as_ = rng.integers(0x08, 0x7F, size=(M, K // 16)).astype(np.uint8)
    ws = rng.integers(0x08, 0x7F, size=(N, K // 16)).astype(np.uint8)
    for path in (LARGE, PAIR):
        y32, yb = run(path, *dev_operands(ac, as_, M, K), 1e-3, *dev_operands(wc, ws, N, K), 2e-3,
                      M, N, K)
        ref = oracle.linear64(oracle.dequantize(ac, as_, np.float32(1e-3)),
                              oracle.dequantize(wc, ws, np.float32(2e-3)))
        H.check_gemm_fp32(y32, ref, "cancellation")


@pytest.mark.parametrize("path,M,N,K", [(LARGE, 200, 272, 320), (LARGE, 512, 768, 1024),
                                        (PAIR, 200, 272, 320), (PAIR, 512, 768, 1024),
                                        (SMALL, 5, 144, 320), (SMALL, 64, 256, 5120),
                                        (AUTO, 64, 128, 256)])
def test_quantize_then_gemm(path, M, N, K):
    xb = workloads.random_bf16((M, K), seed=M + K, std=2.0)
    wb = workloads.random_bf16((N, K), seed=N + K + 1, std=1 / np.sqrt(K))
    xf, wf = H.f32(xb), H.f32(wb)
    a_gs = oracle.global_scale(np.abs(xf).max())
    ac, as_ = nv.nvfp4_quantize_act(H.bf16_dev(xb), float(a_gs))
    wc, ws, (w_gs,) = nv.nvfp4_quantize_weight(H.bf16_dev(wb))
    qx, sx = oracle.quantize(xf, a_gs)
    w_gs_ref = oracle.global_scale(np.abs(wf).max())
    assert np.float32(w_gs) == w_gs_ref
    qw, sw = oracle.quantize(wf, w_gs_ref)
    np.testing.assert_array_equal(H.unpack_codes(ac.cpu().numpy()), qx)
    np.testing.assert_array_equal(H.unpack_codes(wc.cpu().numpy()), qw)
    y32, yb = run(path, ac, as_, float(a_gs), wc, ws, float(w_gs), M, N, K)
    ref = oracle.linear64(oracle.dequantize(qx, sx, a_gs), oracle.dequantize(qw, sw, w_gs_ref))
    H.check_gemm_fp32(y32, ref, "quantize+gemm")
    H.check_bf16_out(yb, y32, ref, "quantize+gemm")


def test_tiny_workload_end_to_end():
    """The tiny configuration: calibrate, quantise, GEMM, bf16 output."""
    w = workloads.WORKLOADS[1]
    calib, live, wbits = workloads.activations(w, calib=True), workloads.activations(w), workloads.weights(w)
    a_gs = nv.nvfp4_global_scale(nv.nvfp4_amax(H.bf16_dev(calib)).item())
    assert np.float32(a_gs) == oracle.global_scale(np.abs(H.f32(calib)).max())
    ac, as_ = nv.nvfp4_quantize_act(H.bf16_dev(live), a_gs)
    wc, ws, (w_gs,) = nv.nvfp4_quantize_weight(H.bf16_dev(wbits))
    y = nv.nvfp4_linear(ac, as_, a_gs, wc, ws, w_gs, w.M, w.N, w.K)
    y32 = nv.nvfp4_linear(ac, as_, a_gs, wc, ws, w_gs, w.M, w.N, w.K, out_dtype=nv.OUT_FP32)
    qx, sx = oracle.quantize(H.f32(live), np.float32(a_gs))
    qw, sw = oracle.quantize(H.f32(wbits), np.float32(w_gs))
    ref = oracle.linear64(oracle.dequantize(qx, sx, a_gs), oracle.dequantize(qw, sw, w_gs))
    H.check_gemm_fp32(y32.cpu().numpy(), ref, "tiny")
    H.check_bf16_out(y.float().cpu().numpy(), y32.cpu().numpy(), ref, "tiny")


def test_output_row_stride_and_no_overwrite():
    """ldy > N: columns past N are never written (every kernel)."""
    M, N, K, ldy = 150, 144, 256, 160
    rng = np.random.default_rng(9)
    ac = rng.integers(0, 16, size=(M, K)).astype(np.uint8)
    wc = rng.integers(0, 16, size=(N, K)).astype(np.uint8)
    as_ = rng.integers(0x30, 0x40, size=(M, K // 16)).astype(np.uint8)
    ws = rng.integers(0x30, 0x40, size=(N, K // 16)).astype(np.uint8)
    A, W = dev_operands(ac, as_, M, K), dev_operands(wc, ws, N, K)
    ref = oracle.linear64(oracle.dequantize(ac, as_, np.float32(0.01)),
                          oracle.dequantize(wc, ws, np.float32(0.02)))
    for path, m in ((LARGE, M), (PAIR, M), (PAIR_NFAST, M), (SMALL, 40)):
        nv.nvfp4_set_gemm_path(path)
        y = torch.full((m, ldy), -7.0, dtype=torch.float32, device="cuda")
        nv.nvfp4_linear(A[0], A[1], 0.01, W[0], W[1], 0.02, m, N, K, y=y[:, :N],
                        out_dtype=nv.OUT_FP32)
        out = y.cpu().numpy()
        assert np.all(out[:, N:] == -7.0)
        H.check_gemm_fp32(out[:, :N], ref[:m], f"ldy path {path}")


@pytest.mark.parametrize("path", [LARGE, PAIR])
@pytest.mark.parametrize("ldy", [152, 160])
def test_bf16_row_stride_both_store_widths(ldy, path):
    """bf16 rows of 304 bytes take 16-byte stores, rows of 320 bytes whole 32-byte sectors."""
    M, N, K = 200, 144, 256
    rng = np.random.default_rng(ldy)
    ac = rng.integers(0, 16, size=(M, K)).astype(np.uint8)
    wc = rng.integers(0, 16, size=(N, K)).astype(np.uint8)
    as_ = rng.integers(0x30, 0x40, size=(M, K // 16)).astype(np.uint8)
    ws = rng.integers(0x30, 0x40, size=(N, K // 16)).astype(np.uint8)
    A, W = dev_operands(ac, as_, M, K), dev_operands(wc, ws, N, K)
    nv.nvfp4_set_gemm_path(path)
    y32 = nv.nvfp4_linear(A[0], A[1], 0.01, W[0], W[1], 0.02, M, N, K, out_dtype=nv.OUT_FP32)
    y = torch.full((M, ldy), 3.0, dtype=torch.bfloat16, device="cuda")
    nv.nvfp4_linear(A[0], A[1], 0.01, W[0], W[1], 0.02, M, N, K, y=y[:, :N])
    out = y.float().cpu().numpy()
    assert np.all(out[:, N:] == 3.0)
    np.testing.assert_array_equal(out[:, :N], H.bf16_round(y32.cpu().numpy()))


# ------------------------------------------------------------ launch overlap
@pytest.fixture
def overlap():
    nv.nvfp4_set_launch_overlap(True)
    yield
    nv.nvfp4_set_launch_overlap(H.LAUNCH_OVERLAP_DEFAULT)


def _decode_layer(M, N, K, seed):
    xb = workloads.random_bf16((M, K), seed=seed, std=1.0)
    wb = workloads.random_bf16((N, K), seed=seed + 1, std=1 / np.sqrt(K))
    a_gs = float(oracle.global_scale(np.abs(H.f32(xb)).max()))
    wc, ws, (w_gs,) = nv.nvfp4_quantize_weight(H.bf16_dev(wb))
    return xb, wb, a_gs, wc, ws, w_gs


@pytest.mark.parametrize("M", [1, 8, 17, 40, 64])
def test_overlap_gives_identical_results(M, overlap):
    """quantise + small-M GEMM chains with launch overlap on equal the plain launches bit for bit."""
    N, K = 1040, 2048
    xb, _, a_gs, wc, ws, w_gs = _decode_layer(M, N, K, seed=M)
    nv.nvfp4_set_launch_overlap(False)
    ac, as_ = nv.nvfp4_quantize_act(H.bf16_dev(xb), a_gs)
    ref = nv.nvfp4_linear(ac, as_, a_gs, wc, ws, w_gs, M, N, K, out_dtype=nv.OUT_FP32).cpu()
    nv.nvfp4_set_launch_overlap(True)
    x = H.bf16_dev(xb)
    for _ in range(3):
        ac2, as2 = nv.nvfp4_quantize_act(x, a_gs)
        y = nv.nvfp4_linear(ac2, as2, a_gs, wc, ws, w_gs, M, N, K, out_dtype=nv.OUT_FP32)
        assert torch.equal(y.cpu(), ref)
        assert torch.equal(ac2.cpu(), ac.cpu()) and torch.equal(as2.cpu(), as_.cpu())
    assert nv.nvfp4_last_device_error()[0] == 0


def test_overlap_keeps_stream_order_of_shared_buffers(overlap):
    """Consecutive layers sharing one code buffer and one output buffer: the
    quantiser of layer i+1 must not overwrite the codes layer i's GEMM still
    reads, and each GEMM must read the codes just written (read-after-write,
    write-after-read and write-after-write through the same buffers)."""
    M, N, K = 16, 2064, 1024
    layers = [_decode_layer(M, N, K, seed=100 + 7 * i) for i in range(4)]
    nv.nvfp4_set_launch_overlap(False)
    expect = []
    for xb, _, a_gs, wc, ws, w_gs in layers:
        ac, as_ = nv.nvfp4_quantize_act(H.bf16_dev(xb), a_gs)
        expect.append(nv.nvfp4_linear(ac, as_, a_gs, wc, ws, w_gs, M, N, K, out_dtype=nv.OUT_FP32).cpu())
    nv.nvfp4_set_launch_overlap(True)
    xs = [H.bf16_dev(l[0]) for l in layers]
    codes = torch.empty((M, K // 2), dtype=torch.uint8, device="cuda")
    scales = torch.empty(nv.nvfp4_scale_bytes(M, K), dtype=torch.uint8, device="cuda")
    outs = [torch.empty((M, N), dtype=torch.float32, device="cuda") for _ in layers]
    y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    for rep in range(5):
        # one code buffer, back-to-back quantise / GEMM launches
        for i, (_, _, a_gs, wc, ws, w_gs) in enumerate(layers):
            nv.nvfp4_quantize_act(xs[i], a_gs, codes=codes, scales=scales)
            nv.nvfp4_linear(codes, scales, a_gs, wc, ws, w_gs, M, N, K, y=outs[i],
                            out_dtype=nv.OUT_FP32)
        for i in range(len(layers)):
            assert torch.equal(outs[i].cpu(), expect[i]), (rep, i)
        # one output buffer: the last GEMM's result stays
        for i, (_, _, a_gs, wc, ws, w_gs) in enumerate(layers):
            nv.nvfp4_quantize_act(xs[i], a_gs, codes=codes, scales=scales)
            nv.nvfp4_linear(codes, scales, a_gs, wc, ws, w_gs, M, N, K, y=y, out_dtype=nv.OUT_FP32)
        assert torch.equal(y.cpu(), expect[-1]), rep
    assert nv.nvfp4_last_device_error()[0] == 0


@pytest.mark.parametrize("path,M", [(AUTO, 300), (LARGE, 200), (PAIR, 300), (PAIR_NFAST, 520)])
def test_overlap_keeps_stream_order_large_gemm(path, M, overlap):
    """The same chain of layers through one code buffer and one output
    buffer on the large-M kernels (one CTA per tile, CTA pairs, both
    rasters), each launched just behind the quantiser that writes its
    activation codes: bit-identical to the launches without overlap."""
    N, K = 2064, 1024
    nv.nvfp4_set_gemm_path(path)
    layers = [_decode_layer(M, N, K, seed=300 + 11 * i) for i in range(3)]
    nv.nvfp4_set_launch_overlap(False)
    expect = []
    for xb, _, a_gs, wc, ws, w_gs in layers:
        ac, as_ = nv.nvfp4_quantize_act(H.bf16_dev(xb), a_gs)
        expect.append(nv.nvfp4_linear(ac, as_, a_gs, wc, ws, w_gs, M, N, K, out_dtype=nv.OUT_FP32).cpu())
    nv.nvfp4_set_launch_overlap(True)
    xs = [H.bf16_dev(l[0]) for l in layers]
    codes = torch.empty((M, K // 2), dtype=torch.uint8, device="cuda")
    scales = torch.empty(nv.nvfp4_scale_bytes(M, K), dtype=torch.uint8, device="cuda")
    outs = [torch.empty((M, N), dtype=torch.float32, device="cuda") for _ in layers]
    y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    for rep in range(3):
        for i, (_, _, a_gs, wc, ws, w_gs) in enumerate(layers):
            nv.nvfp4_quantize_act(xs[i], a_gs, codes=codes, scales=scales)
            nv.nvfp4_linear(codes, scales, a_gs, wc, ws, w_gs, M, N, K, y=outs[i],
                            out_dtype=nv.OUT_FP32)
        for i in range(len(layers)):
            assert torch.equal(outs[i].cpu(), expect[i]), (rep, i)
        for i, (_, _, a_gs, wc, ws, w_gs) in enumerate(layers):
            nv.nvfp4_quantize_act(xs[i], a_gs, codes=codes, scales=scales)
            nv.nvfp4_linear(codes, scales, a_gs, wc, ws, w_gs, M, N, K, y=y, out_dtype=nv.OUT_FP32)
        assert torch.equal(y.cpu(), expect[-1]), rep
    assert nv.nvfp4_last_device_error()[0] == 0


def test_overlap_mlp_chain(overlap):
    """quantise x -> gate_up + SiLU * up + requantisation of h -> down, the
    down GEMM with its stream-K workspace, repeated through the same h and y
    buffers with launch overlap: equal to the chain without overlap."""
    # down: 9 x 10 tiles of 256 x 256 on 74 pairs, so the workspace's
    # stream-K tail runs (flags and partial tiles behind griddep_wait)
    M, Hd, K, N2 = 2304, 640, 512, 2560
    xb = workloads.random_bf16((M, K), seed=71, std=1.0)
    wgu = workloads.random_bf16((2 * Hd, K), seed=72, std=1 / np.sqrt(K))
    wd = workloads.random_bf16((N2, Hd), seed=73, std=1 / np.sqrt(Hd))
    a_gs = float(oracle.global_scale(np.abs(H.f32(xb)).max()))
    wc, ws, (g_gs, u_gs) = nv.nvfp4_quantize_weight(H.bf16_dev(wgu), seg_offsets=[0, Hd])
    dc, dsc, (d_gs,) = nv.nvfp4_quantize_weight(H.bf16_dev(wd))
    h_gs = 0.01
    work = nv.nvfp4_gemm_workspace(torch.device("cuda"))
    x = H.bf16_dev(xb)

    def chain(hc, hs, y):
        ac, as_ = nv.nvfp4_quantize_act(x, a_gs)
        nv.nvfp4_gate_up_silu_quantize(ac, as_, wc, ws, M, Hd, K, a_gs, g_gs, u_gs, h_gs,
                                       h_codes=hc, h_scales=hs)
        segs = [nv.SegmentSpec(0, d_gs, h_gs)]
        nv.nvfp4_fused_linear(hc, hs, dc, dsc, M, N2, Hd, segs, y=y, out_dtype=nv.OUT_FP32,
                              workspace=work)

    hc = torch.empty((M, Hd // 2), dtype=torch.uint8, device="cuda")
    hs = torch.empty(nv.nvfp4_scale_bytes(M, Hd), dtype=torch.uint8, device="cuda")
    y = torch.empty((M, N2), dtype=torch.float32, device="cuda")
    nv.nvfp4_set_launch_overlap(False)
    chain(hc, hs, y)
    ref_h, ref_s, ref_y = hc.cpu(), hs.cpu(), y.cpu()
    nv.nvfp4_set_launch_overlap(True)
    for rep in range(4):
        chain(hc, hs, y)
    assert torch.equal(hc.cpu(), ref_h) and torch.equal(hs.cpu(), ref_s)
    assert torch.equal(y.cpu(), ref_y)
    assert nv.nvfp4_last_device_error()[0] == 0


# ----------------------------------------------- stream-K tail (workspace)
# Shapes with more 256 x 256 tiles than a B200's 74 CTA pairs and a partial
# last wave, so the last 74 + remainder tiles run as equal k-tile ranges per
# pair: 180 tiles with K = 512 (106 tiles of 2 k-tiles in ranges of 2-3
# k-tiles: heads and tails of one k-tile), 320 tiles with K = 1280 (98 tiles
# of 5 k-tiles, ranges of 6-7), ragged M and N inside the shared tiles.
@pytest.mark.parametrize("path,M,N,K", [
    (PAIR, 2304, 5120, 512), (PAIR, 4096, 5120, 1280), (PAIR, 2200, 5104, 512),
    (PAIR_NFAST, 2304, 5120, 512), (AUTO, 4096, 5120, 1280)])
def test_split_last_wave(path, M, N, K):
    rng = np.random.default_rng(M * 17 + N + K)
    ac = rng.integers(0, 16, size=(M, K)).astype(np.uint8)
    wc = rng.integers(0, 16, size=(N, K)).astype(np.uint8)
    as_ = rng.integers(0x28, 0x58, size=(M, K // 16)).astype(np.uint8)
    ws = rng.integers(0x28, 0x58, size=(N, K // 16)).astype(np.uint8)
    a_gs, w_gs = np.float32(0.0173), np.float32(0.00291)
    A, W = dev_operands(ac, as_, M, K), dev_operands(wc, ws, N, K)
    seg = [nv.SegmentSpec(0, float(w_gs), float(a_gs))]
    work = nv.nvfp4_gemm_workspace("cuda")
    nv.nvfp4_set_gemm_path(path)
    y32 = nv.nvfp4_fused_linear(A[0], A[1], W[0], W[1], M, N, K, seg, out_dtype=nv.OUT_FP32,
                                workspace=work)
    y32b = nv.nvfp4_fused_linear(A[0], A[1], W[0], W[1], M, N, K, seg, out_dtype=nv.OUT_FP32,
                                 workspace=work)
    yb = nv.nvfp4_fused_linear(A[0], A[1], W[0], W[1], M, N, K, seg, workspace=work)
    st, info = nv.nvfp4_last_device_error()
    assert st == 0, f"device error word {info:#x}"
    # every call leaves the flags at zero
    assert int(work[:4096].count_nonzero()) == 0
    y32, y32b = y32.cpu().numpy(), y32b.cpu().numpy()
    # head + tail is summed in a fixed order: no run-to-run variation
    np.testing.assert_array_equal(y32, y32b)
    ref = oracle.linear64(oracle.dequantize(ac, as_, a_gs), oracle.dequantize(wc, ws, w_gs))
    H.check_gemm_fp32(y32, ref, f"split {M}x{N}x{K}")
    H.check_bf16_out(yb.float().cpu().numpy(), y32, ref, f"split {M}x{N}x{K}")


def test_split_with_gates_and_small_workspace():
    """GDN gate segments inside tiles shared by two pairs; a workspace too
    small for one partial tile per pair gives exactly the plain result."""
    M, N, K = 2304, 5120, 512
    rng = np.random.default_rng(5)
    ac = rng.integers(0, 16, size=(M, K)).astype(np.uint8)
    wc = rng.integers(0, 16, size=(N, K)).astype(np.uint8)
    as_ = rng.integers(0x28, 0x58, size=(M, K // 16)).astype(np.uint8)
    ws = rng.integers(0x28, 0x58, size=(N, K // 16)).astype(np.uint8)
    A, W = dev_operands(ac, as_, M, K), dev_operands(wc, ws, N, K)
    width = 128
    a_log = torch.from_numpy(rng.uniform(-1, 1.5, width).astype(np.float32)).cuda()
    dt_bias = torch.from_numpy(rng.normal(0, 0.5, width).astype(np.float32)).cuda()
    seg = [nv.SegmentSpec(0, 0.002, 0.02), nv.SegmentSpec(N - 2 * width, 0.003, 0.02, nv.OP_SIGMOID),
           nv.SegmentSpec(N - width, 0.004, 0.02, nv.OP_GDN_DECAY, a_log, dt_bias)]
    nv.nvfp4_set_gemm_path(PAIR)
    plain = nv.nvfp4_fused_linear(A[0], A[1], W[0], W[1], M, N, K, seg, out_dtype=nv.OUT_FP32)
    work = nv.nvfp4_gemm_workspace("cuda")
    split = nv.nvfp4_fused_linear(A[0], A[1], W[0], W[1], M, N, K, seg, out_dtype=nv.OUT_FP32,
                                  workspace=work)
    tiny = torch.zeros(4096 + 262144, dtype=torch.uint8, device="cuda")
    unsplit = nv.nvfp4_fused_linear(A[0], A[1], W[0], W[1], M, N, K, seg, out_dtype=nv.OUT_FP32,
                                    workspace=tiny)
    st, info = nv.nvfp4_last_device_error()
    assert st == 0, f"device error word {info:#x}"
    np.testing.assert_array_equal(unsplit.cpu().numpy(), plain.cpu().numpy())
    xa = oracle.dequantize(ac, as_, np.float32(0.02))
    pre = np.concatenate([oracle.linear64(xa, oracle.dequantize(wc[:N - 2 * width], ws[:N - 2 * width], np.float32(0.002))),
                          oracle.linear64(xa, oracle.dequantize(wc[N - 2 * width:N - width], ws[N - 2 * width:N - width], np.float32(0.003))),
                          oracle.linear64(xa, oracle.dequantize(wc[N - width:], ws[N - width:], np.float32(0.004)))], axis=1)
    out = split.cpu().numpy()
    # gate bars: e = 1e-3 rms of the module's pre-activation through the
    # gates' Lipschitz constants, as in the fused-projection tests
    b_sl, g_sl = slice(N - 2 * width, N - width), slice(N - width, N)
    H.check_gemm_fp32(out[:, :N - 2 * width], pre[:, :N - 2 * width], "split none")
    e_b = 1e-3 * np.sqrt(np.mean(pre[:, b_sl] ** 2))
    assert np.all(np.abs(out[:, b_sl] - oracle.sigmoid64(pre[:, b_sl])) <= 0.25 * e_b + 2e-6)
    e_g = 1e-3 * np.sqrt(np.mean(pre[:, g_sl] ** 2))
    a_log64 = a_log.cpu().numpy().astype(np.float64)
    g_ref = oracle.gdn_decay64(pre[:, g_sl], a_log64, dt_bias.cpu().numpy().astype(np.float64))
    bound = np.exp(a_log64)[None, :] * e_g + 2e-5 * np.abs(g_ref) + 1e-6
    assert np.all(np.abs(out[:, g_sl] - g_ref) <= bound)
