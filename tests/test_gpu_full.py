"""GPU parity at the full sizes of every workload, on sampled outputs.

The CUDA path runs each workload at its full size through the same calls
bench.py times (nvfp4_quantize_act + nvfp4_fused_linear, automatic kernel
choice).  The oracle recomputes sampled rows: the activation rows are
quantised by the oracle (codes and scales must match bit for bit), the
weights are quantised by the oracle with each module's own global scale
(codes and scales of sampled weight rows must match bit for bit), and the
sampled output rows are compared with the float64 product under the stated
bar (fp32 max |err| <= 1e-3 rms, relative Frobenius <= 1e-5; bf16 output =
RNE of the fp32 output; gates within their Lipschitz-propagated bounds).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
import nvfp4_w4a4_quantized_quantizer_b200 as nv
from tests import _helpers as H

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

OPS = {"none": nv.OP_NONE, "sigmoid": nv.OP_SIGMOID, "gdn_decay": nv.OP_GDN_DECAY}


def _sample_rows(M, n, seed):
    """Rows compared at full size: the edge rows, one random row inside every
    128-row block (each 128-row half of every 256-row CTA-pair tile, so every
    M-tile and both CTAs of every pair are compared), then random rows up to n."""
    rng = np.random.default_rng(seed)
    fixed = [0, M - 1] + [r for r in (127, 128, 255, 256) if r < M]
    per_block = [b + int(rng.integers(0, min(128, M - b))) for b in range(0, M, 128)]
    base = np.unique(np.array(fixed + per_block, np.int64))
    pool = np.setdiff1d(np.arange(M), base)
    rest = rng.choice(pool, size=max(0, min(len(pool), n - len(base))), replace=False)
    return np.unique(np.concatenate([base, rest]).astype(np.int64))


def _rows(t, rs):
    """Rows `rs` of a device tensor, gathered on the device, as numpy (bf16
    rows as float32 values)."""
    r = t[torch.from_numpy(rs).to(t.device)]
    return (r.float() if r.dtype == torch.bfloat16 else r).cpu().numpy()


def _oracle_weights(wf, wl, rows=None):
    """Per-module gs (whole module) and dequantised weight rows (all, or `rows`)."""
    offs = wl.seg_offsets + [wl.N]
    gs = [oracle.global_scale(np.abs(wf[offs[i]:offs[i + 1]]).max()) for i in range(len(wl.segments))]
    rows = np.arange(wl.N) if rows is None else np.asarray(rows)
    seg = np.searchsorted(np.array(offs), rows, side="right") - 1
    codes = np.empty((len(rows), wl.K), np.uint8)
    scales = np.empty((len(rows), wl.K // 16), np.uint8)
    what = np.empty((len(rows), wl.K), np.float64)
    for s in range(len(wl.segments)):
        idx = np.nonzero(seg == s)[0]
        for c in range(0, len(idx), 2048):
            sel = idx[c:c + 2048]
            q, sc = oracle.quantize(wf[rows[sel]], gs[s])
            codes[sel], scales[sel] = q, sc
            what[sel] = oracle.dequantize(q, sc, gs[s])
    return gs, codes, scales, what


def _gpu_layer(wl, xbits, wbits, calib_bits):
    a_gs = nv.nvfp4_global_scale(nv.nvfp4_amax(H.bf16_dev(calib_bits)).item())
    ac, as_ = nv.nvfp4_quantize_act(H.bf16_dev(xbits), a_gs)
    wc, ws, w_gs = nv.nvfp4_quantize_weight(H.bf16_dev(wbits), seg_offsets=wl.seg_offsets)
    gate = {}
    if any(s.op == "gdn_decay" for s in wl.segments):
        a_log, dt = workloads.gate_params(wl)
        gate = dict(a_log=torch.from_numpy(a_log).cuda(), dt=torch.from_numpy(dt).cuda())
    specs = [nv.SegmentSpec(o, w_gs[i], a_gs, OPS[s.op],
                            gate.get("a_log") if s.op == "gdn_decay" else None,
                            gate.get("dt") if s.op == "gdn_decay" else None)
             for i, (s, o) in enumerate(zip(wl.segments, wl.seg_offsets))]
    M = xbits.shape[0]
    # with the workspace (a stream-K tail when the tiles do not fill the
    # last wave), so that path is checked at full size too
    work = nv.nvfp4_gemm_workspace("cuda")
    y32 = nv.nvfp4_fused_linear(ac, as_, wc, ws, M, wl.N, wl.K, specs, out_dtype=nv.OUT_FP32,
                                workspace=work)
    yb = nv.nvfp4_fused_linear(ac, as_, wc, ws, M, wl.N, wl.K, specs, workspace=work)
    st, info = nv.nvfp4_last_device_error()
    assert st == 0, hex(info)
    assert int(work[:4096].count_nonzero()) == 0
    if M == 4096:
        # the prefill GEMM's 320 tiles leave a partial last wave on 74 pairs,
        # so the workspace call shares tiles between pairs: their fp32 sums
        # associate differently
        plain = nv.nvfp4_fused_linear(ac, as_, wc, ws, M, wl.N, wl.K, specs, out_dtype=nv.OUT_FP32)
        assert not torch.equal(plain, y32)
        del plain
    return a_gs, w_gs, ac, as_, wc, ws, y32, yb


def _check_layer(wl, M, rows_sample, wrow_sample, seed):
    calib = workloads.activations(wl, calib=True)
    xbits = workloads.activations(wl, M=M)
    wbits = workloads.weights(wl)
    a_gs, w_gs, ac, as_, wc, ws, y32, yb = _gpu_layer(wl, xbits, wbits, calib)
    # calibration: exact
    a_gs_ref = oracle.global_scale(np.abs(H.f32(calib)).max())
    assert np.float32(a_gs) == a_gs_ref
    # activations: sampled rows bit-exact
    rs = _sample_rows(M, rows_sample, seed)
    xf = H.f32(xbits[rs])
    qx, sx = oracle.quantize(xf, a_gs_ref)
    codes_gpu = H.unpack_codes(_rows(ac, rs))
    np.testing.assert_array_equal(codes_gpu, qx)
    np.testing.assert_array_equal(H.sf_logical(as_.cpu().numpy(), M, wl.K)[rs], sx)
    # weights: per-module gs exact, sampled rows bit-exact
    wf = H.f32(wbits)
    gs_ref, wq, wsc, what = _oracle_weights(wf, wl)
    assert [np.float32(g) for g in w_gs] == gs_ref
    ws_rows = _sample_rows(wl.N, wrow_sample, seed + 1)
    np.testing.assert_array_equal(H.unpack_codes(wc.cpu().numpy()[ws_rows]), wq[ws_rows])
    np.testing.assert_array_equal(H.sf_logical(ws.cpu().numpy(), wl.N, wl.K)[ws_rows], wsc[ws_rows])
    # outputs of the sampled rows
    pre = oracle.dequantize(qx, sx, a_gs_ref) @ what.T
    y = _rows(y32, rs)
    ybf = _rows(yb, rs)
    offs = wl.seg_offsets + [wl.N]
    for i, s in enumerate(wl.segments):
        sl = slice(offs[i], offs[i + 1])
        if s.op == "none":
            H.check_gemm_fp32(y[:, sl], pre[:, sl], f"{wl.name} module {s.name}")
            H.check_bf16_out(ybf[:, sl], y[:, sl], pre[:, sl], f"{wl.name} module {s.name}")
            continue
        e = 1e-3 * np.sqrt(np.mean(pre[:, sl] ** 2))
        if s.op == "sigmoid":
            ref = oracle.sigmoid64(pre[:, sl])
            assert np.all(np.abs(y[:, sl] - ref) <= 0.25 * e + 2e-6), s.name
        else:
            a_log, dt = workloads.gate_params(wl)
            ref = oracle.gdn_decay64(pre[:, sl], a_log[None, :], dt[None, :])
            bound = np.exp(a_log)[None, :] * e + 2e-5 * np.abs(ref) + 1e-6
            assert np.all(np.abs(y[:, sl] - ref) <= bound), s.name
        np.testing.assert_array_equal(ybf[:, sl], H.bf16_round(y[:, sl]))


def test_prefill_full():
    _check_layer(workloads.WORKLOADS[2], 4096, 48, 256, seed=20)


def test_gdn_inproj_full():
    _check_layer(workloads.WORKLOADS[3], 8192, 32, 256, seed=30)


@pytest.mark.parametrize("M", [1, 8, 32, 64])
def test_decode_sweep_full(M):
    # with launch overlap, as bench.py runs the decode workload
    nv.nvfp4_set_launch_overlap(True)
    try:
        _check_layer(workloads.WORKLOADS[5], M, M, 256, seed=50 + M)
    finally:
        nv.nvfp4_set_launch_overlap(H.LAUNCH_OVERLAP_DEFAULT)


def test_mlp_pair_full():
    """The MLP pair at full size, launched as bench.py launches it.

    gate_up (16384 x 5120 -> 2 x 17408, two modules): sampled rows (every
    128-row block) of its fp32 and bf16 outputs against the float64 oracle.
    h = the GPU's own SiLU(gate) * up of the bf16 gate_up output, requantised
    under the static down-input scale: the sampled rows' codes and scales
    equal the oracle quantiser's of the same h rows bit for bit, and the
    one-kernel gate_up + SiLU * up + requantisation gives the same codes and
    scales.  The down projection (16384 x 17408 -> 5120) on those codes, on
    the automatic path (the CTA-pair kernel with the activation-sharing
    raster, K = 17408, with the workspace): the sampled output rows against
    the float64 product of the oracle-dequantised operands at the GEMM bar,
    fp32 and bf16.  As an extra, the chain's deviation from the oracle's own
    chain (oracle gate_up -> SiLU * up -> quantise) stays below half of what
    NVFP4 quantisation of h itself costs."""
    wl = workloads.WORKLOADS[4]
    M, K, H2, N2 = wl.M, wl.K, wl.N // 2, workloads.MLP_DOWN_N
    assert workloads.MLP_DOWN_K == H2
    calib = workloads.activations(wl, calib=True)
    xbits = workloads.activations(wl)
    wbits = workloads.weights(wl)
    a_gs, w_gs, ac, as_, wc, ws, y32, yb = _gpu_layer(wl, xbits, wbits, calib)
    a_gs_ref = oracle.global_scale(np.abs(H.f32(calib)).max())
    assert np.float32(a_gs) == a_gs_ref
    rs = _sample_rows(M, 160, 40)
    assert len(np.unique(rs // 128)) == M // 128
    qx, sx = oracle.quantize(H.f32(xbits[rs]), a_gs_ref)
    np.testing.assert_array_equal(H.unpack_codes(_rows(ac, rs)), qx)
    np.testing.assert_array_equal(H.sf_logical(as_.cpu().numpy(), M, K)[rs], sx)
    wf = H.f32(wbits)
    del wbits
    gs_ref, wq, wsc, what = _oracle_weights(wf, wl)
    del wf
    assert [np.float32(g) for g in w_gs] == gs_ref
    wrows = _sample_rows(wl.N, 256, 41)
    np.testing.assert_array_equal(H.unpack_codes(_rows(wc, wrows)), wq[wrows])
    np.testing.assert_array_equal(H.sf_logical(ws.cpu().numpy(), wl.N, K)[wrows], wsc[wrows])
    del wq, wsc
    gu = oracle.dequantize(qx, sx, a_gs_ref) @ what.T          # [rows, 34816] float64
    del what
    y = _rows(y32, rs)
    del y32
    for sl in (slice(0, H2), slice(H2, 2 * H2)):
        H.check_gemm_fp32(y[:, sl], gu[:, sl], "gate_up")
    H.check_bf16_out(_rows(yb, rs), y, gu, "gate_up")

    # the down input's static global scale, calibrated as bench.py does: the
    # chain on the calibration batch (any positive value is a valid input to
    # both sides; this one has the workload's scale)
    nv_calib = H.bf16_dev(calib)
    cc, cs = nv.nvfp4_quantize_act(nv_calib, a_gs)
    segs = [nv.SegmentSpec(o, g, a_gs) for o, g in zip(wl.seg_offsets, w_gs)]
    h_cal = nv.nvfp4_silu_mul(nv.nvfp4_fused_linear(cc, cs, wc, ws, calib.shape[0], wl.N, K, segs), H2)
    a2 = nv.nvfp4_global_scale(nv.nvfp4_amax(h_cal).item())
    del nv_calib, cc, cs, h_cal

    # the GPU's own h, requantised: sampled rows bit for bit against the oracle
    h = nv.nvfp4_silu_mul(yb, H2)
    del yb
    hc, hs = nv.nvfp4_quantize_act(h, a2)
    h_rows = _rows(h, rs)                                       # bf16 values as float32
    del h
    qh, sh = oracle.quantize(h_rows, np.float32(a2))
    np.testing.assert_array_equal(H.unpack_codes(_rows(hc, rs)), qh)
    np.testing.assert_array_equal(H.sf_logical(hs.cpu().numpy(), M, H2)[rs], sh)
    assert not H.sf_padding_rows(hs.cpu().numpy(), M, H2).any()
    # the one-kernel form (as bench.py runs the MLP step): same codes and scales
    fc, fs = nv.nvfp4_gate_up_silu_quantize(ac, as_, wc, ws, M, H2, K, a_gs, w_gs[0], w_gs[1], a2)
    assert torch.equal(fc, hc) and torch.equal(fs, hs)
    del fc, fs, ac, as_, wc, ws

    # down weights: gs exact, sampled rows bit-exact
    w2bits = workloads.down_weights()
    w2f = H.f32(w2bits)
    g2 = oracle.global_scale(np.abs(w2f).max())
    q2, s2 = oracle.quantize(w2f, g2)
    w2hat = oracle.dequantize(q2, s2, g2)
    del w2f
    w2c, w2s, (g2_gpu,) = nv.nvfp4_quantize_weight(H.bf16_dev(w2bits))
    assert np.float32(g2_gpu) == g2
    w2rows = _sample_rows(N2, 256, 42)
    np.testing.assert_array_equal(H.unpack_codes(_rows(w2c, w2rows)), q2[w2rows])
    np.testing.assert_array_equal(H.sf_logical(w2s.cpu().numpy(), N2, H2)[w2rows], s2[w2rows])
    del q2, s2

    # the down GEMM at M = 16384 on the automatic path, with the workspace
    work = nv.nvfp4_gemm_workspace("cuda")
    segs2 = [nv.SegmentSpec(0, g2_gpu, a2)]
    d32 = nv.nvfp4_fused_linear(hc, hs, w2c, w2s, M, N2, H2, segs2, out_dtype=nv.OUT_FP32,
                                workspace=work)
    db = nv.nvfp4_fused_linear(hc, hs, w2c, w2s, M, N2, H2, segs2, workspace=work)
    st, info = nv.nvfp4_last_device_error()
    assert st == 0, hex(info)
    assert int(work[:4096].count_nonzero()) == 0
    d_rows = _rows(d32, rs)
    dref = oracle.dequantize(qh, sh, np.float32(a2)) @ w2hat.T
    H.check_gemm_fp32(d_rows, dref, "down")
    H.check_bf16_out(_rows(db, rs), d_rows, dref, "down")
    del d32, db

    # extra: the oracle's own chain on the same rows (its h from its float64
    # gate_up, rounded as reading R8 states) -- the GPU chain differs from it
    # only where a bf16 rounding of gate, up or h lands on the other side of
    # a rounding boundary, which moves a few codes by a grid step
    h_ref = oracle.silu_mul_bf16(gu[:, :H2], gu[:, H2:])
    assert np.mean(h_ref == h_rows) > 0.99
    qr, sr = oracle.quantize(h_ref, np.float32(a2))
    d_oracle = oracle.dequantize(qr, sr, np.float32(a2)) @ w2hat.T
    quant_err = np.linalg.norm(d_oracle - h_ref.astype(np.float64) @ w2hat.T)
    assert np.linalg.norm(d_rows - d_oracle) <= 0.5 * quant_err
