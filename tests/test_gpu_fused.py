"""GPU parity: fused multi-module projection with per-module global scales and
the GDN gate epilogue, vs the oracle.

The pages describe the global-scale mismatch of fused kernels serving
per-module-calibrated checkpoints and its repair (bayesiansapien wiki, "Two
practical repairs"; aimodeling, "What engineers should actually take away"),
and the sigmoid / softplus-exponential gates (wiki, mechanism study part 2).
Gate tolerances follow from the fp32 GEMM bar e = 1e-3 rms(pre-activation)
through the gates' Lipschitz constants: |dbeta| <= e/4, |dg| <= exp(A_log) e,
plus fp32 evaluation error of exp/log1p.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
import nvfp4_w4a4_quantized_quantizer_b200 as nv
from tests import _helpers as H

_H = H  # the helpers, where a parameter named H (the MLP hidden size) shadows them

pytestmark = pytest.mark.gpu

LARGE, SMALL, AUTO, PAIR, PAIR_NFAST = 1, 2, 0, 3, 4
OPS = {"none": nv.OP_NONE, "sigmoid": nv.OP_SIGMOID, "gdn_decay": nv.OP_GDN_DECAY}


@pytest.fixture(autouse=True)
def _reset_path():
    yield
    nv.nvfp4_set_gemm_path(AUTO)


def _mini_gdn(M, K, seed):
    """A scaled-down GDN in-projection: q | k | v | z | b | a with per-module stds."""
    widths = [64, 64, 192, 192, 48, 48]
    ops = ["none"] * 4 + ["sigmoid", "gdn_decay"]
    rng = np.random.default_rng(seed)
    stds = np.exp(rng.uniform(np.log(0.25), np.log(4.0), size=len(widths))) / np.sqrt(K)
    wbits = np.concatenate([workloads.random_bf16((wd, K), seed=seed + 10 + i, std=float(stds[i]))
                            for i, wd in enumerate(widths)])
    xbits = workloads.random_bf16((M, K), seed=seed + 99, std=1.5)
    a_log = rng.uniform(-1, 1.5, 48).astype(np.float32)
    dt = (rng.standard_normal(48) * 0.5).astype(np.float32)
    return widths, ops, wbits, xbits, a_log, dt


def _run_fused(path, M, K, seed):
    widths, ops, wbits, xbits, a_log, dt = _mini_gdn(M, K, seed)
    N = sum(widths)
    offs = np.cumsum([0] + widths[:-1]).tolist()
    xf, wf = H.f32(xbits), H.f32(wbits)
    a_gs = oracle.global_scale(np.abs(xf).max())
    ac, as_ = nv.nvfp4_quantize_act(H.bf16_dev(xbits), float(a_gs))
    wc, ws, w_gs = nv.nvfp4_quantize_weight(H.bf16_dev(wbits), seg_offsets=offs)
    a_log_d, dt_d = torch.from_numpy(a_log).cuda(), torch.from_numpy(dt).cuda()
    specs = [nv.SegmentSpec(o, w_gs[i], float(a_gs), OPS[ops[i]],
                            a_log_d if ops[i] == "gdn_decay" else None,
                            dt_d if ops[i] == "gdn_decay" else None)
             for i, o in enumerate(offs)]
    nv.nvfp4_set_gemm_path(path)
    y32 = nv.nvfp4_fused_linear(ac, as_, wc, ws, M, N, K, specs, out_dtype=nv.OUT_FP32)
    yb = nv.nvfp4_fused_linear(ac, as_, wc, ws, M, N, K, specs, out_dtype=nv.OUT_BF16)
    assert nv.nvfp4_last_device_error()[0] == 0
    # oracle: its own quantisation (codes checked bit-exact first)
    qx, sx = oracle.quantize(xf, a_gs)
    np.testing.assert_array_equal(H.unpack_codes(ac.cpu().numpy()), qx)
    qw = np.empty((N, K), np.uint8)
    sw = np.empty((N, K // 16), np.uint8)
    segs = []
    for i, (o, wd) in enumerate(zip(offs, widths)):
        gs = oracle.global_scale(np.abs(wf[o:o + wd]).max())
        assert np.float32(w_gs[i]) == gs
        qw[o:o + wd], sw[o:o + wd] = oracle.quantize(wf[o:o + wd], gs)
        segs.append(dict(n_offset=o, width=wd, w_gs=gs, a_gs=a_gs, op=ops[i], a_log=a_log, dt_bias=dt))
    np.testing.assert_array_equal(H.unpack_codes(wc.cpu().numpy()), qw)
    ref = oracle.fused_linear64(qx, sx, qw, sw, segs)
    pre = oracle.fused_linear64(qx, sx, qw, sw, [dict(s, op="none") for s in segs])
    return widths, offs, ops, a_log, y32.cpu().numpy(), yb.float().cpu().numpy(), ref, pre, (qx, sx, qw, sw, segs)


@pytest.mark.parametrize("path,M,K", [(LARGE, 200, 320), (LARGE, 384, 1024), (PAIR, 200, 320),
                                      (PAIR, 600, 1024), (PAIR_NFAST, 600, 1024), (SMALL, 5, 320),
                                      (SMALL, 64, 512), (AUTO, 1, 256)])
def test_fused_gdn_segments_and_gates(path, M, K):
    widths, offs, ops, a_log, y32, yb, ref, pre, _ = _run_fused(path, M, K, seed=M + K)
    for o, wd, op in zip(offs, widths, ops):
        sl = slice(o, o + wd)
        e = 1e-3 * np.sqrt(np.mean(pre[:, sl] ** 2))
        if op == "none":
            H.check_gemm_fp32(y32[:, sl], ref[:, sl], f"segment at {o}")
            H.check_bf16_out(yb[:, sl], y32[:, sl], ref[:, sl], f"segment at {o}")
        elif op == "sigmoid":
            assert np.all(np.abs(y32[:, sl] - ref[:, sl]) <= 0.25 * e + 2e-6)
            assert np.all((y32[:, sl] >= 0) & (y32[:, sl] <= 1))
        else:
            bound = np.exp(a_log)[None, :] * e + 2e-5 * np.abs(ref[:, sl]) + 1e-6
            assert np.all(np.abs(y32[:, sl] - ref[:, sl]) <= bound)
            assert np.all(y32[:, sl] <= 0)
        np.testing.assert_array_equal(yb[:, sl], H.bf16_round(y32[:, sl]))


def test_repair_vs_shared_scale():
    """Serving the fused weight with module 0's scales everywhere mis-scales every other
    module by exactly w_gs[0] / w_gs[s]; per-module alpha repairs it."""
    M, K = 130, 256
    widths, ops, wbits, xbits, _, _ = _mini_gdn(M, K, seed=3)
    N = sum(widths)
    offs = np.cumsum([0] + widths[:-1]).tolist()
    a_gs = oracle.global_scale(np.abs(H.f32(xbits)).max())
    ac, as_ = nv.nvfp4_quantize_act(H.bf16_dev(xbits), float(a_gs))
    wc, ws, w_gs = nv.nvfp4_quantize_weight(H.bf16_dev(wbits), seg_offsets=offs)
    good = [nv.SegmentSpec(o, w_gs[i], float(a_gs)) for i, o in enumerate(offs)]
    bad = [nv.SegmentSpec(o, w_gs[0], float(a_gs)) for o in offs]
    yg = nv.nvfp4_fused_linear(ac, as_, wc, ws, M, N, K, good, out_dtype=nv.OUT_FP32).cpu().numpy()
    yb = nv.nvfp4_fused_linear(ac, as_, wc, ws, M, N, K, bad, out_dtype=nv.OUT_FP32).cpu().numpy()
    for i, (o, wd) in enumerate(zip(offs, widths)):
        sl = slice(o, o + wd)
        ratio = (np.float32(a_gs) * np.float32(w_gs[0])) / (np.float32(a_gs) * np.float32(w_gs[i]))
        np.testing.assert_allclose(yb[:, sl], yg[:, sl] * ratio, rtol=3e-7,
                                   atol=1e-6 * np.abs(yb[:, sl]).max())
        if i > 0:
            assert abs(ratio - 1) > 1e-3        # the modules really do differ


# ------------------------------------------ MLP first half in one kernel
def _gate_up_operands(M, H, K, seed):
    rng = np.random.default_rng(seed)
    xb = workloads.random_bf16((M, K), seed=seed, std=1.0)
    std_g, std_u = 1 / np.sqrt(K), 3 / np.sqrt(K)          # up weights 3x the gate's scale
    wb = np.concatenate([workloads.random_bf16((H, K), seed=seed + 1, std=std_g),
                         workloads.random_bf16((H, K), seed=seed + 2, std=std_u)])
    a_gs = float(oracle.global_scale(np.abs(_H.f32(xb)).max()))
    ac, as_ = nv.nvfp4_quantize_act(_H.bf16_dev(xb), a_gs)
    wc, ws, (g_gs, u_gs) = nv.nvfp4_quantize_weight(_H.bf16_dev(wb), seg_offsets=[0, H])
    return ac, as_, wc, ws, a_gs, g_gs, u_gs, rng



@pytest.mark.parametrize("M,H,K", [(100, 128, 256), (256, 384, 512), (300, 256, 1280),
                                   (600, 640, 320), (2304, 1024, 256)])
def test_gate_up_silu_quantize_equals_the_unfused_chain(M, H, K):
    """One kernel = fused_linear (bf16, gate | up) -> silu_mul -> quantize_act, bit for bit,
    padding rows of the scale buffer included."""
    ac, as_, wc, ws, a_gs, g_gs, u_gs, _ = _gate_up_operands(M, H, K, seed=M + H + K)
    segs = [nv.SegmentSpec(0, g_gs, a_gs), nv.SegmentSpec(H, u_gs, a_gs)]
    nv.nvfp4_set_gemm_path(PAIR)        # the fused kernel is a CTA-pair kernel at every M
    gu = nv.nvfp4_fused_linear(ac, as_, wc, ws, M, 2 * H, K, segs)
    nv.nvfp4_set_gemm_path(AUTO)
    h = nv.nvfp4_silu_mul(gu, H)
    h_gs = float(oracle.global_scale(float(h.float().abs().max().item())))
    ref_c, ref_s = nv.nvfp4_quantize_act(h, h_gs)
    hc = torch.full((M, H // 2), 0xAB, dtype=torch.uint8, device="cuda")
    hs = torch.full((nv.nvfp4_scale_bytes(M, H),), 0xCD, dtype=torch.uint8, device="cuda")
    nv.nvfp4_gate_up_silu_quantize(ac, as_, wc, ws, M, H, K, a_gs, g_gs, u_gs, h_gs,
                                   h_codes=hc, h_scales=hs)
    st, info = nv.nvfp4_last_device_error()
    assert st == 0, f"device error word {info:#x}"
    assert torch.equal(hc, ref_c)
    assert torch.equal(hs, ref_s)


def test_silu_mul_matches_the_oracle_within_one_bf16_step():
    """nvfp4_silu_mul (fp32 steps) against the float64 oracle on the same bf16 gate / up."""
    M, Hd = 64, 4096
    rng = np.random.default_rng(3)
    g = workloads.f32_to_bf16_bits(rng.normal(0, 3, (M, Hd)).astype(np.float32))
    u = workloads.f32_to_bf16_bits(rng.normal(0, 2, (M, Hd)).astype(np.float32))
    gu = np.concatenate([g, u], axis=1)
    h = nv.nvfp4_silu_mul(H.bf16_dev(gu), Hd).float().cpu().numpy()
    ref = oracle.silu_mul_bf16(H.f32(g), H.f32(u))
    # both are bf16-rounded: at most one bf16 step apart (fp32 vs float64 inner steps)
    step = np.abs(ref).astype(np.float64) * 2.0 ** -7 + 1e-30
    assert np.all(np.abs(h.astype(np.float64) - ref) <= step)
    assert np.mean(h == ref) > 0.99


@pytest.mark.parametrize("path,M,K", [(PAIR, 200, 320), (SMALL, 7, 320), (LARGE, 100, 256)])
def test_preharmonised_checkpoint(path, M, K):
    """The pages' other repair: every module of the fused weight quantised under
    one shared global scale ("pre-harmonised"), served with that scale in every
    segment; gates still apply per module."""
    widths, ops, wbits, xbits, a_log, dt = _mini_gdn(M, K, seed=M + 5)
    N = sum(widths)
    offs = np.cumsum([0] + widths[:-1]).tolist()
    xf, wf = H.f32(xbits), H.f32(wbits)
    a_gs = oracle.global_scale(np.abs(xf).max())
    ac, as_ = nv.nvfp4_quantize_act(H.bf16_dev(xbits), float(a_gs))
    wc, ws, (w_gs,) = nv.nvfp4_quantize_weight(H.bf16_dev(wbits))          # one module
    gs_ref = oracle.global_scale(np.abs(wf).max())
    assert np.float32(w_gs) == gs_ref
    a_log_d, dt_d = torch.from_numpy(a_log).cuda(), torch.from_numpy(dt).cuda()
    specs = [nv.SegmentSpec(o, w_gs, float(a_gs), OPS[ops[i]],
                            a_log_d if ops[i] == "gdn_decay" else None,
                            dt_d if ops[i] == "gdn_decay" else None)
             for i, o in enumerate(offs)]
    nv.nvfp4_set_gemm_path(path)
    y32 = nv.nvfp4_fused_linear(ac, as_, wc, ws, M, N, K, specs, out_dtype=nv.OUT_FP32)
    assert nv.nvfp4_last_device_error()[0] == 0
    y32 = y32.cpu().numpy()
    qx, sx = oracle.quantize(xf, a_gs)
    qw, sw = oracle.quantize(wf, gs_ref)
    np.testing.assert_array_equal(H.unpack_codes(wc.cpu().numpy()), qw)
    segs = [dict(n_offset=o, width=wd, w_gs=gs_ref, a_gs=a_gs, op=ops[i], a_log=a_log, dt_bias=dt)
            for i, (o, wd) in enumerate(zip(offs, widths))]
    ref = oracle.fused_linear64(qx, sx, qw, sw, segs)
    pre = oracle.fused_linear64(qx, sx, qw, sw, [dict(s, op="none") for s in segs])
    for o, wd, op in zip(offs, widths, ops):
        sl = slice(o, o + wd)
        e = 1e-3 * np.sqrt(np.mean(pre[:, sl] ** 2))
        if op == "none":
            H.check_gemm_fp32(y32[:, sl], ref[:, sl], f"harmonised segment at {o}")
        elif op == "sigmoid":
            assert np.all(np.abs(y32[:, sl] - ref[:, sl]) <= 0.25 * e + 2e-6)
        else:
            bound = np.exp(a_log)[None, :] * e + 2e-5 * np.abs(ref[:, sl]) + 1e-6
            assert np.all(np.abs(y32[:, sl] - ref[:, sl]) <= bound)
