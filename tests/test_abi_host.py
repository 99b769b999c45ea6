"""The C-ABI library: it loads, exports every symbol include/nvfp4.h declares,
and validates arguments on the host before touching a GPU (CPU only)."""
import ctypes
import os
import re

import pytest

from nvfp4_w4a4_quantized_quantizer_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "nvfp4.h")

INVALID, ALIGN, SHAPE = -1, -2, -3


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(nvfp4_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    return _lib.load()


def test_header_declares_the_layer_entry_points():
    names = declared_functions()
    for must in ("nvfp4_quantize_act", "nvfp4_quantize_weight", "nvfp4_linear",
                 "nvfp4_fused_linear"):
        assert must in names


def test_every_declared_symbol_is_exported_and_bound(lib):
    names = declared_functions()
    assert names, "no declarations parsed"
    for n in names:
        assert hasattr(lib, n), f"{n} not exported by libnvfp4.so"
        assert n in _lib.SIGNATURES, f"{n} has no ctypes signature in the binding"
    assert set(_lib.SIGNATURES) == set(names)


def test_size_helpers(lib):
    assert lib.nvfp4_codes_bytes(64, 256) == 64 * 128
    assert lib.nvfp4_scale_bytes(64, 256) == 128 * 16
    assert lib.nvfp4_scale_bytes(129, 5120) == 256 * 320
    assert lib.nvfp4_scale_bytes(0, 64) == 0
    assert lib.nvfp4_quantize_weight_workspace_bytes(6) == 256


def test_noalloc_limit_matches_header(lib):
    text = open(os.path.join(ROOT, "include", "nvfp4.h")).read()
    m = re.search(r"#define\s+NVFP4_NOALLOC_MAX_SEGMENTS\s+(\d+)", text)
    assert m and lib.nvfp4_noalloc_max_segments() == int(m.group(1))


def test_global_scale_matches_fp32_division(lib):
    import numpy as np
    for amax in (1.0, 123.456, 6.0e4, 3.1e-3):
        assert lib.nvfp4_global_scale(ctypes.c_float(amax)) == float(
            np.float32(np.float32(amax) / np.float32(2688.0)))
    assert lib.nvfp4_global_scale(ctypes.c_float(0.0)) == 1.0


def test_status_strings(lib):
    for s in (0, -1, -2, -3, -4, -5, -6):
        assert lib.nvfp4_status_string(s)


P = ctypes.c_void_p(0x10000)          # a 16-byte-aligned dummy address (never dereferenced)
P_MIS = ctypes.c_void_p(0x10008)      # misaligned
NUL = ctypes.c_void_p(0)


def test_quantize_act_validation(lib):
    q = lib.nvfp4_quantize_act
    assert q(NUL, 4, 64, 64, 1.0, P, P, NUL) == INVALID
    assert q(P, 4, 48, 48, 1.0, P, P, NUL) == SHAPE          # K % 64
    assert q(P, 4, 64, 32, 1.0, P, P, NUL) == SHAPE          # ld < K
    assert q(P_MIS, 4, 64, 64, 1.0, P, P, NUL) == ALIGN
    assert q(P, 4, 64, 68, 1.0, P, P, NUL) == ALIGN          # ld % 8
    assert q(P, 4, 64, 64, 1.0, P_MIS, P, NUL) == ALIGN
    assert q(P, 4, 64, 64, 0.0, P, P, NUL) == INVALID        # gs must be > 0
    assert q(P, 4, 64, 64, float("nan"), P, P, NUL) == INVALID
    assert q(P, 4, 64, 64, float("inf"), P, P, NUL) == INVALID
    assert q(P, -1, 64, 64, 1.0, P, P, NUL) == SHAPE
    assert q(P, 0, 64, 64, 1.0, P, P, NUL) == 0              # M == 0 is a no-op


def _segs(*entries):
    arr = (_lib.Segment * len(entries))()
    for i, (off, op) in enumerate(entries):
        arr[i] = _lib.Segment(off, 1e-3, 1e-2, op, None, None)
    return arr


def test_fused_linear_validation(lib):
    f = lib.nvfp4_fused_linear
    ok = _segs((0, 0), (32, 1))
    args = lambda segs, nseg, M=8, N=64, K=128, ldy=64, dt=0, y=P: (  # noqa: E731
        P, P, P, P, M, N, K, segs, nseg, y, ldy, dt, NUL)
    assert f(*args(ok, 2, K=96)) == SHAPE                     # K % 64
    assert f(*args(ok, 2, N=56)) == SHAPE                     # N % 16
    assert f(*args(ok, 2, ldy=32)) == SHAPE                   # ldy < N
    assert f(*args(ok, 2, ldy=68)) == ALIGN                   # bf16 rows not 16-byte multiples
    assert f(*args(ok, 2, dt=5)) == INVALID
    assert f(*args(ok, 2, y=P_MIS)) == ALIGN
    assert f(*args(_segs((16, 0)), 1)) == INVALID             # first offset must be 0
    assert f(*args(_segs((0, 0), (0, 0)), 2)) == INVALID      # not ascending
    assert f(*args(_segs((0, 0), (24, 0)), 2)) == SHAPE       # offset % 16
    assert f(*args(_segs((0, 0), (64, 0)), 2)) == INVALID     # offset >= N
    assert f(*args(_segs((0, 7)), 1)) == INVALID              # bad op
    assert f(*args(_segs((0, 2)), 1)) == INVALID              # GDN decay needs A_log / dt_bias
    assert f(*args(ok, 0)) == INVALID
    assert f(*args(ok, 33)) == INVALID
    bad_gs = (_lib.Segment * 1)(_lib.Segment(0, 0.0, 1.0, 0, None, None))
    assert f(*args(bad_gs, 1)) == INVALID
    assert f(*args(ok, 2, M=0)) == 0                          # no-op


def test_gemm_workspace(lib):
    # arrival counters + 128 fp32 partial tiles of 2 x 128 x 256
    assert lib.nvfp4_gemm_workspace_bytes() == 4096 + 128 * 2 * 128 * 256 * 4
    f = lib.nvfp4_fused_linear_ws
    ok = _segs((0, 0), (32, 1))
    args = lambda work, M=8, K=128: (P, P, P, P, M, 64, K, ok, 2, P, 64, 0, work,  # noqa: E731
                                     lib.nvfp4_gemm_workspace_bytes(), NUL)
    assert f(*args(P_MIS)) == ALIGN                           # workspace not 16-byte aligned
    assert f(*args(P, K=96)) == SHAPE                         # the fused_linear checks apply
    assert f(*args(P, M=0)) == 0
    assert f(*args(NUL, M=0)) == 0                            # no workspace: plain fused_linear


def test_linear_and_weight_validation(lib):
    assert lib.nvfp4_linear(P, P, 1.0, P, P, 1.0, 4, 64, 64, NUL, 64, 0, NUL) == INVALID
    assert lib.nvfp4_linear(P, P, -1.0, P, P, 1.0, 4, 64, 64, P, 64, 0, NUL) == INVALID
    offs = (ctypes.c_int64 * 2)(0, 24)
    gs = (ctypes.c_float * 2)()
    w = lib.nvfp4_quantize_weight
    assert w(P, 64, 64, 64, offs, 2, gs, P, P, P, NUL) == SHAPE      # offset % 16
    offs2 = (ctypes.c_int64 * 2)(0, 64)
    assert w(P, 64, 64, 64, offs2, 2, gs, P, P, P, NUL) == INVALID   # offset >= N
    assert w(P, 60, 64, 64, None, 1, gs, P, P, P, NUL) == SHAPE      # N % 16
    assert w(P, 64, 64, 64, None, 2, gs, P, P, P, NUL) == INVALID    # nseg > 1 needs offsets
    assert w(P, 64, 64, 64, None, 1, gs, P, P, NUL, NUL) == INVALID  # workspace required


def test_gate_up_silu_quantize_validation(lib):
    f = lib.nvfp4_gate_up_silu_quantize
    args = lambda M=8, H=128, K=128, hc=P, gs=1.0: (P, P, P, P, M, H, K, 1.0, 1.0, 1.0, gs, hc, P,  # noqa: E731
                                                   NUL)
    assert f(*args(H=192)) == SHAPE                           # H % 128
    assert f(*args(H=0)) == SHAPE
    assert f(*args(K=96)) == SHAPE                            # K % 64
    assert f(*args(hc=NUL)) == INVALID
    assert f(*args(hc=P_MIS)) == ALIGN
    assert f(*args(gs=0.0)) == INVALID
    assert f(*args(gs=float("nan"))) == INVALID
    assert f(*args(M=0)) == 0


def test_kv_fp8_validation(lib):
    assert lib.nvfp4_kv_scale(ctypes.c_float(448.0)) == 1.0
    assert lib.nvfp4_kv_scale(ctypes.c_float(0.0)) == 1.0
    q = lib.nvfp4_kv_quantize_fp8
    assert q(NUL, 8, 1.0, P, NUL) == INVALID
    assert q(P, 12, 1.0, P, NUL) == SHAPE                     # n % 8
    assert q(P, -8, 1.0, P, NUL) == SHAPE
    assert q(P_MIS, 8, 1.0, P, NUL) == ALIGN
    assert q(P, 8, 1.0, P_MIS, NUL) == ALIGN
    assert q(P, 8, 0.0, P, NUL) == INVALID
    assert q(P, 0, 1.0, P, NUL) == 0


def test_misc_validation(lib):
    assert lib.nvfp4_set_gemm_path(5) == INVALID
    assert lib.nvfp4_set_gemm_path(0) == 0
    assert lib.nvfp4_set_wait_limit_ns(0) == INVALID
    assert lib.nvfp4_set_launch_overlap(2) == INVALID
    assert lib.nvfp4_set_launch_overlap(1) == 0
    assert lib.nvfp4_set_launch_overlap(0) == 0
    # back to the suite's default (NVFP4_TEST_LAUNCH_OVERLAP)
    lib.nvfp4_set_launch_overlap(1 if os.environ.get("NVFP4_TEST_LAUNCH_OVERLAP") == "1" else 0)
    assert lib.nvfp4_silu_mul(P, 4, 12, 24, P, 12, NUL) == SHAPE       # H % 8
    assert lib.nvfp4_amax(P, 4, 64, 64, NUL, NUL) == INVALID
    assert lib.nvfp4_test_e2m1(NUL, P, 4, NUL) == INVALID
