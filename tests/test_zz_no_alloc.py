"""nvfp4_quantize_weight_noalloc: weight quantisation for callers that cannot
allocate device memory (a runtime that owns all device memory and hands an
operator only its input and output buffers cannot create the workspace
nvfp4_quantize_weight takes).  Its scratch is a fixed array inside the
library.  Each call must give exactly what nvfp4_quantize_weight gives, and a
call must not see the previous call's scratch contents.

This file is collected last so that a run stopping at the first failure has
already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads
import nvfp4_w4a4_quantized_quantizer_b200 as nv
from nvfp4_w4a4_quantized_quantizer_b200 import _lib

pytestmark = pytest.mark.gpu

WIDTHS = [64, 32, 16, 48, 16, 80]
K = 320


def _weight(seed, scale):
    rows = [workloads.random_bf16((wd, K), seed=seed * 100 + i, std=scale * (i + 1) / np.sqrt(K))
            for i, wd in enumerate(WIDTHS)]
    bits = np.concatenate(rows)
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()


def _noalloc_via_abi(lib, w, offs):
    N = w.shape[0]
    codes = torch.empty((N, K // 2), dtype=torch.uint8, device="cuda")
    scales = torch.empty(nv.nvfp4_scale_bytes(N, K), dtype=torch.uint8, device="cuda")
    offs_c = (ctypes.c_int64 * len(offs))(*offs)
    gs_c = (ctypes.c_float * len(offs))()
    st = lib.nvfp4_quantize_weight_noalloc(
        ctypes.c_void_p(w.data_ptr()), N, K, w.stride(0), offs_c, len(offs), gs_c,
        ctypes.c_void_p(codes.data_ptr()), ctypes.c_void_p(scales.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, _lib.STATUS_NAMES.get(st, st)
    return codes, scales, [float(v) for v in gs_c]


def test_noalloc_matches_workspace_entry_point_on_consecutive_calls():
    lib = _lib.load()
    offs = np.cumsum([0] + WIDTHS[:-1]).tolist()
    # the second weight's amax is 16x smaller: scratch left over from the first
    # call would raise its global scales and change every code
    for seed, scale in ((1, 4.0), (2, 0.25)):
        w = _weight(seed, scale)
        ref_codes, ref_scales, ref_gs = nv.nvfp4_quantize_weight(w, seg_offsets=offs)
        codes, scales, gs = _noalloc_via_abi(lib, w, offs)
        torch.cuda.synchronize()
        assert gs == ref_gs
        assert torch.equal(codes, ref_codes)
        assert torch.equal(scales, ref_scales)


def test_noalloc_rejects_more_modules_than_its_scratch_holds():
    lib = _lib.load()
    n = lib.nvfp4_noalloc_max_segments() + 1   # the limit compiled into the library
    N = 16 * n
    w = torch.zeros((N, K), dtype=torch.bfloat16, device="cuda")
    offs_c = (ctypes.c_int64 * n)(*range(0, N, 16))
    gs_c = (ctypes.c_float * n)()
    dummy = torch.empty(16, dtype=torch.uint8, device="cuda")
    st = lib.nvfp4_quantize_weight_noalloc(
        ctypes.c_void_p(w.data_ptr()), N, K, K, offs_c, n, gs_c, ctypes.c_void_p(dummy.data_ptr()),
        ctypes.c_void_p(dummy.data_ptr()), ctypes.c_void_p(0))
    assert st == -1   # NVFP4_ERR_INVALID_ARG
