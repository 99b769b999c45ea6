"""GPU error paths: bounded waits return a status instead of hanging, the
context stays usable afterwards, and shape-path mismatches are rejected.

No test here faults, traps or hangs the GPU: the timeout test waits on an
mbarrier that nothing arrives on, with a short wait limit, and checks that
the kernel gives up and reports NVFP4_ERR_TIMEOUT.
"""
import numpy as np
import pytest
import torch

import nvfp4_w4a4_quantized_quantizer_b200 as nv
import workloads
from tests import _helpers as H

pytestmark = pytest.mark.gpu

TIMEOUT = -5


def test_bounded_wait_reports_timeout_and_context_survives():
    assert nv.nvfp4_last_device_error()[0] == 0
    st = nv.nvfp4_test_wait_timeout(2_000_000)       # 2 ms
    assert st == TIMEOUT
    assert nv.nvfp4_last_device_error()[0] == 0      # cleared by the read
    bits = workloads.random_bf16((16, 64), seed=1)
    c, s = nv.nvfp4_quantize_act(H.bf16_dev(bits), 0.01)
    torch.cuda.synchronize()
    assert c.shape == (16, 32)


def test_small_path_rejects_large_m():
    nv.nvfp4_set_gemm_path(2)
    try:
        z = torch.zeros(1024, dtype=torch.uint8, device="cuda")
        with pytest.raises(nv.NVFP4Error):
            nv.nvfp4_linear(z, z, 1.0, z, z, 1.0, 65, 16, 64)
    finally:
        nv.nvfp4_set_gemm_path(0)


def test_device_error_word_clear_after_normal_work():
    bits = workloads.random_bf16((130, 256), seed=2)
    c, s = nv.nvfp4_quantize_act(H.bf16_dev(bits), 0.05)
    wc, ws, (wg,) = nv.nvfp4_quantize_weight(H.bf16_dev(workloads.random_bf16((256, 256), seed=3)))
    nv.nvfp4_linear(c, s, 0.05, wc, ws, wg, 130, 256, 256)
    st, info = nv.nvfp4_last_device_error()
    assert st == 0 and info == 0
