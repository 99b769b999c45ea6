"""GPU parity: FP8 (E4M3) KV-cache quantisation vs the CPU oracle, bit for bit.

Every finite bf16 value under several calibrated scales (saturation past the
calibrated range and signed zeros included), and a KV-cache-shaped tensor
with its scale calibrated on a separate batch, as the pages' recipe ships
it (nefut abstract: calibrated FP8 KV-cache scales).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
import nvfp4_w4a4_quantized_quantizer_b200 as nv
from tests import _helpers as H

pytestmark = pytest.mark.gpu


def all_finite_bf16_bits():
    bits = np.arange(1 << 16, dtype=np.uint32)
    f = (bits << 16).view(np.float32)
    return bits[np.isfinite(f)].astype(np.uint16)        # 65280 values, a multiple of 8


@pytest.mark.parametrize("amax", [1.0, 448.0, 3.7, 1e-3, 6.5e4])
def test_every_bf16_value(amax):
    bits = all_finite_bf16_bits()
    s = float(nv.nvfp4_kv_scale(amax))
    assert np.float32(s) == oracle.kv_scale(amax)
    got = nv.nvfp4_kv_quantize_fp8(H.bf16_dev(bits), s).cpu().numpy()
    ref = oracle.kv_quantize(H.f32(bits), np.float32(s))
    np.testing.assert_array_equal(got, ref)


def test_kv_cache_tensor_with_a_calibrated_scale():
    # [tokens, kv heads, head dim] of one layer's K, heavy-tailed like activations
    shape = (4096, 8, 128)
    rng = np.random.default_rng(7)
    calib = rng.standard_t(3, size=(512,) + shape[1:]).astype(np.float32)
    live = rng.standard_t(3, size=shape).astype(np.float32)
    cb, lb = workloads.f32_to_bf16_bits(calib), workloads.f32_to_bf16_bits(live)
    amax = nv.nvfp4_amax(H.bf16_dev(cb.reshape(-1, 1024))).item()
    s = float(nv.nvfp4_kv_scale(amax))
    x = H.bf16_dev(lb.reshape(-1, 1024))
    out = torch.full((x.numel() + 64,), 0x55, dtype=torch.uint8, device="cuda")
    nv.nvfp4_kv_quantize_fp8(x, s, out=out[:x.numel()].view(x.shape))
    got = out.cpu().numpy()
    assert np.all(got[x.numel():] == 0x55)                   # nothing past n is written
    ref = oracle.kv_quantize(H.f32(lb).reshape(-1), np.float32(s))
    np.testing.assert_array_equal(got[:x.numel()], ref)
    assert nv.nvfp4_last_device_error()[0] == 0
