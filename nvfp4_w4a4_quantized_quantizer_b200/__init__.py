"""NVFP4 W4A4 linear layer on B200 (sm_100a): Python binding.

Thin marshalling over the C ABI of include/nvfp4.h (loaded from the in-tree
libnvfp4.so through ctypes).  Every step runs in the library's CUDA kernels;
torch is used only to own device memory and to name the current stream.
The functions keep the C names; tensors replace raw pointers, and outputs
that are not passed in are allocated with torch on the input's device.
"""
from __future__ import annotations

import ctypes
from typing import Optional, Sequence, Tuple

import torch

from . import _lib
from ._lib import (NVFP4Error, OP_GDN_DECAY, OP_NONE, OP_SIGMOID, OUT_BF16, OUT_FP32,  # noqa: F401
                   Segment, check, load)

__all__ = [
    "nvfp4_codes_bytes", "nvfp4_scale_bytes", "nvfp4_global_scale", "nvfp4_amax",
    "nvfp4_quantize_act", "nvfp4_quantize_weight", "nvfp4_quantize_weight_noalloc",
    "nvfp4_linear", "nvfp4_fused_linear", "nvfp4_gemm_workspace_bytes", "nvfp4_gemm_workspace",
    "nvfp4_gate_up_silu_quantize", "nvfp4_gdn_recurrence", "nvfp4_silu_mul", "nvfp4_last_device_error",
    "nvfp4_set_gemm_path", "nvfp4_set_launch_overlap", "nvfp4_kv_scale", "nvfp4_kv_quantize_fp8",
    "nvfp4_set_wait_limit_ns", "nvfp4_test_e2m1", "nvfp4_test_e4m3", "nvfp4_test_wait_timeout",
    "SegmentSpec", "NVFP4Error", "OP_NONE", "OP_SIGMOID", "OP_GDN_DECAY",
]


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _ptr(t: Optional[torch.Tensor]) -> ctypes.c_void_p:
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _ld(t: torch.Tensor) -> int:
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError("expected a 2-D row-major tensor")
    return t.stride(0)


def nvfp4_codes_bytes(rows: int, K: int) -> int:
    return load().nvfp4_codes_bytes(rows, K)


def nvfp4_scale_bytes(rows: int, K: int) -> int:
    return load().nvfp4_scale_bytes(rows, K)


def nvfp4_global_scale(amax: float) -> float:
    return load().nvfp4_global_scale(ctypes.c_float(amax))


def nvfp4_amax(x: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Device float tensor [1] holding max |x| of the bf16 matrix x."""
    if out is None:
        out = torch.empty(1, dtype=torch.float32, device=x.device)
    check(load().nvfp4_amax(_ptr(x), x.shape[0], x.shape[1], _ld(x), _ptr(out), _stream(stream)),
          "nvfp4_amax")
    return out


def nvfp4_quantize_act(x: torch.Tensor, a_gs: float, codes: Optional[torch.Tensor] = None,
                       scales: Optional[torch.Tensor] = None, stream=None
                       ) -> Tuple[torch.Tensor, torch.Tensor]:
    """bf16 [M, K] -> (codes uint8 [M, K/2], scales uint8 [scale_bytes]) under static a_gs."""
    M, K = x.shape
    if codes is None:
        codes = torch.empty((M, K // 2), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty(nvfp4_scale_bytes(M, K), dtype=torch.uint8, device=x.device)
    check(load().nvfp4_quantize_act(_ptr(x), M, K, _ld(x), ctypes.c_float(a_gs), _ptr(codes),
                                    _ptr(scales), _stream(stream)), "nvfp4_quantize_act")
    return codes, scales


def nvfp4_quantize_weight(w: torch.Tensor, seg_offsets: Optional[Sequence[int]] = None,
                          codes: Optional[torch.Tensor] = None,
                          scales: Optional[torch.Tensor] = None,
                          workspace: Optional[torch.Tensor] = None, stream=None):
    """bf16 W [N, K] -> (codes, scales, [w_gs per module]).  Synchronises the stream."""
    lib = load()
    N, K = w.shape
    offs = list(seg_offsets) if seg_offsets is not None else [0]
    nseg = len(offs)
    if codes is None:
        codes = torch.empty((N, K // 2), dtype=torch.uint8, device=w.device)
    if scales is None:
        scales = torch.empty(nvfp4_scale_bytes(N, K), dtype=torch.uint8, device=w.device)
    if workspace is None:
        workspace = torch.empty(lib.nvfp4_quantize_weight_workspace_bytes(nseg), dtype=torch.uint8,
                                device=w.device)
    offs_c = (ctypes.c_int64 * nseg)(*offs)
    gs_c = (ctypes.c_float * nseg)()
    check(lib.nvfp4_quantize_weight(_ptr(w), N, K, _ld(w), offs_c, nseg, gs_c, _ptr(codes),
                                    _ptr(scales), _ptr(workspace), _stream(stream)),
          "nvfp4_quantize_weight")
    return codes, scales, [float(v) for v in gs_c]


def nvfp4_quantize_weight_noalloc(w: torch.Tensor, seg_offsets: Optional[Sequence[int]] = None,
                                  codes: Optional[torch.Tensor] = None,
                                  scales: Optional[torch.Tensor] = None, stream=None):
    """nvfp4_quantize_weight for callers that cannot allocate device memory: no
    workspace; the library's fixed scratch array holds the per-module amax.
    (This wrapper allocates outputs only when they are not passed in.)"""
    lib = load()
    N, K = w.shape
    offs = list(seg_offsets) if seg_offsets is not None else [0]
    nseg = len(offs)
    if codes is None:
        codes = torch.empty((N, K // 2), dtype=torch.uint8, device=w.device)
    if scales is None:
        scales = torch.empty(nvfp4_scale_bytes(N, K), dtype=torch.uint8, device=w.device)
    offs_c = (ctypes.c_int64 * nseg)(*offs)
    gs_c = (ctypes.c_float * nseg)()
    check(lib.nvfp4_quantize_weight_noalloc(_ptr(w), N, K, _ld(w), offs_c, nseg, gs_c, _ptr(codes),
                                            _ptr(scales), _stream(stream)),
          "nvfp4_quantize_weight_noalloc")
    return codes, scales, [float(v) for v in gs_c]


class SegmentSpec:
    """One module of a fused projection (mirror of nvfp4_segment)."""

    def __init__(self, n_offset: int, w_gs: float, a_gs: float, op: int = OP_NONE,
                 a_log: Optional[torch.Tensor] = None, dt_bias: Optional[torch.Tensor] = None):
        self.n_offset, self.w_gs, self.a_gs, self.op = n_offset, w_gs, a_gs, op
        self.a_log, self.dt_bias = a_log, dt_bias

    def c(self) -> Segment:
        return Segment(self.n_offset, self.w_gs, self.a_gs, self.op,
                       self.a_log.data_ptr() if self.a_log is not None else None,
                       self.dt_bias.data_ptr() if self.dt_bias is not None else None)


def _out(y, M, N, dtype, device):
    if y is None:
        y = torch.empty((M, N), dtype=torch.float32 if dtype == OUT_FP32 else torch.bfloat16,
                        device=device)
    return y


def nvfp4_linear(a_codes, a_scales, a_gs: float, w_codes, w_scales, w_gs: float, M: int, N: int,
                 K: int, y: Optional[torch.Tensor] = None, out_dtype: int = OUT_BF16,
                 stream=None) -> torch.Tensor:
    y = _out(y, M, N, out_dtype, a_codes.device)
    check(load().nvfp4_linear(_ptr(a_codes), _ptr(a_scales), ctypes.c_float(a_gs), _ptr(w_codes),
                              _ptr(w_scales), ctypes.c_float(w_gs), M, N, K, _ptr(y), _ld(y),
                              out_dtype, _stream(stream)), "nvfp4_linear")
    return y


def nvfp4_gemm_workspace_bytes() -> int:
    return load().nvfp4_gemm_workspace_bytes()


def nvfp4_gemm_workspace(device=None) -> torch.Tensor:
    """A zeroed workspace of nvfp4_gemm_workspace_bytes() for nvfp4_fused_linear."""
    return torch.zeros(nvfp4_gemm_workspace_bytes(), dtype=torch.uint8, device=device)


def nvfp4_fused_linear(a_codes, a_scales, w_codes, w_scales, M: int, N: int, K: int,
                       segments: Sequence[SegmentSpec], y: Optional[torch.Tensor] = None,
                       out_dtype: int = OUT_BF16, stream=None,
                       workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """With `workspace` (see nvfp4_gemm_workspace) the call is
    nvfp4_fused_linear_ws, which splits the last partial wave along K."""
    y = _out(y, M, N, out_dtype, a_codes.device)
    segs = (Segment * len(segments))(*[s.c() for s in segments])
    if workspace is None:
        check(load().nvfp4_fused_linear(_ptr(a_codes), _ptr(a_scales), _ptr(w_codes),
                                        _ptr(w_scales), M, N, K, segs, len(segments), _ptr(y),
                                        _ld(y), out_dtype, _stream(stream)), "nvfp4_fused_linear")
    else:
        check(load().nvfp4_fused_linear_ws(_ptr(a_codes), _ptr(a_scales), _ptr(w_codes),
                                           _ptr(w_scales), M, N, K, segs, len(segments), _ptr(y),
                                           _ld(y), out_dtype, _ptr(workspace),
                                           workspace.numel() * workspace.element_size(),
                                           _stream(stream)), "nvfp4_fused_linear_ws")
    return y


def nvfp4_gate_up_silu_quantize(a_codes, a_scales, w_codes, w_scales, M: int, H: int, K: int,
                                a_gs: float, w_gs_gate: float, w_gs_up: float, h_gs: float,
                                h_codes: Optional[torch.Tensor] = None,
                                h_scales: Optional[torch.Tensor] = None,
                                stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    dev = a_codes.device
    if h_codes is None:
        h_codes = torch.empty((M, H // 2), dtype=torch.uint8, device=dev)
    if h_scales is None:
        h_scales = torch.empty(nvfp4_scale_bytes(M, H), dtype=torch.uint8, device=dev)
    check(load().nvfp4_gate_up_silu_quantize(
        _ptr(a_codes), _ptr(a_scales), _ptr(w_codes), _ptr(w_scales), M, H, K,
        ctypes.c_float(a_gs), ctypes.c_float(w_gs_gate), ctypes.c_float(w_gs_up),
        ctypes.c_float(h_gs), _ptr(h_codes), _ptr(h_scales), _stream(stream)),
        "nvfp4_gate_up_silu_quantize")
    return h_codes, h_scales


def nvfp4_kv_scale(amax: float) -> float:
    return load().nvfp4_kv_scale(ctypes.c_float(amax))


def nvfp4_kv_quantize_fp8(x: torch.Tensor, scale: float, out: Optional[torch.Tensor] = None,
                          stream=None) -> torch.Tensor:
    """bf16 tensor (contiguous, numel % 8 == 0) -> E4M3 codes (uint8, same shape)."""
    if not x.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    if out is None:
        out = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    check(load().nvfp4_kv_quantize_fp8(_ptr(x), x.numel(), ctypes.c_float(scale), _ptr(out),
                                       _stream(stream)), "nvfp4_kv_quantize_fp8")
    return out


def nvfp4_gdn_recurrence(q, k, v, g, beta, group: int = 1, state: Optional[torch.Tensor] = None,
                         o: Optional[torch.Tensor] = None, stream=None):
    """Gated delta rule over one sequence: q, k [T, Hk, 128], v [T, Hv, 128], g and beta
    [T, Hv] (fp32, contiguous).  Returns (o [T, Hv, 128], final state [Hv, 128, 128]);
    `state` (initial state, updated in place) defaults to zeros."""
    T, Hv, D = v.shape
    for t in (q, k, v, g, beta):
        if t.dtype != torch.float32 or not t.is_contiguous():
            raise ValueError("expected contiguous float32 tensors")
    if state is None:
        state = torch.zeros((Hv, D, D), dtype=torch.float32, device=v.device)
    if o is None:
        o = torch.empty((T, Hv, D), dtype=torch.float32, device=v.device)
    check(load().nvfp4_gdn_recurrence(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), T, Hv, group,
                                      D, _ptr(o), _ptr(state), _stream(stream)),
          "nvfp4_gdn_recurrence")
    return o, state


def nvfp4_silu_mul(gu: torch.Tensor, H: int, h: Optional[torch.Tensor] = None,
                   stream=None) -> torch.Tensor:
    M = gu.shape[0]
    if h is None:
        h = torch.empty((M, H), dtype=torch.bfloat16, device=gu.device)
    check(load().nvfp4_silu_mul(_ptr(gu), M, H, _ld(gu), _ptr(h), _ld(h), _stream(stream)),
          "nvfp4_silu_mul")
    return h


def nvfp4_last_device_error(stream=None) -> Tuple[int, int]:
    info = ctypes.c_uint64(0)
    st = load().nvfp4_last_device_error(_stream(stream), ctypes.byref(info))
    return st, info.value


def nvfp4_set_gemm_path(path: int) -> None:
    check(load().nvfp4_set_gemm_path(path), "nvfp4_set_gemm_path")


def nvfp4_set_launch_overlap(on: bool) -> None:
    check(load().nvfp4_set_launch_overlap(1 if on else 0), "nvfp4_set_launch_overlap")


def nvfp4_set_wait_limit_ns(limit_ns: int) -> None:
    check(load().nvfp4_set_wait_limit_ns(limit_ns), "nvfp4_set_wait_limit_ns")


def nvfp4_test_e2m1(v: torch.Tensor, stream=None) -> torch.Tensor:
    out = torch.empty(v.numel(), dtype=torch.uint8, device=v.device)
    check(load().nvfp4_test_e2m1(_ptr(v), _ptr(out), v.numel(), _stream(stream)), "nvfp4_test_e2m1")
    return out


def nvfp4_test_e4m3(v: torch.Tensor, stream=None) -> torch.Tensor:
    out = torch.empty(v.numel(), dtype=torch.uint8, device=v.device)
    check(load().nvfp4_test_e4m3(_ptr(v), _ptr(out), v.numel(), _stream(stream)), "nvfp4_test_e4m3")
    return out


def nvfp4_test_wait_timeout(limit_ns: int, stream=None) -> int:
    return load().nvfp4_test_wait_timeout(limit_ns, _stream(stream))
