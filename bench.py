"""Benchmark of the NVFP4 W4A4 linear layer on B200.

One step = one pass of the layer's hot path over one batch: quantise the bf16
activations (E2M1 codes + E4M3 block scales under the static global scale)
and run the block-scaled FP4 GEMM with the segment epilogue, bf16 output.
Default workload: the single prefill projection M=4096, K=5120, N=5120
(activations Student-t(3)/sqrt(3) with 8 outlier channels x100, weights
N(0, 1/sqrt(K)), static activation scale calibrated on a 512-row batch).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                    [--workload prefill|gdn_inproj|mlp|decode]

--workload mlp times the MLP pair as one step (quantise, gate_up with two
modules, SiLU(gate)*up, requantise, down GEMM); its roofline line is the
gate_up GEMM, the down GEMM and the glue kernels are reported beside it.

Prints one JSON line on rank 0.  Multi-GPU runs (torchrun, one rank per GPU)
are weak-scaled replicas: every rank runs the same layer on its own batch, no
collective touches the data path; the step time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "NVFP4 W4A4 linear TFLOPS & % of B200 FP4 peak; small-M weight GB/s"
FP4_PER_BF16 = 4.0          # nominal dense FP4 / BF16 tensor throughput ratio (9 / 2.25 PFLOP/s)
ROTATE_ACT = 6              # distinct activation buffers (each step uses the next one)
ROTATE_W = 4                # distinct weight copies
# The CTA-pair GEMM's stream-K tail (nvfp4_fused_linear_ws) is correct but
# measured slower than whole tiles on every large configuration here
# (prefill 60.0 vs 56.9 us, GDN in-projection 327 vs 323 us, interleaved
# runs): the main loop is bound by L2 -> shared-memory delivery for the whole
# chip, so the pairs of a partial last wave run their tiles faster, and the
# stream-K partial tiles add traffic.  The bench launches without it.
SPLIT_TAIL = False


# --------------------------------------------------------------- plumbing
def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sus=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, source="fallback")


class ClockSampler:
    """nvidia-smi clock / throttle samples taken while the timed region runs."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or self.path is None:
            return None
        rows = []
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) >= 9:
                try:
                    rows.append((float(f[1]), float(f[2]), float(f[3]), f[5], f[6], f[7], f[8]))
                except ValueError:
                    pass
        os.unlink(self.path)
        if not rows:
            return None
        loaded = [r for r in rows if r[2] > 300.0] or rows
        reasons = set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for r in loaded:
            for name, v in zip(names, r[3:]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": rows[0][1],
                "power_w_max": max(r[2] for r in rows), "samples": len(loaded),
                "reasons": sorted(reasons)}


def _code_only(text: str) -> str:
    """C/C++ source with comments and blank lines removed (string literals kept)."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c == '"' or c == "'":
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            i = text.find("\n", i)
            i = n if i < 0 else i
        elif text.startswith("/*", i):
            i = text.find("*/", i + 2)
            i = n if i < 0 else i + 2
        else:
            out.append(c)
            i += 1
    lines = (ln.rstrip() for ln in "".join(out).splitlines())
    return "\n".join(ln for ln in lines if ln.strip())


def source_digest():
    """Digest of the kernel sources' code (comments do not count): a profile's
    counters apply while this matches the digest recorded with them."""
    h = hashlib.sha256()
    for f in ("ptx.cuh", "gemm.cuh", "quantize.cuh", "gdn.cuh", "api.cu"):
        text = open(os.path.join(ROOT, "nvfp4_w4a4_quantized_quantizer_b200", "csrc", f)).read()
        h.update(_code_only(text).encode())
    return h.hexdigest()[:16]


def ncu_traffic(name: str):
    """dram bytes per launch from the committed ncu summary, if it matches the current source."""
    p = os.path.join(ROOT, "profiles", name)
    if not os.path.exists(p):
        return None
    text = open(p).read()
    m = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
    d = re.search(r"source_digest:\s*([0-9a-f]+)", text)
    if m and d and d.group(1) == source_digest():
        return float(m.group(1))
    return None


# ------------------------------------------------------------ multi-rank
# N > 1: one process per GPU, each a replica of the whole layer on its own
# tokens (weak scaling, no data-path collective); the timed region is
# bracketed by a barrier and a device synchronisation on both sides and the
# reported time is the maximum over ranks.
def timed_region(pg, fn, sync):
    """Barrier + sync, fn() (returns device ms), sync + barrier."""
    if pg is not None:
        pg.barrier()
    sync()
    ms = fn()
    sync()
    if pg is not None:
        pg.barrier()
    return ms


def max_over_ranks(value: float, pg, device) -> float:
    t = torch.tensor([value], dtype=torch.float64, device=device)
    if pg is not None:
        pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def job_value(world: int, flops_per_step: float, ms_step: float) -> float:
    """Whole-job TFLOP/s: every rank runs one step of the workload per step time."""
    return world * flops_per_step / (ms_step * 1e-3) / 1e12


# ------------------------------------------------------------- workloads
def _dev_bf16(bits, device):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


class Layer:
    """Device-resident operands of one workload, with rotated copies."""

    def __init__(self, wl: workloads.Workload, M: int, device, rotate_act=ROTATE_ACT,
                 rotate_w=ROTATE_W):
        import nvfp4_w4a4_quantized_quantizer_b200 as nv
        self.nv, self.wl, self.M, self.N, self.K = nv, wl, M, wl.N, wl.K
        calib = _dev_bf16(workloads.activations(wl, calib=True), device)
        self.a_gs = nv.nvfp4_global_scale(nv.nvfp4_amax(calib).item())
        self.x_host = workloads.activations(wl, M=M)
        x = _dev_bf16(self.x_host, device)
        self.xs = [x] + [x.clone() for _ in range(rotate_act - 1)]
        wbits = _dev_bf16(workloads.weights(wl), device)
        wc, ws, self.w_gs = nv.nvfp4_quantize_weight(wbits, seg_offsets=wl.seg_offsets)
        del wbits
        self.ws = [(wc, ws)] + [(wc.clone(), ws.clone()) for _ in range(rotate_w - 1)]
        self.codes = [torch.empty((M, self.K // 2), dtype=torch.uint8, device=device) for _ in range(2)]
        self.scales = [torch.empty(nv.nvfp4_scale_bytes(M, self.K), dtype=torch.uint8, device=device)
                       for _ in range(2)]
        self.ys = [torch.empty((M, self.N), dtype=torch.bfloat16, device=device) for _ in range(2)]
        # lets the CTA-pair GEMM split its last partial wave of tiles along K
        self.work = nv.nvfp4_gemm_workspace(device)
        self.segs = []
        gate_dev = {}
        if any(s.op == "gdn_decay" for s in wl.segments):
            a_log, dt = workloads.gate_params(wl)
            gate_dev = dict(a_log=torch.from_numpy(a_log).to(device), dt=torch.from_numpy(dt).to(device))
        for s, off, g in zip(wl.segments, wl.seg_offsets, self.w_gs):
            op = {"none": nv.OP_NONE, "sigmoid": nv.OP_SIGMOID, "gdn_decay": nv.OP_GDN_DECAY}[s.op]
            self.segs.append(nv.SegmentSpec(off, g, self.a_gs, op,
                                            gate_dev.get("a_log") if op == nv.OP_GDN_DECAY else None,
                                            gate_dev.get("dt") if op == nv.OP_GDN_DECAY else None))

    def quantize(self, i, stream, x=None):
        xx = self.xs[i % len(self.xs)] if x is None else x
        self.nv.nvfp4_quantize_act(xx, self.a_gs, codes=self.codes[i % 2], scales=self.scales[i % 2],
                                   stream=stream)

    def gemm(self, i, stream):
        wc, ws = self.ws[i % len(self.ws)]
        self.nv.nvfp4_fused_linear(self.codes[i % 2], self.scales[i % 2], wc, ws, self.M, self.N,
                                   self.K, self.segs, y=self.ys[i % 2], stream=stream,
                                   workspace=self.work if SPLIT_TAIL else None)

    @property
    def flops(self):
        return 2.0 * self.M * self.N * self.K

    @property
    def weight_bytes(self):
        return self.N * self.K // 2 + self.nv.nvfp4_scale_bytes(self.N, self.K)


class MlpChain:
    """The MLP pair as one step: quantise x; gate_up (two modules) with
    h = bf16(SiLU(gate) * up) requantised under its calibrated global scale in
    the same kernel; down GEMM.  Activation copies rotate over 3, weight sets
    over 2 (working set > L2)."""

    def __init__(self, device, rotate_act=3, rotate_w=2):
        import nvfp4_w4a4_quantized_quantizer_b200 as nv
        wl = workloads.WORKLOADS[4]
        self.nv, self.wl = nv, wl
        self.M, self.K, self.N = wl.M, wl.K, wl.N
        self.H, self.N2 = wl.N // 2, workloads.MLP_DOWN_N
        assert workloads.MLP_DOWN_K == self.H
        calib = _dev_bf16(workloads.activations(wl, calib=True), device)
        self.a_gs = nv.nvfp4_global_scale(nv.nvfp4_amax(calib).item())
        self.x_host = workloads.activations(wl)
        x = _dev_bf16(self.x_host, device)
        self.xs = [x] + [x.clone() for _ in range(rotate_act - 1)]
        wbits = _dev_bf16(workloads.weights(wl), device)
        wc, ws, self.w_gs = nv.nvfp4_quantize_weight(wbits, seg_offsets=wl.seg_offsets)
        del wbits
        w2bits = _dev_bf16(workloads.down_weights(), device)
        w2c, w2s, (self.w2_gs,) = nv.nvfp4_quantize_weight(w2bits)
        del w2bits
        self.segs = [nv.SegmentSpec(off, g, self.a_gs) for off, g in zip(wl.seg_offsets, self.w_gs)]
        self.work = nv.nvfp4_gemm_workspace(device)
        # the down input's static global scale: the chain on the calibration batch
        cc, cs = nv.nvfp4_quantize_act(calib, self.a_gs)
        gu_cal = nv.nvfp4_fused_linear(cc, cs, wc, ws, calib.shape[0], self.N, self.K, self.segs)
        h_cal = nv.nvfp4_silu_mul(gu_cal, self.H)
        self.a2_gs = nv.nvfp4_global_scale(nv.nvfp4_amax(h_cal).item())
        self.segs2 = [nv.SegmentSpec(0, self.w2_gs, self.a2_gs)]
        del calib, cc, cs, gu_cal, h_cal
        self.ws = [(wc, ws, w2c, w2s)] + [tuple(t.clone() for t in (wc, ws, w2c, w2s))
                                          for _ in range(rotate_w - 1)]
        self.xc = torch.empty((self.M, self.K // 2), dtype=torch.uint8, device=device)
        self.xsc = torch.empty(nv.nvfp4_scale_bytes(self.M, self.K), dtype=torch.uint8, device=device)
        self.hc = torch.empty((self.M, self.H // 2), dtype=torch.uint8, device=device)
        self.hsc = torch.empty(nv.nvfp4_scale_bytes(self.M, self.H), dtype=torch.uint8, device=device)
        # two output buffers: a step's read-back may overlap the next step's kernels
        self.ys = [torch.empty((self.M, self.N2), dtype=torch.bfloat16, device=device)
                   for _ in range(2)]

    def quantize(self, i, stream, x=None):
        xx = self.xs[i % len(self.xs)] if x is None else x
        self.nv.nvfp4_quantize_act(xx, self.a_gs, codes=self.xc, scales=self.xsc, stream=stream)

    def gate_up(self, i, stream):
        """gate_up GEMM + SiLU(gate) * up + requantisation of h, one kernel."""
        wc, ws, _, _ = self.ws[i % len(self.ws)]
        self.nv.nvfp4_gate_up_silu_quantize(self.xc, self.xsc, wc, ws, self.M, self.H, self.K,
                                            self.a_gs, self.w_gs[0], self.w_gs[1], self.a2_gs,
                                            h_codes=self.hc, h_scales=self.hsc, stream=stream)

    def down(self, i, stream):
        _, _, w2c, w2s = self.ws[i % len(self.ws)]
        self.nv.nvfp4_fused_linear(self.hc, self.hsc, w2c, w2s, self.M, self.N2, self.H, self.segs2,
                                   y=self.ys[i % 2], stream=stream,
                                   workspace=self.work if SPLIT_TAIL else None)

    def gemm(self, i, stream):
        """Everything after the first quantisation."""
        self.gate_up(i, stream)
        self.down(i, stream)

    launches_per_step = 3

    @property
    def flops(self):
        return 2.0 * self.M * self.K * self.N + 2.0 * self.M * self.H * self.N2


# Steps are replayed from CUDA graphs: a host call of the library costs more
# than some of its kernels (the quantiser, the decode GEMM), so launches
# issued one by one from Python would leave the GPU idle between kernels and
# the events would time the host.  A graph of GRAPH_STEPS steps covers the
# activation (6), weight (4) and output (2) rotations exactly.
GRAPH_STEPS = 12


def capture(fn, start: int, count: int, stream):
    """CUDA graph of fn(i, stream) for i in [start, start + count)."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(start, start + count):
            fn(i, stream)
    return g


def replay_ms(graphs, stream):
    """Device time of replaying `graphs` in order on `stream` (events on the stream)."""
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        a.record(stream)
        for g in graphs:
            g.replay()
        b.record(stream)
    b.synchronize()
    return a.elapsed_time(b)


def time_steps(layer: Layer, steps: int, warmup: int, stream):
    """Device time of exactly `steps` steps (quantise + GEMM), replayed from graphs."""
    def step(i, st):
        layer.quantize(i, st)
        layer.gemm(i, st)
    for i in range(warmup):
        step(i, stream)
    torch.cuda.synchronize()
    full = capture(step, 0, GRAPH_STEPS, stream)
    tail = capture(step, 0, steps % GRAPH_STEPS, stream) if steps % GRAPH_STEPS else None
    replay_ms([full], stream)                               # first replay uploads the graph
    seq = [full] * (steps // GRAPH_STEPS) + ([tail] if tail is not None else [])
    return replay_ms(seq, stream)


MIN_KERNEL_S = 0.2          # every per-kernel figure is averaged over at least this much device time


def time_each(fns, stream, min_s: float = MIN_KERNEL_S):
    """Mean device time (ms) of each named launch alone: a graph of
    GRAPH_STEPS launches of it, replayed until at least `min_s` seconds of
    device time are covered (the replay count is sized from a first replay)."""
    graphs = {name: capture(fn, 0, GRAPH_STEPS, stream) for name, fn in fns.items()}
    out = {}
    for name, g in graphs.items():
        first = replay_ms([g], stream)                      # uploads the graph
        reps = max(2, int(np.ceil(min_s * 1e3 / max(first, 1e-3))))
        out[name] = replay_ms([g] * reps, stream) / (reps * GRAPH_STEPS)
    return out


def e2e(layer: Layer, steps: int, warmup: int, stream):
    """Same metric through the public API from pinned host buffers: every
    step copies its activations in (H2D), quantises, runs the GEMM and reads
    its bf16 output back (D2H).  Steps are pipelined as a serving loop would
    run them: the copy-in of step i+1 and the copy-out of step i-1 overlap
    step i's kernels (three streams, double-buffered device input and output,
    events order each buffer's reuse); the timed region spans the first
    copy-in to the last copy-out."""
    dev = layer.xs[0].device
    xh = torch.from_numpy(layer.x_host.view(np.int16)).view(torch.bfloat16).pin_memory()
    yh = [torch.empty(tuple(layer.ys[0].shape), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    xd = [torch.empty_like(layer.xs[0]) for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()  # noqa: E731
    in_done, cmp_done, out_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    for e in cmp_done + out_done:
        e.record(stream)            # "done" before the first use of each buffer

    def one(i):
        j = i % 2
        with torch.cuda.stream(s_in):
            s_in.wait_event(cmp_done[j])            # step i-2's kernels are done with xd[j]
            xd[j].copy_(xh, non_blocking=True)
            in_done[j].record(s_in)
        with torch.cuda.stream(stream):
            stream.wait_event(in_done[j])
            stream.wait_event(out_done[j])          # step i-2's copy-out has read ys[j]
            layer.quantize(i, stream, x=xd[j])
            layer.gemm(i, stream)
            cmp_done[j].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(cmp_done[j])
            yh[j].copy_(layer.ys[i % 2], non_blocking=True)
            out_done[j].record(s_out)

    for i in range(warmup):
        one(i)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(s_in)
    for i in range(warmup, warmup + steps):
        one(i)
    s_out.wait_event(cmp_done[(warmup + steps - 1) % 2])
    b.record(s_out)
    b.synchronize()
    ms = a.elapsed_time(b) / steps
    return ms, xh.numel() * 2, yh[0].numel() * 2


def small_m_sweep(device, stream, warmup=10):
    """Decode-shaped sweep on the fused GDN in-projection weights: weight-stream
    GB/s of the GEMM alone (graph replays over the rotated weight copies)."""
    import nvfp4_w4a4_quantized_quantizer_b200 as nv
    wl = workloads.WORKLOADS[5]
    out = {}
    base = Layer(wl, 64, device, rotate_act=1, rotate_w=ROTATE_W)
    for M in wl.m_sweep:
        x = base.xs[0][:M]
        c, s = nv.nvfp4_quantize_act(x, base.a_gs, stream=stream)
        y = torch.empty((M, base.N), dtype=torch.bfloat16, device=device)

        def run(i):
            wc, ws = base.ws[i % len(base.ws)]
            nv.nvfp4_quantize_act(x, base.a_gs, codes=c, scales=s, stream=stream)
            nv.nvfp4_fused_linear(c, s, wc, ws, M, base.N, base.K, base.segs, y=y, stream=stream)

        for i in range(warmup):
            run(i)
        torch.cuda.synchronize()

        def gemm(i, st):
            wc, ws = base.ws[i % len(base.ws)]
            nv.nvfp4_fused_linear(c, s, wc, ws, M, base.N, base.K, base.segs, y=y, stream=st)
        g_ms = time_each({"gemm": gemm}, stream)["gemm"]
        out[f"M={M}"] = {"gemm_us": round(g_ms * 1e3, 2),
                         "weight_GBps": round(base.weight_bytes / (g_ms * 1e-3) / 1e9, 1),
                         "tokens_per_s": round(M / (g_ms * 1e-3), 1)}
    return out


# ------------------------------------------------------------ CPU oracle
def kv_fp8_rate(device, stream):
    """FP8 KV-cache quantisation of one layer's K (32768 tokens x 8 heads x
    128 dims, bf16 -> E4M3 under a calibrated scale), rotated over 3 copies
    (201 MB > L2): graph replay of GRAPH_STEPS launches.  3 bytes per element."""
    import nvfp4_w4a4_quantized_quantizer_b200 as nv
    n = 32768 * 8 * 128
    rng = np.random.default_rng(3)
    x0 = torch.from_numpy(rng.standard_normal(n).astype(np.float32)).to(device).to(torch.bfloat16)
    xs = [x0] + [x0.clone() for _ in range(2)]
    out = torch.empty(n, dtype=torch.uint8, device=device)
    s = nv.nvfp4_kv_scale(float(x0.float().abs().max().item()))

    def run(i, st):
        nv.nvfp4_kv_quantize_fp8(xs[i % 3], s, out=out, stream=st)

    t = time_each({"kv": run}, stream)["kv"]
    gbs = 3.0 * n / (t * 1e-3) / 1e9
    return {"elements": n, "us": round(t * 1e3, 2), "GBps": round(gbs, 1)}


# fp32 FMA peak for ALU-bound kernels: 148 SMs x 128 fp32 lanes x 2 FLOP x 1.965 GHz
FP32_ALU_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


GDN_T, GDN_HV, GDN_GROUP, GDN_D = 8192, 48, 3, 128


def gdn_problem(device):
    """Inputs of the gated delta rule over 8192 tokens of the GDN
    in-projection's heads (48 value heads over 16 key heads, width 128) and
    a launch function fn(i, stream)."""
    import nvfp4_w4a4_quantized_quantizer_b200 as nv
    T, Hv, group, D = GDN_T, GDN_HV, GDN_GROUP, GDN_D
    rng = np.random.default_rng(4)
    f = lambda a: torch.from_numpy(a.astype(np.float32)).to(device)  # noqa: E731
    k = rng.standard_normal((T, Hv // group, D))
    ins = dict(q=f(rng.standard_normal((T, Hv // group, D))),
               k=f(k / np.linalg.norm(k, axis=2, keepdims=True)),
               v=f(rng.standard_normal((T, Hv, D))),
               g=f(-np.log1p(np.exp(rng.normal(-2, 1, (T, Hv))))),
               beta=f(1 / (1 + np.exp(-rng.normal(0, 1.5, (T, Hv))))))
    state = torch.zeros((Hv, D, D), dtype=torch.float32, device=device)
    o = torch.empty((T, Hv, D), dtype=torch.float32, device=device)

    def run(i, st):
        nv.nvfp4_gdn_recurrence(ins["q"], ins["k"], ins["v"], ins["g"], ins["beta"], group=group,
                                state=state, o=o, stream=st)
    return run


def gdn_rate(device, stream):
    """The gated delta rule (gdn_problem), graph replay.  FLOPs counted as
    the definition's 6 D^2 per token and value head."""
    T, Hv, D = GDN_T, GDN_HV, GDN_D
    run = gdn_problem(device)
    t = time_each({"gdn": run}, stream)["gdn"]
    tflops = 6.0 * D * D * T * Hv / (t * 1e-3) / 1e12
    return {"tokens": T, "value_heads": Hv, "us": round(t * 1e3, 1),
            "tokens_per_s": round(T / (t * 1e-3), 1), "tflops": round(tflops, 2),
            "bound": "alu", "peak_tflops": round(FP32_ALU_PEAK_TFLOPS, 1),
            "frac": round(tflops / FP32_ALU_PEAK_TFLOPS, 4)}


def _threads():
    try:
        from threadpoolctl import threadpool_info
        return max([p.get("num_threads", 1) for p in threadpool_info()] or [1])
    except Exception:  # pragma: no cover
        return os.cpu_count()


class OracleSample:
    """The oracle, as it stands, on bounded row samples of a workload.  One
    step = the layer's path for `rows` activation rows: the oracle quantiser,
    then dequantisation and the float64 GEMM against the weights (quantised
    and dequantised once, outside the timing).  For the MLP pair the step is
    quantise x -> gate_up -> SiLU(gate) * up -> quantise h -> down.  The
    quantiser phases and the GEMM phases (dequantise + float64 product) are
    timed separately."""

    def __init__(self, wl: workloads.Workload):
        import oracle
        self.oracle, self.wl = oracle, wl
        self.mlp = wl.name.startswith("mlp")
        f32 = workloads.bf16_bits_to_f32
        calib = f32(workloads.activations(wl, calib=True))
        self.a_gs = oracle.global_scale(np.abs(calib).max())
        self.what = self._dequantized_weights(f32(workloads.weights(wl)), wl.seg_offsets, wl.N)
        if self.mlp:
            self.H, self.N2 = wl.N // 2, workloads.MLP_DOWN_N
            w2 = f32(workloads.down_weights())
            self.w2hat = self._dequantized_weights(w2, [0], self.N2)
            del w2
            # the down input's static scale: the oracle chain on the calibration batch
            h = self._silu(self._gemm(calib, self.a_gs, self.what))
            self.a2_gs = oracle.global_scale(np.abs(h).max())
        self.x = f32(workloads.activations(wl, rows=(0, min(256, wl.M))))
        self.threads = _threads()

    def _dequantized_weights(self, wf, offs, N):
        out = np.empty(wf.shape, np.float64)
        ends = list(offs[1:]) + [N]
        for o, e in zip(offs, ends):
            gs = self.oracle.global_scale(np.abs(wf[o:e]).max())
            q, sc = self.oracle.quantize(wf[o:e], gs)
            out[o:e] = self.oracle.dequantize(q, sc, gs)
        return out

    def _gemm(self, x, gs, what):
        q, sc = self.oracle.quantize(x, gs)
        return self.oracle.linear64(self.oracle.dequantize(q, sc, gs), what)

    def _silu(self, gu):
        return self.oracle.silu_mul_bf16(gu[:, :self.H], gu[:, self.H:])

    def run(self, rows: int):
        """One step; returns (quantiser seconds, GEMM seconds)."""
        o, tq, tg = self.oracle, 0.0, 0.0
        t0 = time.perf_counter()
        q, sc = o.quantize(self.x[:rows], self.a_gs)
        t1 = time.perf_counter()
        y = o.linear64(o.dequantize(q, sc, self.a_gs), self.what)
        t2 = time.perf_counter()
        tq, tg = t1 - t0, t2 - t1
        if self.mlp:
            h = self._silu(y)
            t3 = time.perf_counter()
            q2, s2 = o.quantize(h, self.a2_gs)
            t4 = time.perf_counter()
            o.linear64(o.dequantize(q2, s2, self.a2_gs), self.w2hat)
            t5 = time.perf_counter()
            tq += t4 - t2            # SiLU * up + requantisation: the MLP glue
            tg += t5 - t4
        return tq, tg

    def flops(self, rows: int) -> float:
        f = 2.0 * rows * self.wl.N * self.wl.K
        return f + (2.0 * rows * self.H * self.N2 if self.mlp else 0.0)

    def quant_bytes(self, rows: int) -> float:
        """Algorithmic bytes of the step's quantiser phases (2.5625 B per element)."""
        return 2.5625 * rows * (self.wl.K + (self.H if self.mlp else 0))

    def describe(self, rows: int, reps: int, el: float) -> str:
        what = ("quantise x, dequantise + float64 gate_up GEMM, SiLU(gate)*up, quantise h, "
                "dequantise + float64 down GEMM" if self.mlp else
                "quantise, dequantise + float64 GEMM")
        return (f"{rows} activation rows per step of {self.wl.name} (full K and N): oracle {what}, "
                f"weights pre-dequantised; {reps} steps in {el:.1f} s")

    def timed(self, rows: int, steps: int, warmup: int):
        """(step TFLOP/s, elapsed s, quantiser GB/s, GEMM TFLOP/s) over `steps` steps."""
        for _ in range(warmup):
            self.run(rows)
        tq = tg = 0.0
        t0 = time.perf_counter()
        for _ in range(steps):
            a, b = self.run(rows)
            tq += a
            tg += b
        el = time.perf_counter() - t0
        gemm_flops = self.flops(rows) * steps
        return (gemm_flops / el / 1e12, el, self.quant_bytes(rows) * steps / tq / 1e9,
                gemm_flops / tg / 1e12)


def cpu_baseline(samp: OracleSample, target_s: float = 12.0, rows: int = 32):
    t0 = time.perf_counter()
    samp.run(rows)
    t1 = time.perf_counter() - t0
    steps = max(1, int(target_s / max(t1, 1e-3)))
    tflops, el, q_gbs, g_tflops = samp.timed(rows, steps, 0)
    return {"value": round(tflops, 6), "unit": "TFLOPS", "cores": samp.threads, "kind": "oracle",
            "sample": samp.describe(rows, steps, el), "quantize_GBps": round(q_gbs, 4),
            "gemm_tflops": round(g_tflops, 6)}


# ------------------------------------------------------------------ main
WORKLOAD_BY_NAME = {"prefill": 2, "gdn_inproj": 3, "mlp": 4, "decode": 5}


def config_shape(wl: workloads.Workload) -> dict:
    if wl.name.startswith("mlp"):
        return {"M": wl.M, "K": wl.K, "N_gate_up": wl.N, "N_down": workloads.MLP_DOWN_N,
                "K_down": workloads.MLP_DOWN_K}
    return {"M": wl.M, "N": wl.N, "K": wl.K}


def layer_kernels(layer, pk, stream, fp4_peak):
    """Per-kernel device times of one workload's launches, each timed alone,
    with their roofline fractions (FP4 tensor peak for GEMMs, HBM for the
    quantiser)."""
    nv = layer.nv
    q_bytes = layer.M * layer.K * 2 + layer.M * layer.K // 2 + nv.nvfp4_scale_bytes(layer.M, layer.K)
    if isinstance(layer, MlpChain):
        t = time_each({"quantize": layer.quantize, "gate_up": layer.gate_up, "down": layer.down}, stream)
        gemms = {"gate_up": 2.0 * layer.M * layer.K * layer.N, "down": 2.0 * layer.M * layer.H * layer.N2}
    else:
        t = time_each({"quantize": layer.quantize, "gemm": layer.gemm}, stream)
        gemms = {"gemm": layer.flops}
    out = {"quantize_us": round(t["quantize"] * 1e3, 2),
           "quantize_GBps": round(q_bytes / (t["quantize"] * 1e-3) / 1e9, 1)}
    out["quantize_hbm_frac"] = round(out["quantize_GBps"] / pk["hbm"], 4)
    for name, flops in gemms.items():
        tf = flops / (t[name] * 1e-3) / 1e12
        out[f"{name}_us"] = round(t[name] * 1e3, 2)
        out[f"{name}_tflops"] = round(tf, 1)
        out[f"{name}_frac"] = round(tf / fp4_peak, 4)
    return out


def reference_main(args, wl, rank):
    """--impl reference: the oracle as it stands on this machine's host cores,
    on the same workload, metric and unit, each step a bounded row sample."""
    if rank != 0:
        return
    samp = OracleSample(wl)
    t0 = time.perf_counter()
    samp.run(1)
    t1 = time.perf_counter() - t0
    budget = 120.0 / (args.steps + args.warmup)          # whole run within a few minutes
    rows = int(np.clip(budget / max(t1, 1e-4), 1, 256))
    tflops, el, q_gbs, g_tflops = samp.timed(rows, args.steps, args.warmup)
    line = {"metric": METRIC, "value": round(tflops, 6), "unit": "TFLOPS", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(el / args.steps * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": wl.name, **config_shape(wl), "sample_rows_per_step": rows},
            "cpu_baseline": {"value": round(tflops, 6), "unit": "TFLOPS", "cores": samp.threads,
                             "kind": "oracle", "sample": samp.describe(rows, args.steps, el),
                             "quantize_GBps": round(q_gbs, 4), "gemm_tflops": round(g_tflops, 6)},
            "e2e": {"value": round(tflops, 6), "unit": "TFLOPS", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------ ncu cases
# One kernel of one configuration, launched a few times on its own with one
# set of device-resident operands (a few hundred MB at most), for profiler
# captures (`ncu -k ... python bench.py --kernel-case NAME`).  Setup launches
# (weight quantisation, calibration) come first; the listed kernel's launches
# follow.
KERNEL_CASES = {
    "quantize_prefill": "k_quantize on the 4096 x 5120 prefill activations",
    "gemm_prefill": "k_gemm_tc<2> on the 4096 x 5120 x 5120 prefill projection",
    "gemm_gdn": "k_gemm_tc<2> on the 8192 x 5120 x 16480 GDN in-projection (6 modules, gates)",
    "gate_up_mlp": "k_gemm_tc<2, true> (gate_up + SiLU*up + requantisation), 16384 x 5120 x 2 x 17408",
    "down_mlp": "k_gemm_tc<2> on the 16384 x 17408 x 5120 MLP down projection",
    "decode_m1": "k_gemm_small<16> on the GDN in-projection weights, 1 token",
    "decode_m64": "k_gemm_small<64> on the GDN in-projection weights, 64 tokens",
    "gdn_recurrence": "k_gdn_chunked, the gated delta rule over 8192 tokens x 48 value heads",
}


def kernel_case(name: str, launches: int, device):
    import nvfp4_w4a4_quantized_quantizer_b200 as nv
    st = torch.cuda.current_stream()
    if name == "gdn_recurrence":
        fn = gdn_problem(device)
    elif name in ("gate_up_mlp", "down_mlp"):
        ch = MlpChain(device, rotate_act=1, rotate_w=1)
        ch.quantize(0, st)
        if name == "down_mlp":
            ch.gate_up(0, st)
            fn = ch.down
        else:
            fn = ch.gate_up
    else:
        wl = workloads.WORKLOADS[{"quantize_prefill": 2, "gemm_prefill": 2, "gemm_gdn": 3,
                                  "decode_m1": 5, "decode_m64": 5}[name]]
        M = {"decode_m1": 1, "decode_m64": 64}.get(name, wl.M)
        layer = Layer(wl, M, device, rotate_act=1, rotate_w=1)
        layer.quantize(0, st)
        fn = layer.quantize if name == "quantize_prefill" else layer.gemm
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(st)
    for i in range(launches):
        fn(i, st)
    b.record(st)
    b.synchronize()
    st_err, info = nv.nvfp4_last_device_error()
    print(json.dumps({"kernel_case": name, "what": KERNEL_CASES[name], "launches": launches,
                      "ms_per_launch": round(a.elapsed_time(b) / launches, 4), "status": st_err}),
          flush=True)
    return 0 if st_err == 0 else 1


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default="mlp", choices=sorted(WORKLOAD_BY_NAME),
                    help="the timed step (default: the MLP pair, the largest configuration)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-small-m", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-kernel figures of the other large configurations")
    ap.add_argument("--kernel-case", choices=sorted(KERNEL_CASES),
                    help="launch one kernel of one configuration a few times (profiler captures)")
    ap.add_argument("--launches", type=int, default=3)
    ap.add_argument("--no-overlap", action="store_true",
                    help="launch the quantiser and the GEMMs without launch overlap")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    ws, rank, local = dist_env()
    wl = workloads.WORKLOADS[WORKLOAD_BY_NAME[args.workload]]
    M = wl.M

    if args.impl == "reference":
        reference_main(args, wl, rank)
        return
    if args.kernel_case:
        import nvfp4_w4a4_quantized_quantizer_b200 as nv
        nv.load()
        nv.nvfp4_set_launch_overlap(False)
        torch.cuda.set_device(local)
        sys.exit(kernel_case(args.kernel_case, args.launches, torch.device("cuda", local)))

    import nvfp4_w4a4_quantized_quantizer_b200 as nv
    nv.load()
    # the weights are quantised before any timed launch, so no kernel just
    # ahead of a GEMM writes its weights (the contract of launch overlap)
    nv.nvfp4_set_launch_overlap(not args.no_overlap)
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    pg = None
    if ws > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)
        pg = dist
    stream = torch.cuda.Stream(device)
    mlp = args.workload == "mlp"
    layer = MlpChain(device) if mlp else Layer(wl, M, device)
    torch.cuda.synchronize()
    pk = peaks()
    fp4_peak = pk["bf16"] * FP4_PER_BF16

    with ClockSampler(local) as clk:
        # main timed region: exactly K steps, barrier + sync on both sides, max over ranks
        total_ms = timed_region(pg, lambda: time_steps(layer, args.steps, args.warmup, stream),
                                torch.cuda.synchronize)
        # per-kernel device times (graphs of one kernel each, >= MIN_KERNEL_S per kernel)
        kern = {wl.name: layer_kernels(layer, pk, stream, fp4_peak)}
    clocks = clk.summary()
    total_ms = max_over_ranks(total_ms, pg, device)
    ms_step = total_ms / args.steps
    value = job_value(ws, layer.flops, ms_step)

    if mlp:
        g_name, g_flops = "gate_up", 2.0 * layer.M * layer.K * layer.N     # the dominant kernel
        step_desc = ("quantize_act + gate_up (2 modules) with SiLU(gate)*up and its requantisation "
                     "in the epilogue + down GEMM (bf16 out)")
        profile = f"gemm_tc_{wl.name}.md"
    else:
        g_name, g_flops = "gemm", layer.flops
        step_desc = "quantize_act + fused NVFP4 GEMM (bf16 out)"
        profile = f"gemm_tc_{wl.name}.md"
    g_ms = kern[wl.name][f"{g_name}_us"] * 1e-3
    g_tflops = g_flops / (g_ms * 1e-3) / 1e12
    traffic = ncu_traffic(profile)

    e_ms, h2d, d2h = e2e(layer, max(20, min(200, args.steps // 20)), 3, stream)
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOPS", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4",
        "data": "synthetic",
        "config": {"workload": wl.name, **config_shape(wl),
                   "step": step_desc,
                   "l2": f"inputs rotated over {len(layer.xs)} activation / {len(layer.ws)} weight copies "
                         "(working set > L2)", "parallelism": f"replicas x{ws}",
                   "launch": f"steps replayed from CUDA graphs of {GRAPH_STEPS} steps; launch overlap "
                             + ("off" if args.no_overlap else "on (quantiser and GEMMs)")},
        "roofline": {"bound": "tensor", "kernel": g_name, "achieved": round(g_tflops, 1),
                     "peak": round(fp4_peak, 1), "unit": "TFLOP/s", "frac": round(g_tflops / fp4_peak, 4),
                     "traffic": traffic,
                     "peak_note": f"{pk['source']} bf16 burst {pk['bf16']} x {FP4_PER_BF16} nominal "
                                  "FP4/BF16 (the kernel is timed alone, >= 0.2 s of graph replays)"},
        "kernels": kern,
        "e2e": {"value": round(layer.flops / (e_ms * 1e-3) / 1e12, 2), "unit": "TFLOPS",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": (layer.launches_per_step if mlp else 2) * args.steps,
        "clocks": clocks,
    }
    single = rank == 0 and ws == 1
    if single and not args.no_configs:
        # the other large configurations' kernels, each timed alone
        for name in ("prefill", "gdn_inproj", "mlp"):
            w2 = workloads.WORKLOADS[WORKLOAD_BY_NAME[name]]
            if w2.name in kern:
                continue
            other = MlpChain(device) if name == "mlp" else Layer(w2, w2.M, device)
            with ClockSampler(local) as clk2:
                kern[w2.name] = layer_kernels(other, pk, stream, fp4_peak)
            kern[w2.name]["clocks"] = clk2.summary()
            del other
            torch.cuda.empty_cache()
    if single and not args.no_small_m:
        sm = small_m_sweep(device, stream)
        for v in sm.values():
            v["hbm_frac"] = round(v["weight_GBps"] / pk["hbm"], 4)
        line["small_m"] = sm
        kv = kv_fp8_rate(device, stream)
        kv["hbm_frac"] = round(kv["GBps"] / pk["hbm"], 4)
        line["kv_fp8"] = kv
        line["gdn_recurrence"] = gdn_rate(device, stream)
    if single and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(OracleSample(wl))
    if rank == 0:
        print(json.dumps(line), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()


if __name__ == "__main__":
    main()
