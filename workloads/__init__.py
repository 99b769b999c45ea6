"""Seeded synthetic inputs for the NVFP4 W4A4 linear layer.

This module is the ONLY code shared by the CPU oracle side (tests, the CPU
baseline) and the CUDA side (tests, bench).  It draws random numbers and
shapes them into bf16 tensors; it holds none of the NVFP4 arithmetic (no
global scales, no block scales, no rounding to the E2M1/E4M3 grids).

Workloads follow the synthetic configurations written for the paper "Why Gated
DeltaNet Survives 4-Bit Quantization: NVFP4 W4A4 for the Recurrent Half of a
Hybrid 27B LLM" (the pages give no layer shapes; the shapes below are those of
the hybrid model's GDN in-projection and MLP as the configurations state them).

Recipe (every draw is float64, then cast to float32, then to bf16 with
round-to-nearest-even):

* every array is generated in row blocks of ``ROW_BLOCK`` rows; block ``b`` of
  stream ``s`` of configuration ``c`` uses
  ``numpy.random.Generator(PCG64(SeedSequence([seed, c, s, b])))``, so any row
  range can be regenerated without generating the rows before it;
* streams: 0 live activations, 1 calibration activations, 2 weights,
  3 per-segment weight stds, 4 gate parameters, 5 outlier channels,
  6 second-layer weights;
* "N(0, 1/sqrt(K))" means standard deviation 1/sqrt(K);
* Student-t activations use nu = 3 divided by sqrt(3) (the theoretical
  standard deviation), so the RMS is 1 in expectation;
* outlier channels: 8 column indices drawn once per configuration from
  stream 5 and shared by the live and calibration batches; those columns are
  multiplied by 100 after the t/sqrt(3) scaling;
* the tiny configuration puts one outlier per row at a uniformly drawn column,
  multiplied by 50, in both its live and calibration batches;
* the decode sweep reuses the GDN in-projection's weights, per-module weight
  stds and gate parameters (same streams of configuration 3).
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Sequence, Tuple

import numpy as np

ROW_BLOCK = 256
SEED = 0

ST_ACT, ST_CALIB, ST_W, ST_SEGSTD, ST_GATE, ST_OUTLIER, ST_W2 = range(7)


@dataclasses.dataclass(frozen=True)
class Segment:
    name: str
    width: int
    op: str = "none"          # "none" | "sigmoid" | "gdn_decay"


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic configuration of the linear layer."""
    index: int                # 1-based configuration number
    name: str
    M: int
    K: int
    segments: Tuple[Segment, ...]
    act_kind: str             # "normal_row_outlier" | "t3_channels" | "normal_channels"
    calib_rows: int
    w_std_kind: str           # "unit" | "loguniform" | "gate_up_x3"
    m_sweep: Tuple[int, ...] = ()
    weights_of: int = 0       # draw weights / gate params as configuration `weights_of` does

    @property
    def weight_cfg(self) -> int:
        return self.weights_of or self.index

    @property
    def N(self) -> int:
        return sum(s.width for s in self.segments)

    @property
    def seg_offsets(self) -> List[int]:
        out, o = [], 0
        for s in self.segments:
            out.append(o)
            o += s.width
        return out


GDN_SEGMENTS = (Segment("q", 2048), Segment("k", 2048), Segment("v", 6144),
                Segment("z", 6144), Segment("b", 48, "sigmoid"),
                Segment("a", 48, "gdn_decay"))

WORKLOADS = {
    1: Workload(1, "tiny_64x256x128", 64, 256, (Segment("w", 128),),
                "normal_row_outlier", 64, "unit"),
    2: Workload(2, "prefill_4096x5120x5120", 4096, 5120, (Segment("w", 5120),),
                "t3_channels", 512, "unit"),
    3: Workload(3, "gdn_inproj_8192x5120x16480", 8192, 5120, GDN_SEGMENTS,
                "t3_channels", 512, "loguniform"),
    4: Workload(4, "mlp_gate_up_16384x5120x34816", 16384, 5120,
                (Segment("gate", 17408), Segment("up", 17408)),
                "t3_channels", 512, "gate_up_x3"),
    5: Workload(5, "decode_sweep_Mx5120x16480", 64, 5120, GDN_SEGMENTS,
                "normal_channels", 512, "loguniform", m_sweep=(1, 8, 32, 64), weights_of=3),
}

# Second layer of the MLP pair: down projection [16384 x 17408] -> 5120.
MLP_DOWN_K = 17408
MLP_DOWN_N = 5120


def _rng(cfg: int, stream: int, block: int = 0, seed: int = SEED) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, cfg, stream, block])))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round to nearest even (no NaN input)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def outlier_channels(w: Workload, count: int = 8) -> np.ndarray:
    rng = _rng(w.index, ST_OUTLIER)
    return np.sort(rng.choice(w.K, size=count, replace=False))


def _act_block(w: Workload, stream: int, block: int, K: int) -> np.ndarray:
    rng = _rng(w.index, stream, block)
    if w.act_kind == "normal_row_outlier":
        x = rng.standard_normal((ROW_BLOCK, K))
        cols = rng.integers(0, K, size=ROW_BLOCK)
        x[np.arange(ROW_BLOCK), cols] *= 50.0
    elif w.act_kind == "t3_channels":
        x = rng.standard_t(3, size=(ROW_BLOCK, K)) / np.sqrt(3.0)
        x[:, outlier_channels(w)] *= 100.0
    elif w.act_kind == "normal_channels":
        x = rng.standard_normal((ROW_BLOCK, K))
        x[:, outlier_channels(w)] *= 100.0
    else:
        raise ValueError(w.act_kind)
    return x


def _rows(gen_block, r0: int, r1: int, K: int) -> np.ndarray:
    """Concatenate row-blocks covering [r0, r1) and cut them to that range."""
    if r1 <= r0:
        return np.zeros((0, K), np.uint16)
    b0, b1 = r0 // ROW_BLOCK, (r1 - 1) // ROW_BLOCK
    parts = [f32_to_bf16_bits(gen_block(b).astype(np.float32)) for b in range(b0, b1 + 1)]
    full = np.concatenate(parts, axis=0)
    off = r0 - b0 * ROW_BLOCK
    return np.ascontiguousarray(full[off:off + (r1 - r0)])


def activations(w: Workload, rows: Optional[Tuple[int, int]] = None, calib: bool = False,
                M: Optional[int] = None, set_index: int = 0) -> np.ndarray:
    """bf16 bit patterns [rows, K] of the live (or calibration) activation batch.

    ``set_index`` > 0 selects an independent batch with the same distribution
    (used to rotate inputs between timed iterations).
    """
    stream = ST_CALIB if calib else ST_ACT
    Mtot = w.calib_rows if calib else (M if M is not None else w.M)
    r0, r1 = rows if rows is not None else (0, Mtot)
    base = set_index * 1_000_003
    return _rows(lambda b: _act_block(w, stream, base + b, w.K), r0, r1, w.K)


def segment_stds(w: Workload) -> np.ndarray:
    """Per-segment weight standard deviations."""
    n = len(w.segments)
    base = 1.0 / np.sqrt(w.K)
    if w.w_std_kind == "unit":
        return np.full(n, base)
    if w.w_std_kind == "loguniform":
        rng = _rng(w.weight_cfg, ST_SEGSTD)
        return base * np.exp(rng.uniform(np.log(0.25), np.log(4.0), size=n))
    if w.w_std_kind == "gate_up_x3":
        return np.array([base, 3.0 * base])
    raise ValueError(w.w_std_kind)


def weights(w: Workload, rows: Optional[Tuple[int, int]] = None) -> np.ndarray:
    """bf16 bit patterns [rows, K] of the (fused) weight matrix W [N, K]."""
    stds = segment_stds(w)
    offs = np.array(w.seg_offsets + [w.N])

    def block(b):
        rng = _rng(w.weight_cfg, ST_W, b)
        z = rng.standard_normal((ROW_BLOCK, w.K))
        r = b * ROW_BLOCK + np.arange(ROW_BLOCK)
        seg = np.clip(np.searchsorted(offs, r, side="right") - 1, 0, len(stds) - 1)
        return z * stds[seg][:, None]

    r0, r1 = rows if rows is not None else (0, w.N)
    return _rows(block, r0, r1, w.K)


def down_weights(rows: Optional[Tuple[int, int]] = None) -> np.ndarray:
    """bf16 bit patterns of the MLP down projection W2 [5120, 17408], std 1/sqrt(17408)."""
    K = MLP_DOWN_K
    std = 1.0 / np.sqrt(K)

    def block(b):
        return _rng(4, ST_W2, b).standard_normal((ROW_BLOCK, K)) * std

    r0, r1 = rows if rows is not None else (0, MLP_DOWN_N)
    return _rows(block, r0, r1, K)


def gate_params(w: Workload, heads: int = 48) -> Tuple[np.ndarray, np.ndarray]:
    """(A_log, dt_bias) float32 [heads]: A_log ~ U(-1, 1.5), dt_bias ~ N(0, 0.5)."""
    rng = _rng(w.weight_cfg, ST_GATE)
    a_log = rng.uniform(-1.0, 1.5, size=heads).astype(np.float32)
    dt_bias = (rng.standard_normal(heads) * 0.5).astype(np.float32)
    return a_log, dt_bias


def random_bf16(shape: Sequence[int], seed: int, std: float = 1.0) -> np.ndarray:
    """Generic seeded N(0, std) bf16 bits for edge-case tests (ragged shapes)."""
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, 99])))
    return f32_to_bf16_bits((rng.standard_normal(tuple(shape)) * std).astype(np.float32))
