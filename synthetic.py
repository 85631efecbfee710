"""Seeded synthetic inputs for the SVDQuant-style W4A4 linear layer.

This module only draws random numbers and lays them out.  It holds none of the
method's arithmetic (no smoothing, no quantisation, no low-rank factorisation):
both the CPU oracle and the CUDA path take their inputs from here, and neither
shares any other code with the other.

The shapes and value distributions follow the workloads described on the pages:

* "MiniMax-H3 NVFP4 -- what the smoothing scale should be calibrated on"
  (yitongl/minimax-h3-nvfp4-lambda-modality), opening paragraphs and section
  "The metric that picks the winner also hides the cost": a packed
  [text | video | audio] sequence in which video is 98.6 % of the rows, with
  per-modality channel profiles that are uncorrelated or anti-correlated
  (section "Why"), and per-modality scoring on 4096 rows per modality.
* The same page, table "The runs": rank-32 low-rank branch; seed 1101.
* "DeltaQuant on MiniMax-H3" section "Two things that were wrong on the way":
  block linears are handed 3-D activations, which callers flatten into rows.

Every array is produced in float32 and rounded once to bfloat16; bf16 arrays
are returned as ``numpy.uint16`` bit patterns (the storage format both sides
read).  Seeds are ``1101 + config index`` (``numpy.random.default_rng``).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

BASE_SEED = 1101

# Mixing of the packed sequence (page 1: video is 98.6 % of the rows).
NON_VIDEO_FRACTION = 0.014
# Per-modality channel profile: p[j] = exp(PROFILE_LOG_SD * z_j), z_j ~ N(0,1),
# independent per modality (page 1 measures near-zero / negative correlation),
# and OUTLIER_FRACTION of channels scaled by U(20, 100).
PROFILE_LOG_SD = 0.75
OUTLIER_FRACTION = 0.01
OUTLIER_RANGE = (20.0, 100.0)
WEIGHT_STD = 0.02
BIAS_STD = 0.02


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round to nearest even) and return the bit patterns.

    Done with torch's CPU conversion: this is input preparation, not part of
    the quantiser under test.
    """
    import torch

    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float32."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


@dataclasses.dataclass
class Segment:
    name: str
    begin: int
    end: int  # half-open


def packed_modality_counts(m: int) -> Tuple[int, int, int]:
    """(text, video, audio) row counts of a packed sequence of m rows.

    Non-video rows are round(0.014 m), split with the extra row going to text.
    M=4096 gives (29, 4039, 28); M=16384 gives (115, 16155, 114).
    """
    n_nv = int(round(NON_VIDEO_FRACTION * m))
    n_text = (n_nv + 1) // 2
    n_audio = n_nv // 2
    return n_text, m - n_nv, n_audio


def packed_segments(m: int) -> List[Segment]:
    """Row segments of the packed [text | video | audio] order (page 1, first paragraph)."""
    t, v, a = packed_modality_counts(m)
    return [Segment("text", 0, t), Segment("video", t, t + v), Segment("audio", t + v, m)]


def modality_profile(rng: np.random.Generator, k: int) -> np.ndarray:
    """One modality's per-channel scale profile (float32, length k)."""
    p = np.exp(PROFILE_LOG_SD * rng.standard_normal(k)).astype(np.float32)
    n_out = max(1, int(round(OUTLIER_FRACTION * k)))
    idx = rng.choice(k, size=n_out, replace=False)
    p[idx] *= rng.uniform(*OUTLIER_RANGE, size=n_out).astype(np.float32)
    return p


def _normal(rng: np.random.Generator, shape, scale: float = 1.0) -> np.ndarray:
    out = rng.standard_normal(shape, dtype=np.float32)
    if scale != 1.0:
        out *= np.float32(scale)
    return out


def _gelu_erf(h: np.ndarray) -> np.ndarray:
    """Exact (erf) GELU in float32; used only to shape config 3's activations."""
    from scipy.special import erf

    return (0.5 * h * (1.0 + erf(h / np.float32(math.sqrt(2.0))))).astype(np.float32)


@dataclasses.dataclass
class LayerInputs:
    """One synthetic linear layer: activations, weight, bias and row segments."""

    name: str
    x: np.ndarray  # uint16 bf16 bits [M, K]
    w: np.ndarray  # uint16 bf16 bits [N, K]
    bias: np.ndarray  # uint16 bf16 bits [N]
    rank: int
    segments: List[Segment]
    # Row sets lambda is calibrated on (each a list of segment names).
    calib_sets: Dict[str, List[str]]

    @property
    def m(self) -> int:
        return int(self.x.shape[0])

    @property
    def k(self) -> int:
        return int(self.x.shape[1])

    @property
    def n(self) -> int:
        return int(self.w.shape[0])

    def seg_ranges(self, names: Sequence[str]) -> List[Tuple[int, int]]:
        by = {s.name: s for s in self.segments}
        return [(by[n].begin, by[n].end) for n in names]


# Descriptions of the five workloads (sizes used by the tests and the bench).
CONFIGS = {
    0: dict(name="tiny", m=256, k=512, n=512, rank=16),
    1: dict(name="dit_attn_proj", m=4096, k=5120, n=5120, rank=32),
    2: dict(name="ffn_up", m=16384, k=5120, n=20480, rank=32),
    3: dict(name="ffn_down", m=16384, k=20480, n=5120, rank=32),
    4: dict(name="lambda_sweep", m=3 * 4096, k=5120, n=None, rank=32, layers=48),
}

SWEEP_N_CYCLE = (5120, 5120, 5120, 5120, 15360, 20480)
SWEEP_ROWS_PER_MODALITY = 4096


def _packed_x(rng: np.random.Generator, m: int, k: int, segments: List[Segment],
              heavy: Optional[np.ndarray] = None) -> np.ndarray:
    """Packed activations: row i of modality s is p_s * N(0,1) (times heavy, if given)."""
    x = np.empty((m, k), dtype=np.float32)
    for seg in segments:
        prof = modality_profile(rng, k)
        if heavy is not None:
            prof = prof * heavy
        rows = seg.end - seg.begin
        if rows:
            x[seg.begin:seg.end] = _normal(rng, (rows, k)) * prof[None, :]
    return x


def make_layer(config: int, m: Optional[int] = None, k: Optional[int] = None,
               n: Optional[int] = None, layer: int = 0) -> LayerInputs:
    """Build the seeded inputs of one workload.

    ``m``/``k``/``n`` override the sizes (to make small cases with the same
    recipe); ``layer`` selects the layer of the lambda sweep (config 4).
    """
    spec = CONFIGS[config]
    m = spec["m"] if m is None else m
    k = spec["k"] if k is None else k
    if config == 4:
        n_default = SWEEP_N_CYCLE[layer % len(SWEEP_N_CYCLE)]
    else:
        n_default = spec["n"]
    n = n_default if n is None else n
    rank = spec["rank"]
    seed = [BASE_SEED + config, layer] if config == 4 else BASE_SEED + config
    rng = np.random.default_rng(seed)

    if config == 0:
        x = _normal(rng, (m, k))
        out_ch = rng.choice(k, size=4, replace=False)
        x[:, out_ch] *= np.float32(50.0)
        segments = [Segment("all", 0, m)]
        calib = {"all": ["all"]}
    elif config in (1, 2):
        segments = packed_segments(m)
        x = _packed_x(rng, m, k, segments)
        calib = {"all": ["text", "video", "audio"]}
    elif config == 3:
        segments = packed_segments(m)
        heavy = np.abs(rng.standard_t(3, size=k)).astype(np.float32)
        h = _packed_x(rng, m, k, segments, heavy=heavy)
        x = _gelu_erf(h)
        calib = {"all": ["text", "video", "audio"], "video": ["video"]}
    elif config == 4:
        per = m // 3
        segments = [Segment("text", 0, per), Segment("video", per, 2 * per),
                    Segment("audio", 2 * per, m)]
        x = _packed_x(rng, m, k, segments)
        calib = {"all": ["text", "video", "audio"], "video": ["video"], "text": ["text"]}
    else:
        raise ValueError(f"unknown config {config}")

    w = _normal(rng, (n, k), WEIGHT_STD)
    b = _normal(rng, (n,), BIAS_STD)
    return LayerInputs(
        name=f"{spec['name']}" + (f"_l{layer}" if config == 4 else ""),
        x=f32_to_bf16_bits(x), w=f32_to_bf16_bits(w), bias=f32_to_bf16_bits(b),
        rank=rank, segments=segments, calib_sets=calib)


def power_iteration_sketch(k: int, rank: int, oversample: int = 8, seed: int = BASE_SEED) -> np.ndarray:
    """Gaussian test matrix [k, rank + oversample] for a randomized range finder.

    Random numbers a factorisation draws are inputs, so they come from here.
    """
    rng = np.random.default_rng([seed, k, rank, oversample])
    return rng.standard_normal((k, rank + oversample))


def random_bf16(shape, seed: int, scale: float = 1.0) -> np.ndarray:
    """Plain N(0, scale^2) bf16 bits, for reduction tests (score, calib)."""
    rng = np.random.default_rng(seed)
    return f32_to_bf16_bits(_normal(rng, shape, scale))
