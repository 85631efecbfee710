"""CPU oracle for the SVDQuant-style NVFP4 W4A4 linear layer.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or run
this module: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It is
plain NumPy, slow and literal, and shares no code with the CUDA path (the two
meet only in the seeded input generator ``synthetic.py``).

What it computes, and where the pages say so
--------------------------------------------
Pages are cited by title and section.

* "MiniMax-H3 NVFP4 -- what the smoothing scale should be calibrated on",
  section "Why": NVFP4 puts 16 consecutive input channels under one FP8 scale
  set by that group's absmax; the kernel sees X / lambda; one weight W * lambda
  is shared by all modalities.  -> ``quantize_blocks``, ``calib``.
* Same page, section "Calibration" and table "The runs": lambda comes from
  activation absmax statistics accumulated under a modality mask; runs use a
  rank-32 low-rank branch; run 1 (lambda = 1, no branch) is plain W4A4.
  -> ``calib`` (row segments), ``lowrank_factors``, ``linear``.
* Same page, section "The metric that picks the winner also hides the cost":
  candidates are scored by relative L2 against bf16 on chosen row sets
  (proportional rows, or 4096 rows per modality).  -> ``score``.
* "MiniMax-H3 . SVDQuant W4A4 (int4, rank 32, GPTQ)", opening section:
  activation outliers are absorbed into a 16-bit rank-32 low-rank branch, the
  residual is quantised to 4 bit, activations are quantised per token at run
  time, and everything runs as one fused kernel.  -> ``residual``, ``linear``.
* "DeltaQuant on MiniMax-H3", section "The activation scale bound held": the
  activation global (FP32) scale is static, derived from a bound, and
  saturated NVFP4 groups are counted at run time.  -> ``calib`` (s_g) and the
  saturation count of ``quantize_blocks``.
* The number formats (E2M1 codes, one E4M3 scale per 16 elements, one FP32
  tensor scale) are those the pages name for NVFP4.

Readings where the pages are silent:
  R1 E2M1 rounding is round-to-nearest, ties to the even code, magnitudes
     above 6 saturate to 6, the sign bit is always kept (so -0.1 -> code 0x8).
  R2 The E4M3 block scale is the round-to-nearest-even encoding of
     t = amax / (6 * s_g), saturating at 448; subnormal scales are allowed.
  R3 The FP32 tensor scale is static: s_g = max_j(amax_j / lambda_j) / (6 * 448).
  R4 Per block: one fp32 division (t), one fp32 reciprocal (1/S), and one fp32
     multiply per element; a zero scale quantises every element to a signed 0.
  R5 x / lambda is computed as x * RN32(1 / lambda) in fp32 and never re-rounded.
  R6 Groups are 16 consecutive channels in natural order.
  R7 Packed codes: element 2i in the low nibble, 2i+1 in the high nibble.
  R8 lambda_j = sqrt(amax|X_j| / amax|W_j|) (exponent 0.5), 1 where either
     absmax is 0; s_g = 1 if every amax is 0.
  R9 Low-rank split L1 = V_r S_r^(1/2), L2 = S_r^(1/2) U_r^T of W * lambda;
     the down factor is stored with lambda folded in (L1s = diag(1/lambda) L1)
     as a [r, K] "down" weight and L2^T as an [N, r] "up" weight, both bf16.
  R10 rel-L2 of a segment is ||Yq - Yref||_F / ||Yref||_F over its rows.
  R11 fp64 results stored as bf16 (the residual, the layer output compared
      in bf16) are rounded fp64 -> fp32 -> bf16, each step to nearest, ties
      to even.
  R15 The bits-lost proxy uses per-modality channel absmax statistics: the
      channel's absmax is RN32(ax_j * (1/lambda_j)) (the smoothed statistic
      the kernel's group scale sees; max over rows commutes with the monotone
      rounded product), the group absmax is the largest of its 16 channels,
      and the figure for a modality is the mean of log2(group / channel) over
      the channels whose smoothed absmax is > 0 (a zero channel has nothing to
      lose); 0 if none counts.
  R16 Candidate smoothing scales over a migration-strength grid:
      lambda_j(alpha) = ax_j^alpha / aw_j^(1 - alpha) (R8 is alpha = 0.5),
      evaluated as RN32(2^(alpha log2 ax_j - (1 - alpha) log2 aw_j)) in fp64
      from the fp32 alpha; 1 where either absmax is 0; 1/lambda and s_g per
      candidate as in R5 and R3.
  R17 The grid: 39 evenly spaced alpha in [0.05, 0.95] (the pages give only
      the count of candidates).
  R18 Selection: the candidate with the smallest sum over modalities of
      w_m * rel_m (weights given by the caller: rows-proportional weights
      reproduce the uniform-rows column, equal weights the per-modality view);
      ties go to the lower index.
  R19 MXFP8 ("MiniMax-H3 -- MXFP8 (weight-quantized, vLLM-Omni native layout)",
      section "Quant format": OCP microscaling FP8, E4M3 elements with one
      E8M0 scale per 32 consecutive elements, symmetric round-to-nearest,
      activations quantised dynamically per 32): per block the shared
      exponent is e = floor(log2 amax) - 8 (8 = the exponent of E4M3's largest
      power of two), clamped to [-127, 127] and -127 for an all-zero block; the
      scale byte is e + 127; each element is the E4M3 code of v * 2^-e (an
      exact product) rounded to nearest, ties to even, saturating at 448, sign
      kept (-0 -> 0x80).  No smoothing, no low-rank branch, no tensor scale.

Pins (``tests/test_oracle_*.py``) hold every function to something other
than itself: independent float-format rounding, the bf16 format's definition,
torch's float8 conversion, exact rational brute force on tiny blocks, exactly
representable inputs whose W4A4 product equals a plain fp64 matmul, full-rank
low-rank branches, closed forms, worked values that separate each reading
from its nearest alternative, and reduction identities.
``tests/oracle_mutation_audit.py`` plants plausible slips in a copy of this
module and checks that each one fails a pin.  The scale-factor memory layout (``sf_to_mma_layout``)
is a hardware operand layout, not a page formula: it is pinned as a
bijection and by the GPU GEMM that consumes it.
"""
from __future__ import annotations

import math
from typing import Iterable, List, Optional, Sequence, Tuple

import numpy as np

BLOCK = 16                      # NVFP4 group size (page 1, "Why")
E2M1_MAX = 6.0
E4M3_MAX = 448.0
SF_ROWS_PER_ATOM = 128          # tcgen05 scale-factor atom: 128 rows x 4 scales
SF_COLS_PER_ATOM = 4

# Magnitudes of E2M1 codes 0..7 (sign in bit 3).
E2M1_MAGNITUDES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)


def _e4m3_table() -> np.ndarray:
    """Values of the 127 non-negative finite E4M3 (OCP E4M3FN) codes 0x00..0x7E."""
    vals = np.empty(127, dtype=np.float64)
    for c in range(127):
        e, m = c >> 3, c & 7
        vals[c] = (m / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return vals


E4M3_VALUES = _e4m3_table()


# ----------------------------------------------------------------------------
# bf16 helpers
# ----------------------------------------------------------------------------

def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return bf16_to_f32(bits).astype(np.float64)


def f32_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even fp32 -> bf16, returned as bit patterns (torch CPU conversion)."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def f64_to_bf16(x: np.ndarray) -> np.ndarray:
    """fp64 -> fp32 (round to nearest) -> bf16 (round to nearest even)."""
    return f32_to_bf16(np.asarray(x, dtype=np.float64).astype(np.float32))


# ----------------------------------------------------------------------------
# Number formats (R1, R2)
# ----------------------------------------------------------------------------

def _nearest_index_ties_even(v: np.ndarray, grid: np.ndarray) -> np.ndarray:
    """Index of the grid value nearest to v (v >= 0, grid ascending); ties -> even index.

    Differences are exact in float64 for the values that can sit on a tie, so
    ties are detected exactly.
    """
    v = np.asarray(v, dtype=np.float64)
    hi = np.clip(np.searchsorted(grid, v, side="left"), 0, len(grid) - 1)
    lo = np.clip(hi - 1, 0, len(grid) - 1)
    d_lo = v - grid[lo]
    d_hi = grid[hi] - v
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    return np.where(pick_hi, hi, lo)


def e2m1_encode(q: np.ndarray) -> np.ndarray:
    """fp32 values -> E2M1 codes 0..15 (R1: nearest, ties to even code, saturate at 6, keep sign)."""
    q = np.asarray(q, dtype=np.float32)
    mag = np.minimum(np.abs(q).astype(np.float64), E2M1_MAX)
    code = _nearest_index_ties_even(mag, E2M1_MAGNITUDES).astype(np.uint8)
    return code | (np.signbit(q).astype(np.uint8) << 3)


def e2m1_decode(code: np.ndarray) -> np.ndarray:
    code = np.asarray(code, dtype=np.uint8)
    mag = E2M1_MAGNITUDES[code & 7]
    return np.where(code & 8, -mag, mag)


def e4m3_encode_nonneg(t: np.ndarray) -> np.ndarray:
    """Non-negative fp32 -> E4M3 byte (R2: nearest, ties to even, satfinite at 448)."""
    t = np.asarray(t, dtype=np.float32).astype(np.float64)
    if np.any(t < 0) or np.any(np.isnan(t)):
        raise ValueError("block scales are non-negative and finite")
    code = _nearest_index_ties_even(np.minimum(t, E4M3_MAX), E4M3_VALUES)
    return code.astype(np.uint8)


def e4m3_decode(b: np.ndarray) -> np.ndarray:
    b = np.asarray(b, dtype=np.uint8)
    if np.any((b & 0x7F) == 0x7F):
        raise ValueError("E4M3 NaN code")
    mag = E4M3_VALUES[b & 0x7F]
    return np.where(b & 0x80, -mag, mag)


# ----------------------------------------------------------------------------
# Activation / weight quantisation (page 1 "Why"; R1-R7)
# ----------------------------------------------------------------------------

def quantize_blocks(x_bits: np.ndarray, inv_lambda: Optional[np.ndarray], s_g: float
                    ) -> Tuple[np.ndarray, np.ndarray, int]:
    """Quantise bf16 rows to NVFP4 with the fixed fp32 op sequence.

    Returns (codes uint8 [M, K] with values 0..15, natural scale bytes uint8
    [M, K/16], number of blocks whose scale saturated).
    """
    x_bits = np.asarray(x_bits, dtype=np.uint16)
    m, k = x_bits.shape
    if k % BLOCK:
        raise ValueError("K must be a multiple of 16")
    s_g = np.float32(s_g)
    if not (np.isfinite(s_g) and s_g > 0):
        raise ValueError("s_g must be positive and finite")
    xf = bf16_to_f32(x_bits)
    if inv_lambda is None:
        xs = xf.copy()
    else:
        xs = xf * np.asarray(inv_lambda, dtype=np.float32)[None, :]        # R5
    blocks = xs.reshape(m, k // BLOCK, BLOCK)
    a = np.abs(blocks).max(axis=2)                                          # group absmax
    d = np.float32(np.float32(6.0) * s_g)
    t = (a / d).astype(np.float32)
    n_sat = int(np.count_nonzero(t > np.float32(E4M3_MAX)))
    sf = e4m3_encode_nonneg(t)
    scale = (e4m3_decode(sf).astype(np.float32) * s_g).astype(np.float32)  # S
    with np.errstate(divide="ignore"):
        r_s = np.where(scale == 0, np.float32(0.0),
                       (np.float32(1.0) / scale).astype(np.float32)).astype(np.float32)
    q = (blocks * r_s[:, :, None]).astype(np.float32)
    codes = e2m1_encode(q).reshape(m, k)
    return codes, sf, n_sat


def pack_codes(codes: np.ndarray) -> np.ndarray:
    """[M, K] codes -> [M, K/2] bytes, element 2i in the low nibble (R7)."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)


def unpack_codes(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty((p.shape[0], p.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = p & 0xF
    out[:, 1::2] = p >> 4
    return out


def sf_layout_offsets(m: int, k: int) -> np.ndarray:
    """Byte offset of natural scale [row, group] in the tensor-core scale-factor layout.

    Rows are padded to 128; each 128-row x 4-group atom is 512 bytes with row r
    at (r % 32) * 16 + (r // 32 % 4) * 4; atoms run along K first.
    """
    g = k // BLOCK
    rows = np.arange(m)[:, None]
    cols = np.arange(g)[None, :]
    atom = (rows // 128) * (g // 4) + cols // 4
    return (atom * 512 + (rows % 32) * 16 + ((rows % 128) // 32) * 4 + cols % 4).astype(np.int64)


def sf_to_mma_layout(sf_nat: np.ndarray) -> np.ndarray:
    m, g = sf_nat.shape
    if g % 4:
        raise ValueError("K must be a multiple of 64")
    mp = -(-m // 128) * 128
    out = np.zeros(mp * g, dtype=np.uint8)
    out[sf_layout_offsets(m, g * BLOCK).ravel()] = np.asarray(sf_nat, dtype=np.uint8).ravel()
    return out


def sf_from_mma_layout(flat: np.ndarray, m: int, k: int) -> np.ndarray:
    return np.asarray(flat, dtype=np.uint8)[sf_layout_offsets(m, k)]


def dequantize(codes: np.ndarray, sf: np.ndarray) -> np.ndarray:
    """codes [R, K] (0..15), natural scales [R, K/16] -> fp64 [R, K] (without the tensor scale)."""
    r, k = codes.shape
    vals = e2m1_decode(codes).reshape(r, k // BLOCK, BLOCK)
    return (vals * e4m3_decode(sf)[:, :, None]).reshape(r, k)


# ----------------------------------------------------------------------------
# Calibration (page 1 "Calibration", "Why"; page 2 "The activation scale bound held")
# ----------------------------------------------------------------------------

def select_rows(m: int, segments: Optional[Sequence[Tuple[int, int]]]) -> np.ndarray:
    if segments is None:
        return np.arange(m)
    idx = [np.arange(b, e) for b, e in segments]
    return np.concatenate(idx) if idx else np.arange(0)


def calib(x_bits: np.ndarray, segments: Optional[Sequence[Tuple[int, int]]],
          w_bits: Optional[np.ndarray]):
    """Per-channel absmax of X (selected rows) and W, lambda, 1/lambda and the static s_g.

    Returns dict(ax, aw, lam, inv_lam, s_g) (fp32 values).  Without W, lambda is
    1 and s_g comes from the activation absmax alone.
    """
    x = np.abs(bf16_to_f32(x_bits))
    rows = select_rows(x.shape[0], segments)
    k = x.shape[1]
    ax = x[rows].max(axis=0) if len(rows) else np.zeros(k, np.float32)
    ax = ax.astype(np.float32)
    if w_bits is not None:
        aw = np.abs(bf16_to_f32(w_bits)).max(axis=0).astype(np.float32)
        ok = (ax > 0) & (aw > 0)
        with np.errstate(divide="ignore", invalid="ignore"):
            ratio = np.where(ok, ax / np.where(ok, aw, np.float32(1)), np.float32(1)).astype(np.float32)
        lam = np.where(ok, np.sqrt(ratio).astype(np.float32), np.float32(1.0)).astype(np.float32)
    else:
        aw = None
        lam = np.ones(k, dtype=np.float32)
    inv_lam = (np.float32(1.0) / lam).astype(np.float32)
    smoothed = (ax * inv_lam).astype(np.float32)
    top = np.float32(smoothed.max()) if k else np.float32(0)
    s_g = np.float32(top / np.float32(E2M1_MAX * E4M3_MAX)) if top > 0 else np.float32(1.0)
    return dict(ax=ax, aw=aw, lam=lam, inv_lam=inv_lam, s_g=np.float32(s_g))


# ----------------------------------------------------------------------------
# Low-rank branch and residual (page 3 opening section; page 1 "The runs")
# ----------------------------------------------------------------------------

def lowrank_factors(w_bits: np.ndarray, lam: np.ndarray, rank: int,
                    sketch: Optional[np.ndarray] = None, power_iters: int = 2):
    """Rank-r factors of W * diag(lambda) (R9), returned as bf16 bits.

    With ``sketch`` None the full SVD is used; otherwise a randomized range
    finder with ``power_iters`` subspace iterations (Halko, Martinsson and
    Tropp 2011) built from the given Gaussian test matrix [N, r + p].
    Returns (down [r, K] = (diag(1/lambda) L1)^T, up [N, r] = L2^T).
    """
    w = bf16_to_f64(w_bits)
    lam = np.asarray(lam, dtype=np.float32).astype(np.float64)
    a = (w * lam[None, :]).T                        # [K, N] = (W diag(lambda))^T
    if rank == 0:
        k, n = a.shape
        return np.zeros((0, k), np.uint16), np.zeros((n, 0), np.uint16)
    if sketch is None:
        u, s, vt = np.linalg.svd(a, full_matrices=False)
    else:
        q, _ = np.linalg.qr(a @ sketch)
        for _ in range(power_iters):
            z, _ = np.linalg.qr(a.T @ q)
            q, _ = np.linalg.qr(a @ z)
        ub, s, vt = np.linalg.svd(q.T @ a, full_matrices=False)
        u = q @ ub
    root = np.sqrt(s[:rank])
    l1 = u[:, :rank] * root[None, :]                # [K, r]
    l2 = root[:, None] * vt[:rank]                  # [r, N]
    down = f64_to_bf16((l1 / lam[:, None]).T)       # [r, K]
    up = f64_to_bf16(l2.T)                          # [N, r]
    return down, up


def residual(w_bits: np.ndarray, lam: np.ndarray, down_bits: np.ndarray, up_bits: np.ndarray
             ) -> np.ndarray:
    """R = W diag(lambda) - (diag(lambda) L1s L2)^T, in fp64, rounded fp64 -> fp32 -> bf16.

    R[n, k] = W[n, k] * lam[k] - lam[k] * sum_j down[j, k] * up[n, j], the sum
    taken in j order.
    """
    w = bf16_to_f64(w_bits)
    lam = np.asarray(lam, dtype=np.float32).astype(np.float64)
    down = bf16_to_f64(down_bits)
    up = bf16_to_f64(up_bits)
    acc = np.zeros_like(w)
    for j in range(down.shape[0]):
        acc += up[:, j][:, None] * down[j][None, :]
    r64 = w * lam[None, :] - lam[None, :] * acc
    return f64_to_bf16(r64)


def lowrank_down(x_bits: np.ndarray, down_bits: np.ndarray) -> np.ndarray:
    """D = X L1s = (X / lambda) L1 in fp64, [M, r]."""
    return bf16_to_f64(x_bits) @ bf16_to_f64(down_bits).T


# ----------------------------------------------------------------------------
# The W4A4 linear (page 3 opening section; spec formula)
# ----------------------------------------------------------------------------

def linear(a_codes: np.ndarray, a_sf: np.ndarray, s_g_act: float,
           w_codes: np.ndarray, w_sf: np.ndarray, s_g_w: float,
           d: Optional[np.ndarray] = None, up_bits: Optional[np.ndarray] = None,
           bias_bits: Optional[np.ndarray] = None) -> np.ndarray:
    """Y = s_gA s_gW deq(A) deq(W)^T + D L2 + b, all in fp64.

    a_codes [M, K] / a_sf [M, K/16] natural, w_codes [N, K] / w_sf [N, K/16],
    d [M, r] fp64, up_bits [N, r] bf16, bias [N] bf16.
    """
    a = dequantize(a_codes, a_sf)
    w = dequantize(w_codes, w_sf)
    y = (np.float64(np.float32(s_g_act)) * np.float64(np.float32(s_g_w))) * (a @ w.T)
    if d is not None and up_bits is not None and up_bits.shape[1] > 0:
        y = y + d @ bf16_to_f64(up_bits).T
    if bias_bits is not None:
        y = y + bf16_to_f64(bias_bits)[None, :]
    return y


def reference_linear(x_bits: np.ndarray, w_bits: np.ndarray, bias_bits: Optional[np.ndarray]
                     ) -> np.ndarray:
    """The unquantised layer X W^T + b in fp64 (what rel-L2 is measured against)."""
    y = bf16_to_f64(x_bits) @ bf16_to_f64(w_bits).T
    if bias_bits is not None:
        y = y + bf16_to_f64(bias_bits)[None, :]
    return y


# ----------------------------------------------------------------------------
# Scoring (page 1 "The metric that picks the winner also hides the cost")
# ----------------------------------------------------------------------------

def score(yq_bits: np.ndarray, yref_bits: np.ndarray, segments: Sequence[Tuple[int, int]]):
    """Per segment: num = sum (Yq - Yref)^2, den = sum Yref^2, rel = sqrt(num / den) (R10)."""
    yq = bf16_to_f64(yq_bits)
    yr = bf16_to_f64(yref_bits)
    num, den, rel = [], [], []
    for b, e in segments:
        diff = yq[b:e] - yr[b:e]
        n_s = float(np.sum(diff * diff))
        d_s = float(np.sum(yr[b:e] * yr[b:e]))
        num.append(n_s)
        den.append(d_s)
        rel.append(math.sqrt(n_s / d_s) if d_s > 0 else (0.0 if n_s == 0 else math.inf))
    return np.array(num), np.array(den), np.array(rel)


def bits_lost(ax: np.ndarray, inv_lam: Optional[np.ndarray]) -> np.ndarray:
    """Mean bits a channel loses to its group's shared scale, per candidate and modality.

    "MiniMax-H3 NVFP4 -- what the smoothing scale should be calibrated on",
    section "Why": 16 consecutive input channels share one FP8 scale set by the
    group's absmax, so a channel whose own absmax is below the group's loses
    log2(group_absmax / channel_absmax) bits; lambda reshapes that profile
    because the kernel sees X / lambda (statistics only, no GEMM).  Reading R15.

    ax: fp32 [n_mod, K] per-modality channel absmax of X (``calib`` over the
    modality's rows); inv_lam: fp32 [n_cand, K] candidate 1/lambda rows, or None
    for lambda = 1.  Returns fp64 [n_cand, n_mod].
    """
    ax = np.asarray(ax, dtype=np.float32)
    ax = ax.reshape(1, -1) if ax.ndim == 1 else ax
    n_mod, k = ax.shape
    assert k % BLOCK == 0
    il = np.ones((1, k), np.float32) if inv_lam is None else np.asarray(inv_lam, np.float32).reshape(-1, k)
    out = np.zeros((il.shape[0], n_mod), dtype=np.float64)
    for c in range(il.shape[0]):
        for m in range(n_mod):
            chan = (ax[m] * il[c]).astype(np.float32)                  # RN32 product (R5)
            group = np.repeat(chan.reshape(-1, BLOCK).max(axis=1), BLOCK)
            counted = chan > 0
            if counted.any():
                ratio = group[counted].astype(np.float64) / chan[counted].astype(np.float64)
                out[c, m] = float(np.mean(np.log2(ratio)))
    return out


def alpha_grid(n: int = 39, lo: float = 0.05, hi: float = 0.95) -> np.ndarray:
    """The migration-strength grid of R17 as fp32 values."""
    return np.linspace(lo, hi, n).astype(np.float32)


def lambda_grid(ax: np.ndarray, aw: np.ndarray, alphas: np.ndarray):
    """Candidate lambda, 1/lambda and s_g for every alpha (R16).

    "MiniMax-H3 NVFP4 -- what the smoothing scale should be calibrated on",
    section "Calibration": a grid of lambda candidates built from absmax
    statistics.  Returns (lam [n, K] fp32, inv_lam [n, K] fp32, s_g [n] fp32).
    """
    ax = np.asarray(ax, np.float32)
    aw = np.asarray(aw, np.float32)
    ok = (ax > 0) & (aw > 0)
    lx = np.log2(np.where(ok, ax, np.float32(1)).astype(np.float64))
    lw = np.log2(np.where(ok, aw, np.float32(1)).astype(np.float64))
    lams, invs, sgs = [], [], []
    for a in np.asarray(alphas, np.float32):
        a64 = float(a)
        t = a64 * lx - (1.0 - a64) * lw
        lam = np.where(ok, np.exp2(t).astype(np.float32), np.float32(1.0)).astype(np.float32)
        inv = (np.float32(1.0) / lam).astype(np.float32)
        top = np.float32((ax * inv).astype(np.float32).max()) if ax.size else np.float32(0)
        s_g = np.float32(top / np.float32(E2M1_MAX * E4M3_MAX)) if top > 0 else np.float32(1.0)
        lams.append(lam)
        invs.append(inv)
        sgs.append(s_g)
    return np.array(lams), np.array(invs), np.array(sgs, dtype=np.float32)


def select_candidate(rel: np.ndarray, weights: np.ndarray) -> int:
    """Index of the candidate with the smallest weighted sum of per-modality rel-L2 (R18)."""
    total = np.asarray(rel, np.float64) @ np.asarray(weights, np.float64)
    return int(np.argmin(total))


# ----------------------------------------------------------------------------
# MXFP8 W8A8 (page 5 "Quant format"; R19)
# ----------------------------------------------------------------------------

MX_BLOCK = 32
E4M3_EMAX = 8                       # 448 = 1.75 * 2^8


def e4m3_encode(v: np.ndarray) -> np.ndarray:
    """Signed fp32 values -> E4M3 bytes: nearest, ties to even, satfinite at 448, sign kept."""
    v = np.asarray(v, dtype=np.float32)
    mag = e4m3_encode_nonneg(np.abs(v))
    return (mag | np.where(np.signbit(v), np.uint8(0x80), np.uint8(0))).astype(np.uint8)


def mx_shared_exponent(amax: np.ndarray) -> np.ndarray:
    """floor(log2 amax) - 8, clamped to [-127, 127]; -127 where amax is 0 (R19)."""
    amax = np.asarray(amax, dtype=np.float64)
    _, e2 = np.frexp(amax)                    # amax = m 2^e2 with m in [0.5, 1): floor(log2) = e2 - 1
    e = np.where(amax > 0, e2.astype(np.int64) - 1 - E4M3_EMAX, -127)
    return np.clip(e, -127, 127)


def mx_quantize(x_bits: np.ndarray):
    """bf16 [R, K] -> (E4M3 codes u8 [R, K], E8M0 scale bytes u8 [R, K/32]) (R19)."""
    x = bf16_to_f64(x_bits)
    r, k = x.shape
    if k % MX_BLOCK:
        raise ValueError("K must be a multiple of 32")
    blocks = x.reshape(r, k // MX_BLOCK, MX_BLOCK)
    e = mx_shared_exponent(np.abs(blocks).max(axis=2))
    scaled = blocks * np.exp2(-e.astype(np.float64))[:, :, None]      # exact: a power of two
    codes = e4m3_encode(scaled.astype(np.float32))
    return codes.reshape(r, k), (e + 127).astype(np.uint8)


def mx_dequantize(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """E4M3 codes [R, K] and E8M0 scale bytes [R, K/32] -> fp64 [R, K]."""
    r, k = codes.shape
    vals = e4m3_decode(codes).reshape(r, k // MX_BLOCK, MX_BLOCK)
    return (vals * np.exp2(np.asarray(scales, np.float64) - 127.0)[:, :, None]).reshape(r, k)


def mx_linear(a_codes, a_sf, w_codes, w_sf, bias_bits: Optional[np.ndarray]) -> np.ndarray:
    """The W8A8 MXFP8 linear in fp64: dequant(A) dequant(W)^T + b."""
    y = mx_dequantize(a_codes, a_sf) @ mx_dequantize(w_codes, w_sf).T
    if bias_bits is not None:
        y = y + bf16_to_f64(bias_bits)[None, :]
    return y


# ----------------------------------------------------------------------------
# Whole-layer helpers used by the tests
# ----------------------------------------------------------------------------

def convert_weight(w_bits: np.ndarray, lam: np.ndarray, rank: int, sketch=None):
    """Offline conversion of one weight: factors, residual and its NVFP4 encoding."""
    down, up = lowrank_factors(w_bits, lam, rank, sketch)
    r = residual(w_bits, lam, down, up) if rank > 0 else f64_to_bf16(
        bf16_to_f64(w_bits) * np.asarray(lam, np.float32).astype(np.float64)[None, :])
    cw = calib(r, None, None)
    codes, sf, _ = quantize_blocks(r, None, cw["s_g"])
    return dict(down=down, up=up, residual=r, s_g=cw["s_g"], codes=codes, sf=sf)


def layer_forward(x_bits, inv_lam, s_g_act, down_bits, wconv, bias_bits):
    """Quantise X, run the W4A4 linear with the low-rank branch; returns (Y64, parts)."""
    codes, sf, n_sat = quantize_blocks(x_bits, inv_lam, s_g_act)
    d = lowrank_down(x_bits, down_bits) if down_bits is not None and down_bits.shape[0] else None
    y = linear(codes, sf, s_g_act, wconv["codes"], wconv["sf"], wconv["s_g"],
               d, wconv["up"] if d is not None else None, bias_bits)
    return y, dict(codes=codes, sf=sf, n_sat=n_sat, d=d)
