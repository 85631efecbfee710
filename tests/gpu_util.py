"""Helpers for the GPU parity tests: moving bf16 bit patterns to and from the
device, and the comparison rules for floating-point outputs."""
import numpy as np
import pytest
import torch

from oracle import svdq_oracle as O

requires_cuda = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")


def dev_bits(bits: np.ndarray) -> torch.Tensor:
    """uint16 bf16 bit patterns -> int16 CUDA tensor (the library reads raw bits)."""
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda()


def host_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def dev_f32(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def check_sf(flat_gpu: torch.Tensor, sf_nat: np.ndarray, m: int, k: int) -> None:
    """Scale bytes: bit-exact after un-swizzling, pad rows zero."""
    flat = flat_gpu.cpu().numpy()
    got = O.sf_from_mma_layout(flat, m, k)
    mism = np.argwhere(got != sf_nat)
    assert mism.size == 0, f"{len(mism)} scale mismatches, first {mism[:4].tolist()}"
    mask = np.ones(flat.size, bool)
    mask[O.sf_layout_offsets(m, k).ravel()] = False
    assert not flat[mask].any(), "pad scale bytes must be zero"


def check_codes(codes_gpu: torch.Tensor, codes_nat: np.ndarray, rows=None) -> None:
    got = O.unpack_codes(codes_gpu.cpu().numpy())
    want = codes_nat
    if rows is not None:
        got = got[rows]
    mism = np.argwhere(got != want)
    assert mism.size == 0, f"{len(mism)} code mismatches, first {mism[:4].tolist()}: " \
                           f"{got[tuple(mism[0])] if mism.size else ''} vs {want[tuple(mism[0])] if mism.size else ''}"


def rel_l2(a: np.ndarray, b: np.ndarray) -> float:
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


# Tolerances: rel-L2 <= 2e-3 and max-abs <= 1e-2 x RMS of the output.  A bf16
# output is compared with the oracle rounded once to bf16; there a one-ulp flip
# at an outlier can exceed 1e-2 x RMS, so max-abs allows max(1e-2 RMS, 1 ulp).
REL_L2 = 2e-3
MAX_ABS_RMS = 1e-2


def bf16_ulp(v: np.ndarray) -> np.ndarray:
    a = np.abs(v.astype(np.float32))
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.exp2(e - 7.0)


def check_linear_bf16(y_gpu_bits: np.ndarray, y64: np.ndarray, tight_rel: float = None):
    g = O.bf16_to_f64(y_gpu_bits)
    yb = O.bf16_to_f64(O.f64_to_bf16(y64))
    rms = float(np.sqrt(np.mean(y64 * y64)))
    rel = rel_l2(g, yb)
    err = np.abs(g - yb)
    bound = np.maximum(MAX_ABS_RMS * rms, bf16_ulp(yb) * 1.0001)
    assert rel <= REL_L2, f"rel-L2 vs bf16(oracle) {rel:.3e}"
    bad = np.argwhere(err > bound)
    assert bad.size == 0, f"{len(bad)} outputs beyond max-abs bound, first {bad[:3].tolist()}"
    if tight_rel is not None:
        assert rel <= tight_rel, f"rel-L2 {rel:.3e} above the expected {tight_rel:.1e}"
    return rel, float(err.max() / rms)


def check_linear_f32(y_gpu: np.ndarray, y64: np.ndarray, tight_rel: float = None):
    g = y_gpu.astype(np.float64)
    rms = float(np.sqrt(np.mean(y64 * y64)))
    rel = rel_l2(g, y64)
    mx = float(np.abs(g - y64).max() / rms)
    assert rel <= REL_L2 and mx <= MAX_ABS_RMS, f"fp32 output rel-L2 {rel:.3e}, max-abs/RMS {mx:.3e}"
    if tight_rel is not None:
        assert rel <= tight_rel, f"rel-L2 {rel:.3e} above the expected {tight_rel:.1e}"
    return rel, mx


def d_tolerance(x_bits: np.ndarray, down_bits: np.ndarray) -> np.ndarray:
    """Bound on |D_gpu - D64|: D is accumulated in fp32 over K/16 MMA steps (16
    exact bf16 products each) and a split-K sum of at most 4 partials, so the
    recursive-summation bound (n additions, unit roundoff 2^-24) applies with
    n = K/16 + 20: |error| <= n * 2^-24 * sum_k |x_k down_k|."""
    k = x_bits.shape[1]
    n = k // 16 + 20
    ax = np.abs(O.bf16_to_f64(x_bits))
    ad = np.abs(O.bf16_to_f64(down_bits))
    return n * 2.0 ** -24 * (ax @ ad.T) + 1e-30


def check_d(d_gpu: np.ndarray, d64: np.ndarray, x_bits: np.ndarray, down_bits: np.ndarray) -> float:
    """D against the fp64 value: every element within the worst-case bound of
    d_tolerance, and the whole array norm-wise within ((K/16)/2 + 4) * 2^-24.

    The recursive-summation bound gives each element an error of at most
    n 2^-24 sum|x down| for n = K/16 MMA steps.  The tensor core does not round
    like n sequential fp32 additions, so the typical error is not a random walk
    of roundings either: norm-wise it came out at 0.64 n 2^-24 relative on the
    16384 x 20480 FFN down-projection input (n = 1280) and lower on the smaller
    K.  Half of the factor n, applied to the norm, still fails an accumulation
    that went wrong on average -- a dropped or doubled partial, a lost split-K
    term, a partial rounded to bf16 -- although each element may still fit the
    worst case."""
    k = x_bits.shape[1]
    assert np.all(np.abs(d_gpu - d64) <= d_tolerance(x_bits, down_bits))
    rel = rel_l2(d_gpu.astype(np.float64), d64)
    bound = ((k / 16) / 2 + 4) * 2.0 ** -24          # + 4 units: the roundings of a single MMA step
    assert rel <= bound, f"D rel-L2 {rel:.3e} above {bound:.3e}"
    return rel
