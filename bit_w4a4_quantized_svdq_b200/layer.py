"""SVDQuant-style W4A4 linear layer built on the C ABI.

"MiniMax-H3 . SVDQuant W4A4 (int4, rank 32, GPTQ)", opening section: the
layer keeps a 16-bit rank-r branch for the outliers, stores the residual in
4 bit, and quantises activations per token at run time.  "MiniMax-H3 NVFP4 --
what the smoothing scale should be calibrated on", sections "Calibration" and
"Why": lambda comes from activation absmax statistics on chosen rows, and the
quantiser sees X / lambda against the shared weight W * lambda.

Offline conversion (``SVDQW4A4Linear.convert``) takes the rank-r factors of
W * diag(lambda) with a randomized range finder (library QR / SVD calls on the
device: the only library arithmetic, used once per weight), then builds the
residual, its tensor scale and its NVFP4 encoding with this library's kernels.
The forward pass is two kernels: ``svdq_quantize_act`` and ``svdq_linear``.
"""
from __future__ import annotations

from typing import Optional, Sequence, Tuple

import numpy as np
import torch

from . import ops


def lowrank_factors_device(w: torch.Tensor, lam: torch.Tensor, rank: int, oversample: int = 8,
                           power_iters: int = 2, seed: int = 0) -> Tuple[torch.Tensor, torch.Tensor]:
    """Rank-r factors of W diag(lambda): (down [r, K] = (diag(1/lambda) L1)^T, up [N, r] = L2^T), bf16.

    L1 = U_r S^(1/2), L2 = S^(1/2) V_r^T for (W diag(lambda))^T = U S V^T,
    from a randomized range finder with ``power_iters`` subspace iterations
    (Halko, Martinsson and Tropp 2011), in fp64 on the device.
    """
    if rank == 0:
        n, k = w.shape
        return (torch.zeros((0, k), dtype=torch.bfloat16, device=w.device),
                torch.zeros((n, 0), dtype=torch.bfloat16, device=w.device))
    if w.dtype in (torch.int16, torch.uint16):
        w = w.view(torch.bfloat16)                               # raw bf16 bit patterns
    lam64 = lam.to(torch.float64)
    a = (w.to(torch.float64) * lam64[None, :]).t()              # [K, N]
    gen = torch.Generator(device=w.device)
    gen.manual_seed(seed)
    omega = torch.randn((a.shape[1], rank + oversample), dtype=torch.float64, device=w.device, generator=gen)
    q, _ = torch.linalg.qr(a @ omega)
    for _ in range(power_iters):
        z, _ = torch.linalg.qr(a.t() @ q)
        q, _ = torch.linalg.qr(a @ z)
    ub, s, vt = torch.linalg.svd(q.t() @ a, full_matrices=False)
    u = q @ ub
    root = s[:rank].sqrt()
    down = ((u[:, :rank] * root[None, :]) / lam64[:, None]).t().contiguous()
    up = (vt[:rank].t() * root[None, :]).contiguous()
    return down.to(torch.bfloat16), up.to(torch.bfloat16)


class SVDQW4A4Linear:
    """A converted linear layer: NVFP4 residual weight, rank-r branch, lambda, bias."""

    def __init__(self, w_codes, w_sf, s_g_w, down, up, bias, inv_lam, s_g_act, in_features, out_features):
        self.w_codes = w_codes
        self.w_sf = w_sf
        self.s_g_w = s_g_w
        self.down = down if down is not None and down.shape[0] > 0 else None
        self.up = up if self.down is not None else None
        self.bias = bias
        self.inv_lam = inv_lam
        self.s_g_act = s_g_act
        self.in_features = in_features
        self.out_features = out_features

    @staticmethod
    def calibrate(x: torch.Tensor, w: torch.Tensor, segs: Optional[Sequence[Tuple[int, int]]] = None,
                  smooth: bool = True) -> dict:
        """lambda, 1/lambda and the static activation scale from the chosen rows of x."""
        return ops.svdq_calib_lambda(x, segs, w if smooth else None)

    @classmethod
    def convert(cls, w: torch.Tensor, bias: Optional[torch.Tensor], calib: dict, rank: int,
                seed: int = 0) -> "SVDQW4A4Linear":
        """Offline conversion of a bf16 weight [N, K] with a calibration result."""
        lam = calib["lam"]
        down, up = lowrank_factors_device(w, lam, rank, seed=seed)
        residual = ops.svdq_residual(w, lam, down if rank else None, up if rank else None)
        wc = ops.svdq_calib_lambda(residual, None, None)
        q = ops.svdq_quantize_act(residual, None, wc["s_g"])
        n, k = w.shape
        return cls(q["codes"], q["sf"], wc["s_g"], down, up, bias, calib["inv_lam"], calib["s_g"], k, n)

    def quantize(self, x: torch.Tensor, sat_count: Optional[torch.Tensor] = None, out=None, stream=None) -> dict:
        return ops.svdq_quantize_act(x, self.inv_lam, self.s_g_act, self.down, sat_count, out, stream)

    def forward(self, x: torch.Tensor, out_dtype: torch.dtype = torch.bfloat16, q_out=None, y_out=None,
                stream=None) -> torch.Tensor:
        """Y = X W^T + b through the W4A4 path; x is [..., K] (leading dims flattened into rows)."""
        lead = x.shape[:-1]
        x2 = x.reshape(-1, x.shape[-1])
        q = self.quantize(x2, out=q_out, stream=stream)
        y = ops.svdq_linear(q["codes"], q["sf"], self.s_g_act, q["d"], self.w_codes, self.w_sf, self.s_g_w,
                            self.up, self.bias, out_dtype=out_dtype, out=y_out, stream=stream)
        return y.reshape(*lead, self.out_features)

    __call__ = forward


def alpha_grid(n: int = 39, lo: float = 0.05, hi: float = 0.95) -> torch.Tensor:
    """Migration strengths of the lambda search: n evenly spaced values in [lo, hi] (fp32, host)."""
    return torch.from_numpy(np.linspace(lo, hi, n).astype(np.float32))


def search_lambda(x: torch.Tensor, w: torch.Tensor, bias: Optional[torch.Tensor], rank: int,
                  calib_segs: Optional[Sequence[Tuple[int, int]]], modality_segs: Sequence[Tuple[int, int]],
                  weights: Optional[Sequence[float]] = None, alphas: Optional[torch.Tensor] = None,
                  yref: Optional[torch.Tensor] = None, seed: int = 0) -> dict:
    """Pick the smoothing scale from a grid of candidates by per-modality rel-L2 of the W4A4 output.

    "MiniMax-H3 NVFP4 -- what the smoothing scale should be calibrated on":
    section "Calibration" (lambda picked from a grid of candidates built from
    absmax statistics under a modality mask) and section "The metric that picks
    the winner also hides the cost" (rank candidates by rel-L2 against the bf16
    layer on rows of each modality, not only on proportional rows).

    Candidates lambda(alpha) = ax^alpha / aw^(1 - alpha) from the absmax of X over
    ``calib_segs`` and of W (``svdq_lambda_grid``); each is converted (rank-r
    factors, residual, NVFP4 weight), the activations quantised, and the linear
    scored against ``yref`` (default: the bf16 layer, X W^T + b by a library GEMM)
    on every modality in the GEMM's epilogue without writing its output
    (``svdq_linear_score``).  The winner has the smallest sum of weights[m] *
    rel[m] (equal weights by default; ties to the lower index).  The bits-lost
    proxy of every candidate on every modality's statistics comes along
    (``svdq_bits_lost``, one launch).

    Returns dict(alpha [n] host fp32, lam / inv_lam [n, K], s_g [n], rel [n, n_mod]
    and bits [n, n_mod] (device fp64), best (int), layer (the best candidate converted)).
    """
    dev = x.device
    alphas = alpha_grid() if alphas is None else alphas.to(torch.float32).cpu()
    n_mod = len(modality_segs)
    wts = torch.ones(n_mod, dtype=torch.float64) if weights is None else torch.tensor(weights, dtype=torch.float64)
    if wts.numel() != n_mod:
        raise ValueError("one weight per modality")
    cal = ops.svdq_calib_lambda(x, calib_segs, w)
    grid = ops.svdq_lambda_grid(cal["amax_x"], cal["amax_w"], alphas.to(dev))
    ax_mod = torch.stack([ops.svdq_calib_lambda(x, [seg], None)["amax_x"] for seg in modality_segs])
    bits = ops.svdq_bits_lost(ax_mod, grid["inv_lam"])
    if yref is None:
        xb, wb = x.view(torch.bfloat16), w.view(torch.bfloat16)
        yref = xb @ wb.t()
        if bias is not None:
            yref = yref + bias.view(torch.bfloat16)
    ws = torch.empty(ops.linear_score_workspace_bytes(n_mod), dtype=torch.uint8, device=dev)
    rel = torch.empty((alphas.numel(), n_mod), dtype=torch.float64, device=dev)
    for c in range(alphas.numel()):
        cand = dict(lam=grid["lam"][c], inv_lam=grid["inv_lam"][c], s_g=grid["s_g"][c:c + 1])
        layer = SVDQW4A4Linear.convert(w, bias, cand, rank, seed=seed)
        q = layer.quantize(x)
        _, _, _, rel[c] = ops.svdq_linear_score(q["codes"], q["sf"], layer.s_g_act, q["d"], layer.w_codes,
                                                layer.w_sf, layer.s_g_w, layer.up, layer.bias, yref, modality_segs,
                                                write_out=False, workspace=ws)
    total = rel.cpu() @ wts
    best = int(torch.argmin(total))
    cand = dict(lam=grid["lam"][best], inv_lam=grid["inv_lam"][best], s_g=grid["s_g"][best:best + 1])
    return dict(alpha=alphas, lam=grid["lam"], inv_lam=grid["inv_lam"], s_g=grid["s_g"], rel=rel, bits=bits,
                best=best, layer=SVDQW4A4Linear.convert(w, bias, cand, rank, seed=seed))
