"""Benchmark of the SVDQuant-style NVFP4 W4A4 linear on B200.

One step = one pass of the whole hot path over one batch: svdq_calib_lambda
(absmax over the packed rows), svdq_quantize_act (smooth + NVFP4 + fused
down-projection), svdq_linear (FP4 tcgen05 GEMM + low-rank + bias) and
svdq_score_lambda (per-modality rel-L2 against the bf16 layer).  The workload
is the DiT attention projection: 4096 packed rows (text 29 | video 4039 |
audio 28), K = N = 5120, rank 32, synthetic seeded data.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl svdq|reference]

Under torchrun (N > 1) every rank runs the same workload on its own GPU
(independent batches, no collective on the data path: weak scaling); the
reported time is the max over ranks.  ``--impl reference`` times the CPU
oracle on a bounded row sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "W4A4 linear TFLOP/s and % of B200 dense-FP4 peak; quantize GB/s vs HBM peak"
UNIT = "TFLOP/s"
WORKLOAD = "dit_attention_projection_M4096_K5120_N5120_r32"
CONFIG_INDEX = 1
L2_FLUSH_BYTES = 256 << 20
FP4_PER_BF16 = 4.0          # nominal dense FP4 / BF16 tensor throughput ratio (9 / 2.25 PFLOP/s)
# DRAM bytes (read + write) per launch from one ncu capture of the current kernels on this
# workload (the kernels' ncu summaries under profiles/); set to None
# whenever the kernel changes until it is captured again.
LINEAR_TRAFFIC_BYTES = 27.45e6 + 0.68e6      # ncu dram read + write per launch (launch-list capture)
QUANTIZE_TRAFFIC_BYTES = 42.32e6 + 0.11e6


def read_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return dict(hbm=float(p["hbm_gbs"]), bf16=float(p["bf16_tflops"]),
                    bf16_sus=float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), source="measured")
    except (OSError, KeyError, ValueError):
        return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, source="fallback")


def workload_bytes(m, k, n, r, m_cal):
    """Algorithmic bytes of the HBM-bound kernels (one launch each)."""
    quant = m * k * 2 + m * k // 2 + m * k // 16 + m * r * 4
    calib = m_cal * k * 2 + n * k * 2
    score = 2 * m * n * 2
    return dict(quantize=quant, calib=calib, score=score)


def max_over_ranks(ms: float, device=None) -> float:
    """The job's time: the largest of the ranks' times (the default process group's
    MAX all-reduce; the value itself when there is no group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(ms)
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(flops_per_rank: float, world: int, ms_max: float) -> float:
    """Whole-job throughput: every rank's units over the slowest rank's time."""
    return flops_per_rank * world / (ms_max * 1e-3) / 1e12


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""

    def __init__(self, index: int):
        self.proc = None
        self.path = os.path.join(tempfile.gettempdir(), f"svdq_bench_clocks_rank{index}.csv")
        self.index = index

    def start(self):
        os.makedirs(os.path.dirname(self.path), exist_ok=True)
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx = float(parts[2])
                except ValueError:
                    continue
                for nm, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# CPU oracle arm (also the cpu_baseline of the GPU arm)
# ---------------------------------------------------------------------------

class OracleArm:
    """The CPU oracle's hot path (calib, quantize, W4A4 linear, score) on a row sample."""

    def __init__(self, layer):
        from oracle import svdq_oracle as O

        import synthetic as S

        self.O = O
        self.layer = layer
        segs = layer.seg_ranges(layer.calib_sets["all"])
        self.c = O.calib(layer.x, segs, layer.w)
        self.conv = O.convert_weight(layer.w, self.c["lam"], layer.rank,
                                     sketch=S.power_iteration_sketch(layer.n, layer.rank))

    def run(self, rows: int):
        """Returns (TFLOP/s, seconds, rows) of one timed pass over `rows` evenly spaced rows."""
        O, layer = self.O, self.layer
        idx = np.linspace(0, layer.m - 1, rows).astype(np.int64)
        x = layer.x[idx]
        yref = O.f64_to_bf16(O.reference_linear(x, layer.w, layer.bias))
        t0 = time.perf_counter()
        c2 = O.calib(x, None, layer.w)
        y64, _ = O.layer_forward(x, c2["inv_lam"], self.c["s_g"], self.conv["down"], self.conv, layer.bias)
        O.score(O.f64_to_bf16(y64), yref, [(0, rows)])
        dt = time.perf_counter() - t0
        return 2.0 * rows * layer.n * layer.k / dt / 1e12, dt, rows


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import synthetic as S

    layer = S.make_layer(CONFIG_INDEX)
    arm = OracleArm(layer)
    rows = 256
    for _ in range(min(args.warmup, 1)):
        arm.run(8)
    times, vals = [], []
    for _ in range(args.steps):
        v, dt, rows = arm.run(rows)
        times.append(dt)
        vals.append(v)
    value = statistics.median(vals)
    cores = _oracle_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * statistics.median(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "rows_per_step": rows, "note": "CPU oracle on a row sample"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{rows} of 4096 rows per step, full K and N"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


def _oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        n = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
        return int(n)
    except Exception:
        return os.cpu_count() or 1


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

def _graph_ms(fn, flush, flush_read, reps=10, warmup=3):
    """Median time of `fn` captured as one CUDA graph, L2 flushed before each replay."""
    import torch
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            fn()
    torch.cuda.current_stream().wait_stream(side)
    for _ in range(warmup):
        g.replay()
    times = []
    for i in range(reps):
        flush.fill_(i & 0xFF)
        flush_read.sum()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    del g
    return float(np.median(times))


LARGE_SHAPES = ((2, "ffn_up_projection_M16384_K5120_N20480_r32"), (3, "ffn_down_projection_M16384_K20480_N5120_r32"))


def largest_shapes(P, S, dev, fp4_peak, flush, flush_read, steps=10, warmup=3):
    """The fused W4A4 linear on the two largest configured shapes, inputs
    prepared by the same path (calibration, weight conversion, quantisation);
    each call is one CUDA graph, timed with CUDA events, L2 flushed before each."""
    import torch
    out = {}
    for cfg, name in LARGE_SHAPES:
        L = S.make_layer(cfg)
        x = torch.from_numpy(np.ascontiguousarray(L.x).view(np.int16)).to(dev)
        w = torch.from_numpy(np.ascontiguousarray(L.w).view(np.int16)).to(dev)
        bias = torch.from_numpy(np.ascontiguousarray(L.bias).view(np.int16)).to(dev)
        segs = L.seg_ranges(L.calib_sets["all"])
        cal = P.svdq_calib_lambda(x, segs, w)
        lin = P.SVDQW4A4Linear.convert(w, bias, cal, L.rank)
        q = P.svdq_quantize_act(x, cal["inv_lam"], lin.s_g_act, lin.down)
        y = torch.empty((L.m, L.n), dtype=torch.bfloat16, device=dev)
        ms = _graph_ms(lambda: P.svdq_linear(q["codes"], q["sf"], lin.s_g_act, q["d"], lin.w_codes, lin.w_sf,
                                             lin.s_g_w, lin.up, lin.bias, out=y), flush, flush_read,
                       reps=steps, warmup=warmup)
        flops = 2.0 * L.m * L.n * L.k
        # accuracy against the bf16 layer (sanity: the same quantity the step scores)
        yref = torch.matmul(x.view(torch.bfloat16), w.view(torch.bfloat16).t()) + bias.view(torch.bfloat16)
        rel = float(torch.linalg.vector_norm(y.float() - yref.float()) / torch.linalg.vector_norm(yref.float()))
        out[name] = {"M": L.m, "K": L.k, "N": L.n, "rank": L.rank, "linear_ms": ms,
                     "linear_tflops": flops / (ms * 1e-3) / 1e12,
                     "frac_of_fp4_peak": flops / (ms * 1e-3) / 1e12 / fp4_peak, "rel_l2_vs_bf16": rel}
        del x, w, bias, cal, lin, q, y, yref
        torch.cuda.empty_cache()
    return out


def all_configs(P, S, dev, fp4_peak, hbm_peak, flush, flush_read):
    """Every call of the path on every configured workload (sweep: one layer per N,
    every lambda candidate), each timed alone from a cold L2."""
    import torch

    def to_dev(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev)

    def layer_calls(L, calib_name):
        x, w, bias = to_dev(L.x), to_dev(L.w), to_dev(L.bias)
        segs_cal = L.seg_ranges(L.calib_sets[calib_name]) if calib_name != "1" else \
            L.seg_ranges(L.calib_sets["all"])
        w_cal = None if calib_name == "1" else w
        segs_mod = [(sg.begin, sg.end) for sg in L.segments]
        cal = P.svdq_calib_lambda(x, segs_cal, w_cal)
        lin = P.SVDQW4A4Linear.convert(w, bias, cal, L.rank)
        q = P.svdq_quantize_act(x, cal["inv_lam"], lin.s_g_act, lin.down)
        y = torch.empty((L.m, L.n), dtype=torch.bfloat16, device=dev)
        yref = torch.matmul(x.view(torch.bfloat16), w.view(torch.bfloat16).t()) + bias.view(torch.bfloat16)
        ws = torch.empty(P.score_workspace_bytes(segs_mod, L.n), dtype=torch.uint8, device=dev)
        m_sel = sum(e - b for b, e in segs_cal)
        r = {}
        t = _graph_ms(lambda: P.svdq_calib_lambda(x, segs_cal, w_cal), flush, flush_read)
        by = 2.0 * m_sel * L.k + (2.0 * L.n * L.k if w_cal is not None else 0.0)
        r["calib"] = {"ms": t, "GB/s": by / (t * 1e-3) / 1e9, "frac_hbm": by / (t * 1e-3) / 1e9 / hbm_peak}
        t = _graph_ms(lambda: P.svdq_quantize_act(x, cal["inv_lam"], lin.s_g_act, lin.down, out=q), flush,
                      flush_read)
        by = (2 + 0.5 + 0.0625) * L.m * L.k + 4.0 * L.m * L.rank
        r["quantize"] = {"ms": t, "GB/s": by / (t * 1e-3) / 1e9, "frac_hbm": by / (t * 1e-3) / 1e9 / hbm_peak}
        t = _graph_ms(lambda: P.svdq_linear(q["codes"], q["sf"], lin.s_g_act, q["d"], lin.w_codes, lin.w_sf,
                                            lin.s_g_w, lin.up, lin.bias, out=y), flush, flush_read)
        fl = 2.0 * L.m * L.n * L.k
        r["linear"] = {"ms": t, "TFLOP/s": fl / (t * 1e-3) / 1e12, "frac_fp4": fl / (t * 1e-3) / 1e12 / fp4_peak}
        t = _graph_ms(lambda: P.svdq_score_lambda(y, yref, segs_mod, workspace=ws), flush, flush_read)
        by = 4.0 * L.m * L.n
        r["score"] = {"ms": t, "GB/s": by / (t * 1e-3) / 1e9, "frac_hbm": by / (t * 1e-3) / 1e9 / hbm_peak}
        _, _, rel = P.svdq_score_lambda(y, yref, segs_mod, workspace=ws)
        r["rel_l2_vs_bf16"] = dict(zip([sg.name for sg in L.segments], rel.cpu().tolist()))
        # the scoring fused into the linear's epilogue, with and without writing the output
        wf = torch.empty(P.linear_score_workspace_bytes(len(segs_mod)), dtype=torch.uint8, device=dev)
        la = (q["codes"], q["sf"], lin.s_g_act, q["d"], lin.w_codes, lin.w_sf, lin.s_g_w, lin.up, lin.bias)
        sep = r["linear"]["ms"] + r["score"]["ms"]
        for key, write in (("linear_score", True), ("linear_score_only", False)):
            t = _graph_ms(lambda: P.svdq_linear_score(*la, yref=yref, segs=segs_mod, out=y if write else None,
                                                      write_out=write, workspace=wf), flush, flush_read)
            _, _, _, rel_f = P.svdq_linear_score(*la, yref=yref, segs=segs_mod, out=y if write else None,
                                                 write_out=write, workspace=wf)
            same = bool(np.allclose(rel_f.cpu().numpy(), rel.cpu().numpy(), rtol=1e-9, atol=0))
            r[key] = {"ms": t, "TFLOP/s": fl / (t * 1e-3) / 1e12, "linear_plus_score_ms": sep,
                      "speedup_vs_separate": sep / t, "rel_matches_separate": same}
        if calib_name == "all":
            # the MXFP8 W8A8 variant of the same layer (no smoothing, no low-rank branch)
            qa = P.svdq_quantize_mxfp8(x)
            qw = P.svdq_quantize_mxfp8(w)
            t = _graph_ms(lambda: P.svdq_quantize_mxfp8(x, out=qa), flush, flush_read)
            by = (2 + 1 + 1.0 / 32) * L.m * L.k
            r["mxfp8_quantize"] = {"ms": t, "GB/s": by / (t * 1e-3) / 1e9,
                                   "frac_hbm": by / (t * 1e-3) / 1e9 / hbm_peak}
            t = _graph_ms(lambda: P.svdq_linear_mxfp8(qa["codes"], qa["sf"], qw["codes"], qw["sf"], lin.bias, out=y),
                          flush, flush_read)
            fp8_peak = fp4_peak / 2.0
            r["mxfp8_linear"] = {"ms": t, "TFLOP/s": fl / (t * 1e-3) / 1e12,
                                 "frac_fp8": fl / (t * 1e-3) / 1e12 / fp8_peak, "fp8_peak": fp8_peak}
            _, _, rel_mx = P.svdq_score_lambda(y, yref, segs_mod, workspace=ws)
            r["mxfp8_rel_l2_vs_bf16"] = dict(zip([sg.name for sg in L.segments], rel_mx.cpu().tolist()))
            del qa, qw
        del x, w, bias, cal, lin, q, y, yref, ws, wf
        torch.cuda.empty_cache()
        return r

    out = {}
    for cfg in (0, 1, 2, 3):
        L = S.make_layer(cfg)
        names = ["all", "video"] if cfg == 3 else ["all"]
        for name in names:
            out[f"config{cfg}_M{L.m}_K{L.k}_N{L.n}_r{L.rank}_lambda_{name}"] = layer_calls(L, name)
        del L
    for layer in (0, 4, 5):                          # one sweep layer per N (5120, 15360, 20480)
        L = S.make_layer(4, layer=layer)
        for name in ("1", "all", "video", "text"):
            out[f"config4_layer{layer}_M{L.m}_K{L.k}_N{L.n}_r{L.rank}_lambda_{name}"] = layer_calls(L, name)
        del L
    out.update(lambda_search(P, S, dev, flush, flush_read))
    return out


def lambda_search(P, S, dev, flush, flush_read):
    """The 39-candidate lambda search on one sweep layer (rank 32, three modalities):
    wall time of the whole search (host-driven; the randomized rank-32 factorisation of
    every candidate is library QR/SVD), and the grid and bits-lost kernels timed alone."""
    import time
    import torch

    def to_dev(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev)

    L = S.make_layer(4, layer=0)
    x, w, bias = to_dev(L.x), to_dev(L.w), to_dev(L.bias)
    segs_mod = [(sg.begin, sg.end) for sg in L.segments]
    calib_segs = L.seg_ranges(L.calib_sets["all"])
    P.search_lambda(x, w, bias, L.rank, calib_segs, segs_mod, alphas=P.alpha_grid(3))      # warm-up
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    res = P.search_lambda(x, w, bias, L.rank, calib_segs, segs_mod)
    torch.cuda.synchronize()
    wall = time.perf_counter() - t0
    n = int(res["alpha"].numel())
    cal = P.svdq_calib_lambda(x, calib_segs, w)
    alphas = res["alpha"].to(dev)
    ax_mod = torch.stack([P.svdq_calib_lambda(x, [sg], None)["amax_x"] for sg in segs_mod])
    t_grid = _graph_ms(lambda: P.svdq_lambda_grid(cal["amax_x"], cal["amax_w"], alphas), flush, flush_read)
    inv = res["inv_lam"]
    t_bits = _graph_ms(lambda: P.svdq_bits_lost(ax_mod, inv), flush, flush_read)
    rel = res["rel"].cpu().numpy()
    names = [sg.name for sg in L.segments]
    return {f"lambda_search_config4_layer0_M{L.m}_K{L.k}_N{L.n}_r{L.rank}": {
        "candidates": n, "wall_s": wall, "ms_per_candidate": wall / n * 1e3,
        "best_alpha": float(res["alpha"][res["best"]]),
        "rel_best": dict(zip(names, rel[res["best"]].tolist())),
        "rel_alpha_0.5": dict(zip(names, rel[int(np.argmin(np.abs(res["alpha"].numpy() - 0.5)))].tolist())),
        "lambda_grid_ms": t_grid, "bits_lost_ms": t_bits,
        "bits_lost_best": dict(zip(names, res["bits"][res["best"]].cpu().tolist()))}}


def profile_case(name: str) -> int:
    """A few launches of one kernel on the attention-projection workload, for a profiler:
    two warm-up launches, then three (capture with -s 2 -c 1..3 on the kernel's name)."""
    import torch

    import bit_w4a4_quantized_svdq_b200 as P
    import synthetic as S

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    L = S.make_layer(CONFIG_INDEX)

    def to_dev(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev)

    x, w, bias = to_dev(L.x), to_dev(L.w), to_dev(L.bias)
    segs_mod = [(sg.begin, sg.end) for sg in L.segments]
    if name == "linear_score":
        cal = P.svdq_calib_lambda(x, L.seg_ranges(L.calib_sets["all"]), w)
        lin = P.SVDQW4A4Linear.convert(w, bias, cal, L.rank)
        q = P.svdq_quantize_act(x, cal["inv_lam"], lin.s_g_act, lin.down)
        yref = x.view(torch.bfloat16) @ w.view(torch.bfloat16).t() + bias.view(torch.bfloat16)
        wf = torch.empty(P.linear_score_workspace_bytes(len(segs_mod)), dtype=torch.uint8, device=dev)
        args = (q["codes"], q["sf"], lin.s_g_act, q["d"], lin.w_codes, lin.w_sf, lin.s_g_w, lin.up, lin.bias)
        run = lambda: P.svdq_linear_score(*args, yref=yref, segs=segs_mod, write_out=False, workspace=wf)
    elif name in ("mxfp8_linear", "mxfp8_quantize"):
        qa = P.svdq_quantize_mxfp8(x)
        qw = P.svdq_quantize_mxfp8(w)
        y = torch.empty((L.m, L.n), dtype=torch.bfloat16, device=dev)
        if name == "mxfp8_linear":
            run = lambda: P.svdq_linear_mxfp8(qa["codes"], qa["sf"], qw["codes"], qw["sf"], bias, out=y)
        else:
            run = lambda: P.svdq_quantize_mxfp8(x, out=qa)
    else:
        raise SystemExit(f"unknown profile case {name}")
    torch.cuda.synchronize()
    for _ in range(5):
        run()
    torch.cuda.synchronize()
    assert P.svdq_device_error() == 0
    print(json.dumps({"profile_case": name, "launches": 5}))
    return 0


def run_gpu(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    import bit_w4a4_quantized_svdq_b200 as P
    import synthetic as S

    layer = S.make_layer(CONFIG_INDEX)
    m, k, n, r = layer.m, layer.k, layer.n, layer.rank
    segs_all = layer.seg_ranges(layer.calib_sets["all"])
    segs_mod = [(s.begin, s.end) for s in layer.segments]

    def dev_bits(b):
        return torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).to(dev)

    x = dev_bits(layer.x)
    w = dev_bits(layer.w)
    bias = dev_bits(layer.bias)
    # offline: calibration and weight conversion, the bf16 reference output
    calib = P.svdq_calib_lambda(x, segs_all, w)
    lin = P.SVDQW4A4Linear.convert(w, bias, calib, r)
    yref = torch.matmul(x.view(torch.bfloat16), w.view(torch.bfloat16).t()) + bias.view(torch.bfloat16)
    q_out = dict(codes=torch.empty((m, k // 2), dtype=torch.uint8, device=dev),
                 sf=torch.empty(P.sf_bytes(m, k), dtype=torch.uint8, device=dev),
                 d=torch.empty((m, r), dtype=torch.float32, device=dev))
    y = torch.empty((m, n), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(P.score_workspace_bytes(segs_mod, n), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_read = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def step(xx, ev=None):
        if ev is not None:
            ev[0].record()
        cal = P.svdq_calib_lambda(xx, segs_all, w)
        if ev is not None:
            ev[1].record()
        q = P.svdq_quantize_act(xx, cal["inv_lam"], lin.s_g_act, lin.down, out=q_out)
        if ev is not None:
            ev[2].record()
        P.svdq_linear(q["codes"], q["sf"], lin.s_g_act, q["d"], lin.w_codes, lin.w_sf, lin.s_g_w, lin.up,
                      lin.bias, out=y)
        if ev is not None:
            ev[3].record()
        res = P.svdq_score_lambda(y, yref, segs_mod, workspace=ws)
        if ev is not None:
            ev[4].record()
        return res

    # calib (zero + reduce), quantize, linear, score (one cooperative kernel; rows are back to back)
    launches_per_step = 2 + 1 + 1 + 1
    for _ in range(args.warmup):
        step(x)
    torch.cuda.synchronize()

    # One CUDA graph per call of the step, so the device-timed region measures
    # the kernels and not the host-side argument marshalling between them.
    graphs = [torch.cuda.CUDAGraph() for _ in range(4)]
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(graphs[0], stream=side):
            g_cal = P.svdq_calib_lambda(x, segs_all, w)
        with torch.cuda.graph(graphs[1], stream=side, pool=graphs[0].pool()):
            P.svdq_quantize_act(x, g_cal["inv_lam"], lin.s_g_act, lin.down, out=q_out)
        with torch.cuda.graph(graphs[2], stream=side, pool=graphs[0].pool()):
            P.svdq_linear(q_out["codes"], q_out["sf"], lin.s_g_act, q_out["d"], lin.w_codes, lin.w_sf, lin.s_g_w,
                          lin.up, lin.bias, out=y)
        with torch.cuda.graph(graphs[3], stream=side, pool=graphs[0].pool()):
            g_res = P.svdq_score_lambda(y, yref, segs_mod, workspace=ws)
        # the whole step (calib -> quantize -> linear -> score) as one graph
        g_step = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_step, stream=side, pool=graphs[0].pool()):
            s_cal = P.svdq_calib_lambda(x, segs_all, w)
            P.svdq_quantize_act(x, s_cal["inv_lam"], lin.s_g_act, lin.down, out=q_out)
            P.svdq_linear(q_out["codes"], q_out["sf"], lin.s_g_act, q_out["d"], lin.w_codes, lin.w_sf, lin.s_g_w,
                          lin.up, lin.bias, out=y)
            s_res = P.svdq_score_lambda(y, yref, segs_mod, workspace=ws)
    torch.cuda.current_stream().wait_stream(side)
    for _ in range(args.warmup):
        g_step.replay()
        for g in graphs:
            g.replay()
    torch.cuda.synchronize()

    # ---- device-timed region: inputs resident in HBM, L2 flushed between steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    step_evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    for i in range(args.steps):
        # L2 flush between steps, outside the events: write a buffer larger than
        # L2, then read another one so the write-back of the dirty lines happens
        # here and every step starts from a cold, clean L2.
        flush.fill_(i & 0xFF)
        flush_read.sum()
        step_evs[i][0].record()
        g_step.replay()
        step_evs[i][1].record()
    # per-call breakdown: the same calls, one graph each, events between them
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        flush_read.sum()
        evs[i][0].record()
        for j, g in enumerate(graphs):
            g.replay()
            evs[i][j + 1].record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    per = np.array([[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(4)] for i in range(args.steps)])
    step_ms = float(np.mean([e[0].elapsed_time(e[1]) for e in step_evs]))
    kern_ms = per.mean(axis=0)       # calib, quantize, linear, score
    step_ms_max = max_over_ranks(step_ms, dev)

    flops = 2.0 * m * n * k
    value = whole_job_tflops(flops, world, step_ms_max)
    peaks = read_peaks()
    fp4_peak = peaks["bf16"] * FP4_PER_BF16
    lin_tflops = flops / (kern_ms[2] * 1e-3) / 1e12
    by = workload_bytes(m, k, n, r, m)
    quant_gbs = by["quantize"] / (kern_ms[1] * 1e-3) / 1e9
    calib_gbs = by["calib"] / (kern_ms[0] * 1e-3) / 1e9
    score_gbs = by["score"] / (kern_ms[3] * 1e-3) / 1e9

    # ---- end to end through the public layer API with host buffers.  Every
    # step copies its activations from pinned host memory and reads its scores
    # back; the copy of step i + 1 runs on a second stream while step i computes
    # (two device buffers), so the step costs max(copy, compute), not their sum.
    x_host = torch.from_numpy(np.ascontiguousarray(layer.x).view(np.int16)).pin_memory()
    x_devs = [torch.empty_like(x), torch.empty_like(x)]
    rel_host = torch.empty(len(segs_mod), dtype=torch.float64).pin_memory()
    comp = torch.cuda.current_stream()
    copy_stream = torch.cuda.Stream()
    copied = [torch.cuda.Event(), torch.cuda.Event()]
    consumed = [torch.cuda.Event(), torch.cuda.Event()]

    def issue_copy(i):
        b = i % 2
        with torch.cuda.stream(copy_stream):
            if i >= 2:
                copy_stream.wait_event(consumed[b])      # step i - 2 has finished reading this buffer
            x_devs[b].copy_(x_host, non_blocking=True)
            copied[b].record(copy_stream)

    def run_step(i):
        b = i % 2
        comp.wait_event(copied[b])
        res = step(x_devs[b])
        consumed[b].record(comp)
        rel_host.copy_(res[2], non_blocking=True)

    def pipeline(n, start_event=None):
        if start_event is not None:
            copy_stream.wait_event(start_event)
        issue_copy(0)
        for i in range(n):
            if i + 1 < n:
                issue_copy(i + 1)
            run_step(i)

    pipeline(max(2, args.warmup))
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    pipeline(args.steps, start_event=e0)
    e1.record(comp)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, dev)
    e2e_value = whole_job_tflops(flops, world, e2e_ms)
    rel = rel_host.tolist()
    # the graphs replay the same calls on the same data: same scores, bit for bit
    graph_matches_eager = bool(torch.equal(g_res[2].cpu(), rel_host) and torch.equal(s_res[2].cpu(), rel_host))

    err = P.svdq_device_error()
    large = None
    if world == 1 and not args.no_large:
        large = largest_shapes(P, S, dev, fp4_peak, flush, flush_read)
    per_config = None
    if world == 1 and args.all_configs:
        per_config = all_configs(P, S, dev, fp4_peak, peaks["hbm"], flush, flush_read)
    line = None
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            # the whole workload (all rows), two passes: about 10 s of host work
            arm = OracleArm(layer)
            runs = [arm.run(m) for _ in range(2)]
            dt = sum(r[1] for r in runs)
            v = 2 * 2.0 * m * n * k / dt / 1e12
            cpu = {"value": v, "unit": UNIT, "cores": _oracle_threads(), "kind": "oracle",
                   "sample": f"the full step (all {m} rows, K={k}, N={n}) twice, {dt:.1f} s"}
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": step_ms_max, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "nvfp4 (e2m1 x e4m3/16) -> fp32 accum, bf16 out", "data": "synthetic",
            "config": {"workload": WORKLOAD, "M": m, "K": k, "N": n, "rank": r, "rows_per_gpu": m,
                       "segments": {s.name: [s.begin, s.end] for s in layer.segments},
                       "parallelism": f"replicas x{world}",
                       "l2": "flushed between steps: 256 MiB write, then 256 MiB read (cold, clean L2)",
                       "timing": "the step as one CUDA graph, CUDA events around it; kernels_ms from one graph per call"},
            "kernels_ms": {"calib": kern_ms[0], "quantize": kern_ms[1], "linear": kern_ms[2],
                           "score": kern_ms[3]},
            "linear_tflops": lin_tflops, "quantize_gbs": quant_gbs, "calib_gbs": calib_gbs, "score_gbs": score_gbs,
            "roofline": {"bound": "tensor", "kernel": "svdq_linear", "achieved": lin_tflops, "peak": fp4_peak,
                         "unit": "TFLOP/s", "frac": lin_tflops / fp4_peak, "traffic": LINEAR_TRAFFIC_BYTES,
                         "peak_source": f"{peaks['source']} bf16 burst {peaks['bf16']} x {FP4_PER_BF16:g} "
                                        "(nominal dense FP4/BF16 ratio)"},
            "roofline_hbm": {"kernel": "svdq_quantize_act", "achieved": quant_gbs, "peak": peaks["hbm"],
                             "unit": "GB/s", "frac": quant_gbs / peaks["hbm"], "traffic": QUANTIZE_TRAFFIC_BYTES,
                             "bound": "hbm"},
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": m * k * 2,
                    "d2h_bytes_per_step": 8 * len(segs_mod),
                    "how": "public API, eager calls; each step's activations copied from pinned host memory "
                           "(the next step's copy overlapped on a second stream), its scores read back"},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks,
            "rel_l2_vs_bf16": dict(zip([s.name for s in layer.segments], rel)),
            "device_error": err,
            "graph_replay_matches_eager": graph_matches_eager,
            "largest_shapes": large,
            "all_configs": per_config,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line))
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="svdq", choices=["svdq", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-large", action="store_true", help="skip the two largest-shape GEMM measurements")
    ap.add_argument("--profile-case", default=None, choices=["linear_score", "mxfp8_linear", "mxfp8_quantize"],
                    help="only launch one kernel five times on the attention-projection workload (for ncu)")
    ap.add_argument("--all-configs", action="store_true",
                    help="also time every call on every configured workload (adds a few minutes)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "svdq":
        args.warmup = 3
    if args.profile_case:
        return profile_case(args.profile_case)
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
