"""Benchmark of the SVDQuant-style NVFP4 W4A4 linear on B200.

One step = one pass of the whole hot path over one batch: calibration
(svdq_calib_lambda_stored_w: absmax over the packed rows, lambda against the
weight's absmax kept from conversion, 1/lambda, the static tensor scale),
svdq_quantize_act (smooth + NVFP4 + fused down-projection), svdq_linear (FP4
tcgen05 GEMM + low-rank + bias) and svdq_score_lambda (per-modality rel-L2
against the bf16 layer).  The headline workload is the largest configured
layer, the FFN down-projection: 16384 packed rows (text 115 | video 16155 |
audio 114), K = 20480, N = 5120, rank 32, lambda calibrated on all rows,
synthetic seeded data.  The attention projection (4096 x 5120 x 5120) and the
FFN up-projection (16384 x 5120 -> 20480) are reported beside it.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl svdq|reference]

Under torchrun (N > 1) every rank runs the same workload on its own GPU
(independent batches, no collective on the data path: weak scaling); the
reported time is the max over ranks.  ``--impl reference`` times the CPU
oracle on a bounded row sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
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
HEADLINE_CONFIG = 3
WORKLOADS = {
    0: "tiny_M256_K512_N512_r16",
    1: "dit_attention_projection_M4096_K5120_N5120_r32",
    2: "ffn_up_projection_M16384_K5120_N20480_r32",
    3: "ffn_down_projection_M16384_K20480_N5120_r32",
}
SECONDARY_CONFIGS = (1, 2)
L2_BYTES = 126 << 20
L2_FLUSH_BYTES = 256 << 20
FP4_PER_BF16 = 4.0          # nominal dense FP4 / BF16 tensor throughput ratio (9 / 2.25 PFLOP/s)
# DRAM bytes (read + write) per launch of the linear on each workload, from one
# ncu capture of the current kernel (summaries under profiles/); None until the
# current kernel has been captured on that workload.
LINEAR_TRAFFIC_BYTES = {3: 496.65e6 + 155.86e6}
QUANTIZE_TRAFFIC_BYTES = {3: 673.66e6 + 171.37e6}
# Our kernels per step: calib (zeroing + stream), quantize, linear, score (one
# cooperative kernel when rows are back to back).
LAUNCHES_PER_STEP = 5


def read_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return dict(hbm=float(p["hbm_gbs"]), bf16=float(p["bf16_tflops"]),
                    bf16_sus=float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), source="measured")
    except (OSError, KeyError, ValueError):
        return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, source="fallback")


def workload_bytes(m, k, n, r, m_cal, with_w=True):
    """Algorithmic bytes of the HBM-bound kernels (one launch each)."""
    quant = m * k * 2 + m * k // 2 + m * k // 16 + m * r * 4
    calib = m_cal * k * 2 + (n * k * 2 if with_w else 0)
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
        with open(self.path) as f:
            return parse_clocks(f)


CLOCK_REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]


def parse_clocks(lines):
    """Median SM clock, max clock and the throttle reasons seen active, from
    nvidia-smi lines of the query above (csv, no header, no units); None when no
    line could be read."""
    sm, mx, reasons = [], None, set()
    for line in lines:
        parts = [p.strip() for p in line.split(",")]
        if len(parts) < 9:
            continue
        try:
            sm.append(float(parts[1]))
            mx = float(parts[2])
        except ValueError:
            continue
        for nm, v in zip(CLOCK_REASONS, parts[5:9]):
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


def _oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        n = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
        return int(n)
    except Exception:
        return os.cpu_count() or 1


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import synthetic as S

    cfg = args.config
    layer = S.make_layer(cfg)
    arm = OracleArm(layer)
    # W untimed warm-up steps on the timed sample (a step costs ~2 s on 16 host
    # threads, most of it the oracle reading and dequantising the whole weight)
    rows = min(layer.m, 128)
    for _ in range(args.warmup):
        arm.run(rows)
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
        "config": {"workload": WORKLOADS[cfg], "M": layer.m, "K": layer.k, "N": layer.n, "rank": layer.rank,
                   "rows_per_step": rows, "note": "CPU oracle on a row sample"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{rows} evenly spaced of {layer.m} rows per step, full K and N "
                                   "(calibration of the sample, quantisation, fp64 W4A4 linear, score)"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

def _to_dev(a, dev):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev)


def _capture(fn):
    """`fn` captured as one CUDA graph (on a side stream, as capture requires)."""
    import torch
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            fn()
    torch.cuda.current_stream().wait_stream(side)
    return g


def _graph_ms(fn, flush, flush_read, reps=10, warmup=3):
    """Median time of `fn` captured as one CUDA graph, L2 flushed before each replay."""
    import torch
    fn()
    torch.cuda.synchronize()
    g = _capture(fn)
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


class Workload:
    """One configured layer on the device: inputs, the converted layer, the bf16
    reference output and the step's buffers, plus the step itself."""

    def __init__(self, P, S, cfg, dev, calib_name="all"):
        import torch
        self.P, self.cfg, self.dev = P, cfg, dev
        L = S.make_layer(cfg)
        self.layer = L
        self.m, self.k, self.n, self.r = L.m, L.k, L.n, L.rank
        self.segs_all = L.seg_ranges(L.calib_sets[calib_name])
        self.segs_mod = [(s.begin, s.end) for s in L.segments]
        self.m_cal = sum(e - b for b, e in self.segs_all)
        self.x = _to_dev(L.x, dev)
        self.w = _to_dev(L.w, dev)
        self.bias = _to_dev(L.bias, dev)
        # offline: calibration and weight conversion, the bf16 reference output; the
        # weight's absmax is a constant of the converted layer, kept for the step's
        # calibration (which then reads X alone)
        cal = P.svdq_calib_lambda(self.x, self.segs_all, self.w)
        self.amax_w = cal["amax_w"]
        self.lin = P.SVDQW4A4Linear.convert(self.w, self.bias, cal, self.r)
        self.yref = (torch.matmul(self.x.view(torch.bfloat16), self.w.view(torch.bfloat16).t())
                     + self.bias.view(torch.bfloat16))
        m, k, n, r = self.m, self.k, self.n, self.r
        self.q_out = dict(codes=torch.empty((m, k // 2), dtype=torch.uint8, device=dev),
                          sf=torch.empty(P.sf_bytes(m, k), dtype=torch.uint8, device=dev),
                          d=torch.empty((m, r), dtype=torch.float32, device=dev))
        self.y = torch.empty((m, n), dtype=torch.bfloat16, device=dev)
        self.ws = torch.empty(P.score_workspace_bytes(self.segs_mod, n), dtype=torch.uint8, device=dev)
        self.flops = 2.0 * m * n * k

    # the four calls of the step (eager; also what the graphs capture)
    def calib(self, xx):
        return self.P.svdq_calib_lambda_stored_w(xx, self.segs_all, self.amax_w)

    def quantize(self, xx, cal):
        lin = self.lin
        return self.P.svdq_quantize_act(xx, cal["inv_lam"], lin.s_g_act, lin.down, out=self.q_out)

    def linear(self, q, y):
        lin = self.lin
        return self.P.svdq_linear(q["codes"], q["sf"], lin.s_g_act, q["d"], lin.w_codes, lin.w_sf, lin.s_g_w,
                                  lin.up, lin.bias, out=y)

    def score(self, y):
        return self.P.svdq_score_lambda(y, self.yref, self.segs_mod, workspace=self.ws)

    def step(self, xx, y=None):
        y = self.y if y is None else y
        cal = self.calib(xx)
        q = self.quantize(xx, cal)
        self.linear(q, y)
        return self.score(y)

    def kernel_times(self, flush, flush_read, reps):
        """Each call of the step as its own CUDA graph, timed from a cold L2."""
        x = self.x
        cal = self.calib(x)
        q = self.quantize(x, cal)
        out = {}
        out["calib"] = _graph_ms(lambda: self.calib(x), flush, flush_read, reps)
        out["quantize"] = _graph_ms(lambda: self.quantize(x, cal), flush, flush_read, reps)
        out["linear"] = _graph_ms(lambda: self.linear(q, self.y), flush, flush_read, reps)
        out["score"] = _graph_ms(lambda: self.score(self.y), flush, flush_read, reps)
        return out

    def fractions(self, kern_ms, peaks):
        fp4_peak = peaks["bf16"] * FP4_PER_BF16
        by = workload_bytes(self.m, self.k, self.n, self.r, self.m_cal, with_w=False)
        lin_tflops = self.flops / (kern_ms["linear"] * 1e-3) / 1e12
        rates = {name: by[name] / (kern_ms[name] * 1e-3) / 1e9 for name in ("calib", "quantize", "score")}
        return {
            "kernels_ms": kern_ms,
            "linear_tflops": lin_tflops, "linear_frac_of_fp4_peak": lin_tflops / fp4_peak,
            "gbs": rates, "frac_of_hbm": {k: v / peaks["hbm"] for k, v in rates.items()},
            "algorithmic_bytes": by,
        }


def time_step(wl, steps, warmup, flush=None, flush_read=None, world=1):
    """ms per step of the whole step captured as one CUDA graph.  With flush
    buffers, the L2 is flushed before every step outside the events (per-step
    events, mean); without, the steps run back to back between one pair of events."""
    import torch
    import torch.distributed as dist
    g = _capture(lambda: wl.step(wl.x))
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    if flush is None:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / steps
    else:
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
        for i in range(steps):
            flush.fill_(i & 0xFF)
            flush_read.sum()
            evs[i][0].record()
            g.replay()
            evs[i][1].record()
        torch.cuda.synchronize()
        ms = float(np.mean([a.elapsed_time(b) for a, b in evs]))
    if world > 1:
        dist.barrier()
    del g
    return ms


def time_e2e(wl, steps, warmup, world=1):
    """The same step end to end through the public API: every step copies its
    activations from pinned host memory to the device and its result (Y, bf16
    [M, N]) and per-modality rel-L2 back.  Copies run on their own streams,
    double-buffered, so step i's compute overlaps step i+1's upload and step i-1's
    download.  Returns (ms per step, h2d bytes, d2h bytes, rel of the last step)."""
    import torch
    import torch.distributed as dist
    x_host = torch.from_numpy(np.ascontiguousarray(wl.layer.x).view(np.int16)).pin_memory()
    x_devs = [torch.empty_like(wl.x) for _ in range(2)]
    y_devs = [torch.empty_like(wl.y) for _ in range(2)]
    y_host = [torch.empty(wl.y.shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    n_seg = len(wl.segs_mod)
    rel_host = [torch.empty(n_seg, dtype=torch.float64).pin_memory() for _ in range(2)]
    comp = torch.cuda.current_stream()
    h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
    copied = [torch.cuda.Event() for _ in range(2)]
    consumed = [torch.cuda.Event() for _ in range(2)]
    computed = [torch.cuda.Event() for _ in range(2)]
    drained = [torch.cuda.Event() for _ in range(2)]

    def upload(i):
        b = i % 2
        with torch.cuda.stream(h2d):
            if i >= 2:
                h2d.wait_event(consumed[b])          # step i - 2 has finished reading x_devs[b]
            x_devs[b].copy_(x_host, non_blocking=True)
            copied[b].record(h2d)

    def compute(i):
        b = i % 2
        comp.wait_event(copied[b])
        if i >= 2:
            comp.wait_event(drained[b])              # step i - 2's output has left y_devs[b]
        res = wl.step(x_devs[b], y_devs[b])
        consumed[b].record(comp)
        computed[b].record(comp)
        with torch.cuda.stream(d2h):
            d2h.wait_event(computed[b])
            y_host[b].copy_(y_devs[b], non_blocking=True)
            rel_host[b].copy_(res[2], non_blocking=True)
            res[2].record_stream(d2h)                # allocated on the compute stream, read here
            drained[b].record(d2h)

    def pipeline(n, start=None):
        if start is not None:
            h2d.wait_event(start)
        upload(0)
        for i in range(n):
            if i + 1 < n:
                upload(i + 1)
            compute(i)
        comp.wait_event(drained[(n - 1) % 2])

    pipeline(max(2, warmup))
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    pipeline(steps, start=e0)
    e1.record(comp)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    last = (steps - 1) % 2
    rel = rel_host[last].tolist()
    # the output that came back to the host is the layer's output of the device-timed step
    same = bool(torch.equal(y_host[last].view(torch.int16), wl.y.cpu().view(torch.int16)))
    h2d_bytes = wl.x.numel() * 2
    d2h_bytes = wl.y.numel() * 2 + 8 * n_seg
    del x_host, x_devs, y_devs, y_host
    return ms, h2d_bytes, d2h_bytes, rel, same


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

    peaks = read_peaks()
    fp4_peak = peaks["bf16"] * FP4_PER_BF16
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_read = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    cfg = args.config
    wl = Workload(P, S, cfg, dev)
    m, k, n, r = wl.m, wl.k, wl.n, wl.r
    for _ in range(args.warmup):
        wl.step(wl.x)
    torch.cuda.synchronize()
    eager_rel = wl.step(wl.x)[2].cpu()

    # ---- device-timed region: inputs resident in HBM.  Inputs larger than L2
    # run back to back; smaller ones get an L2 flush before every step.
    big = wl.x.numel() * 2 > L2_BYTES and wl.w.numel() * 2 > L2_BYTES
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    step_ms = time_step(wl, args.steps, args.warmup, None if big else flush, None if big else flush_read, world)
    clocks = sampler.stop()
    step_ms_max = max_over_ranks(step_ms, dev)
    value = whole_job_tflops(wl.flops, world, step_ms_max)
    graph_rel = wl.score(wl.y)[2].cpu()
    graph_matches_eager = bool(torch.equal(graph_rel, eager_rel))

    # per-call breakdown (each call one graph, cold L2) and the roofline figures
    kern = wl.kernel_times(flush, flush_read, reps=max(5, min(args.steps, 20)))
    fr = wl.fractions(kern, peaks)

    # ---- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        e2e_ms, h2d_b, d2h_b, rel, same = time_e2e(wl, args.steps, args.warmup, world)
        e2e_ms_max = max_over_ranks(e2e_ms, dev)
        e2e = {"value": whole_job_tflops(wl.flops, world, e2e_ms_max), "unit": UNIT, "ms_per_step": e2e_ms_max,
               "h2d_bytes_per_step": h2d_b, "d2h_bytes_per_step": d2h_b, "output_matches_device_step": same,
               "how": "public API, eager calls; each step copies X from pinned host memory to the device and "
                      "Y (bf16) plus the per-modality rel-L2 back to pinned host memory, the copies on their own "
                      "streams overlapping the neighbouring steps' compute (two device buffers each way)"}
    else:
        rel = eager_rel.tolist()
    err = P.svdq_device_error()

    names = [s.name for s in wl.layer.segments]
    layer = wl.layer
    del wl
    torch.cuda.empty_cache()

    # ---- the other configured layers (1 GPU only): the step and its calls
    others = {}
    if world == 1 and not args.no_secondary:
        for c2 in SECONDARY_CONFIGS:
            if c2 == cfg:
                continue
            w2 = Workload(P, S, c2, dev)
            big2 = w2.x.numel() * 2 > L2_BYTES and w2.w.numel() * 2 > L2_BYTES
            ms2 = time_step(w2, max(10, min(args.steps, 20)), args.warmup, None if big2 else flush,
                            None if big2 else flush_read)
            k2 = w2.kernel_times(flush, flush_read, reps=10)
            f2 = w2.fractions(k2, peaks)
            others[WORKLOADS[c2]] = {"M": w2.m, "K": w2.k, "N": w2.n, "rank": w2.r, "ms_per_step": ms2,
                                     "tflops_per_step": w2.flops / (ms2 * 1e-3) / 1e12,
                                     "l2": "back to back (inputs larger than L2)" if big2 else
                                           "flushed before every step", **f2}
            del w2
            torch.cuda.empty_cache()
    per_config = None
    if world == 1 and args.all_configs:
        per_config = all_configs(P, S, dev, fp4_peak, peaks["hbm"], flush, flush_read)
    if world == 1 and (args.all_configs or args.sweep_layers):
        per_config = dict(per_config or {})
        per_config.update(sweep(P, S, dev, fp4_peak, peaks["hbm"], flush, flush_read,
                                n_layers=args.sweep_layers or None))

    line = None
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            # a bounded row sample of the same workload: about 10-20 s of host work
            # (each run also reads and dequantises the whole weight, ~1.5-2 s)
            arm = OracleArm(layer)
            rows = min(layer.m, 2048)
            runs = [arm.run(rows) for _ in range(2)]
            dt = sum(x[1] for x in runs)
            cpu = {"value": 2 * 2.0 * rows * n * k / dt / 1e12, "unit": UNIT, "cores": _oracle_threads(),
                   "kind": "oracle",
                   "sample": f"{rows} evenly spaced of the {m} rows, full K={k} and N={n}, twice ({dt:.1f} s): "
                             "calibration of the sample, quantisation, the W4A4 linear in fp64, scores"}
        lin_tflops = fr["linear_tflops"]
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": step_ms_max, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "nvfp4 (e2m1 x e4m3/16) -> fp32 accum, bf16 out", "data": "synthetic",
            "config": {"workload": WORKLOADS[cfg], "M": m, "K": k, "N": n, "rank": r, "rows_per_gpu": m,
                       "lambda": "calibrated on all rows",
                       "segments": {s.name: [s.begin, s.end] for s in layer.segments},
                       "parallelism": f"replicas x{world}",
                       "l2": ("inputs larger than L2 (X %d MB, W %d MB vs 126 MB): steps back to back" %
                              (m * k * 2 // 10**6, n * k * 2 // 10**6)) if big else
                             "flushed between steps: 256 MiB write, then 256 MiB read (cold, clean L2)",
                       "timing": "the step (calib + quantize + linear + score) as one CUDA graph, CUDA events "
                                 "around the K replays; kernels_ms from one graph per call, cold L2"},
            **fr,
            "roofline": {"bound": "tensor", "kernel": "svdq_linear", "achieved": lin_tflops, "peak": fp4_peak,
                         "unit": "TFLOP/s", "frac": lin_tflops / fp4_peak,
                         "traffic": LINEAR_TRAFFIC_BYTES.get(cfg),
                         "peak_source": f"{peaks['source']} bf16 burst {peaks['bf16']} x {FP4_PER_BF16:g} "
                                        "(nominal dense FP4/BF16 ratio)"},
            "roofline_hbm": {"bound": "hbm", "kernel": "svdq_quantize_act", "achieved": fr["gbs"]["quantize"],
                             "peak": peaks["hbm"], "unit": "GB/s", "frac": fr["frac_of_hbm"]["quantize"],
                             "traffic": QUANTIZE_TRAFFIC_BYTES.get(cfg),
                             "peak_source": f"{peaks['source']} copy bandwidth"},
            "e2e": e2e,
            "gpu_launches": LAUNCHES_PER_STEP * args.steps,
            "clocks": clocks,
            "rel_l2_vs_bf16": dict(zip(names, rel)),
            "device_error": err,
            "graph_replay_matches_eager": graph_matches_eager,
            "other_configs": others or None,
            "all_configs": per_config,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line))
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def all_configs(P, S, dev, fp4_peak, hbm_peak, flush, flush_read):
    """Every call of the path on every configured workload (sweep: one layer per N,
    every lambda candidate), each timed alone from a cold L2."""
    import torch

    def to_dev(a):
        return _to_dev(a, dev)

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


SWEEP_CANDIDATES = ("1", "all", "video", "text")


def sweep(P, S, dev, fp4_peak, hbm_peak, flush, flush_read, n_layers=None):
    """The whole lambda scoring sweep: every layer (K 5120, N cycling 5120 x 4 /
    15360 / 20480, 3 x 4096 rows) x every candidate {1, all, video, text}.

    Per candidate: the calibration (one graph) and the candidate's pass -- the
    activation quantiser and the linear with the per-modality rel-L2 scoring in its
    epilogue, output not written (one graph) -- each timed from a cold L2 and summed
    over the sweep.  The weight conversion of each candidate (randomized rank-32
    factorisation with library QR/SVD, residual, weight quantisation) and the bf16
    reference output of each layer (a cuBLAS GEMM, shared by the candidates) are
    the sweep's preparation and are reported as wall times beside it.  The host
    builds the next layers' inputs on worker threads while the device runs."""
    import torch
    from concurrent.futures import ThreadPoolExecutor

    layers = S.CONFIGS[4]["layers"] if n_layers is None else n_layers
    t_calib = t_pass = 0.0
    flop = q_bytes = s_bytes = c_bytes = 0.0
    conv_s = ref_s = 0.0
    rel_sum = {c: None for c in SWEEP_CANDIDATES}
    names = None
    wall0 = time.perf_counter()
    with ThreadPoolExecutor(max_workers=3) as pool:
        pending = [pool.submit(S.make_layer, 4, None, None, None, l) for l in range(min(3, layers))]
        for l in range(layers):
            L = pending.pop(0).result()
            if l + 3 < layers:
                pending.append(pool.submit(S.make_layer, 4, None, None, None, l + 3))
            x, w, bias = _to_dev(L.x, dev), _to_dev(L.w, dev), _to_dev(L.bias, dev)
            segs_mod = [(sg.begin, sg.end) for sg in L.segments]
            names = [sg.name for sg in L.segments]
            torch.cuda.synchronize()
            t0 = time.perf_counter()
            yref = torch.matmul(x.view(torch.bfloat16), w.view(torch.bfloat16).t()) + bias.view(torch.bfloat16)
            torch.cuda.synchronize()
            ref_s += time.perf_counter() - t0
            wf = torch.empty(P.linear_score_workspace_bytes(len(segs_mod)), dtype=torch.uint8, device=dev)
            for cand in SWEEP_CANDIDATES:
                segs_cal = L.seg_ranges(L.calib_sets["all" if cand == "1" else cand])
                w_cal = None if cand == "1" else w
                t_calib += _graph_ms(lambda: P.svdq_calib_lambda(x, segs_cal, w_cal), flush, flush_read,
                                     reps=3, warmup=3)
                c_bytes += 2.0 * sum(e - b for b, e in segs_cal) * L.k + (2.0 * L.n * L.k if w_cal is not None
                                                                          else 0.0)
                cal = P.svdq_calib_lambda(x, segs_cal, w_cal)
                torch.cuda.synchronize()
                t0 = time.perf_counter()
                lin = P.SVDQW4A4Linear.convert(w, bias, cal, L.rank)
                torch.cuda.synchronize()
                conv_s += time.perf_counter() - t0
                q = P.svdq_quantize_act(x, cal["inv_lam"], lin.s_g_act, lin.down)

                def candidate_pass():
                    P.svdq_quantize_act(x, cal["inv_lam"], lin.s_g_act, lin.down, out=q)
                    return P.svdq_linear_score(q["codes"], q["sf"], lin.s_g_act, q["d"], lin.w_codes, lin.w_sf,
                                               lin.s_g_w, lin.up, lin.bias, yref=yref, segs=segs_mod, out=None,
                                               write_out=False, workspace=wf)
                t_pass += _graph_ms(candidate_pass, flush, flush_read, reps=3, warmup=3)
                rel = candidate_pass()[3].cpu().numpy()
                rel_sum[cand] = rel if rel_sum[cand] is None else rel_sum[cand] + rel
                flop += 2.0 * L.m * L.n * L.k
                q_bytes += (2 + 0.5 + 0.0625) * L.m * L.k + 4.0 * L.m * L.rank
                s_bytes += 2.0 * L.m * L.n * 2          # what a separate scoring pass reads: Yq and Yref
                del cal, lin, q
            del x, w, bias, yref, wf, L
            torch.cuda.empty_cache()
    wall = time.perf_counter() - wall0
    dev_ms = t_calib + t_pass
    return {f"config4_sweep_{layers}_layers_x_{len(SWEEP_CANDIDATES)}_candidates": {
        "layers": layers, "candidates": list(SWEEP_CANDIDATES),
        "gemm_flop": flop, "quantize_bytes": q_bytes, "score_bytes_separate_pass": s_bytes,
        "calib_bytes": c_bytes,
        "device_ms": dev_ms, "calib_ms": t_calib, "quantize_linear_score_ms": t_pass,
        "TFLOP/s_device": flop / (dev_ms * 1e-3) / 1e12,
        "TFLOP/s_quantize_linear_score": flop / (t_pass * 1e-3) / 1e12,
        "frac_fp4_quantize_linear_score": flop / (t_pass * 1e-3) / 1e12 / fp4_peak,
        "calib_GB/s": c_bytes / (t_calib * 1e-3) / 1e9, "calib_frac_hbm": c_bytes / (t_calib * 1e-3) / 1e9 / hbm_peak,
        "weight_conversion_wall_s": conv_s, "bf16_reference_wall_s": ref_s, "wall_s_incl_host_inputs": wall,
        "mean_rel_l2_vs_bf16": {c: dict(zip(names, (rel_sum[c] / layers).tolist())) for c in SWEEP_CANDIDATES},
        "timing": "each call one CUDA graph from a cold L2, median of 3 replays after 3, summed over the sweep"}}


def lambda_search(P, S, dev, flush, flush_read):
    """The 39-candidate lambda search on one sweep layer (rank 32, three modalities):
    wall time of the whole search (host-driven; the randomized rank-32 factorisation of
    every candidate is library QR/SVD), and the grid and bits-lost kernels timed alone."""
    import torch

    def to_dev(a):
        return _to_dev(a, dev)

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


PROFILE_CASES = ("step", "calib", "quantize", "linear", "score", "linear_score", "mxfp8_linear", "mxfp8_quantize")


def profile_case(name: str, cfg: int) -> int:
    """A few launches of one call on one configured workload, for a profiler: two
    warm-up launches, then three (capture with -s 2 -c 1..3 on the kernel's name)."""
    import torch

    import bit_w4a4_quantized_svdq_b200 as P
    import synthetic as S

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    if name in ("mxfp8_linear", "mxfp8_quantize"):
        L = S.make_layer(cfg)
        x, w, bias = _to_dev(L.x, dev), _to_dev(L.w, dev), _to_dev(L.bias, dev)
        qa = P.svdq_quantize_mxfp8(x)
        qw = P.svdq_quantize_mxfp8(w)
        y = torch.empty((L.m, L.n), dtype=torch.bfloat16, device=dev)
        if name == "mxfp8_linear":
            run = lambda: P.svdq_linear_mxfp8(qa["codes"], qa["sf"], qw["codes"], qw["sf"], bias, out=y)
        else:
            run = lambda: P.svdq_quantize_mxfp8(x, out=qa)
    else:
        wl = Workload(P, S, cfg, dev)
        cal = wl.calib(wl.x)
        q = wl.quantize(wl.x, cal)
        if name == "step":
            run = lambda: wl.step(wl.x)
        elif name == "calib":
            run = lambda: wl.calib(wl.x)
        elif name == "quantize":
            run = lambda: wl.quantize(wl.x, cal)
        elif name == "linear":
            run = lambda: wl.linear(q, wl.y)
        elif name == "score":
            run = lambda: wl.score(wl.y)
        else:
            wf = torch.empty(P.linear_score_workspace_bytes(len(wl.segs_mod)), dtype=torch.uint8, device=dev)
            lin = wl.lin
            args = (q["codes"], q["sf"], lin.s_g_act, q["d"], lin.w_codes, lin.w_sf, lin.s_g_w, lin.up, lin.bias)
            run = lambda: P.svdq_linear_score(*args, yref=wl.yref, segs=wl.segs_mod, write_out=False, workspace=wf)
    torch.cuda.synchronize()
    for _ in range(5):
        run()
    torch.cuda.synchronize()
    assert P.svdq_device_error() == 0
    print(json.dumps({"profile_case": name, "config": cfg, "launches": 5}))
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="svdq", choices=["svdq", "reference"])
    ap.add_argument("--config", type=int, default=HEADLINE_CONFIG, choices=sorted(WORKLOADS),
                    help="configured workload of the step (default: the FFN down-projection, the largest)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-secondary", action="store_true", help="skip the other configured layers")
    ap.add_argument("--profile-case", default=None, choices=PROFILE_CASES,
                    help="only launch one call five times on the --config workload (for ncu)")
    ap.add_argument("--all-configs", action="store_true",
                    help="also time every call on every configured workload and the whole lambda "
                         "scoring sweep (adds several minutes)")
    ap.add_argument("--sweep-layers", type=int, default=0,
                    help="also time the lambda scoring sweep over its first N layers")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "svdq":
        args.warmup = 3
    if args.profile_case:
        return profile_case(args.profile_case, args.config)
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
