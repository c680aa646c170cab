"""Benchmark of the FP4 quantized linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--layer I] [--impl ours|reference] [--no-e2e] [--no-cpu-baseline]
                    [--no-graph]

A step is one forward pass of every linear layer of the workload (default:
the 7B decoder block's four linears at M = 16384 tokens, bf16, the largest
configuration; its clamp quantile alpha = 0.99 is the headline and every other
alpha of the workload, 0.999, is measured the same way and reported in
`alpha_sweep`): for each layer the
weight is quantized column-wise (the method quantizes W and A at the start of
every linear forward), then the activation goes through the fused threshold /
clamp / quantize pass, the dA . W correction and the FP4 GEMM with its
dequantization epilogue.  Inputs are synthetic (seeded, see workloads/) and
resident in HBM before timing; L2 is flushed (256 MiB write) between timed
steps.  The step's library calls are captured once into a CUDA graph and the
graph is replayed once per timed step (the cooperative and cluster launches
capture like any other); the step time is the device time between two events
around each replay.  Per-kernel times come from a second pass over the same
steps, launched eagerly with events between the calls (`kernels`,
`roofline`; those intervals also carry the launch gaps the events add, so
they sum to `breakdown_ms_per_step`, a little above `ms_per_step`).  One JSON
line is printed by rank 0.

Multi-GPU: one process per GPU (torchrun); every rank runs its own replica of
the workload (weak scaling, no data-path collective); the timed region is
bracketed by barrier + synchronize and the max over ranks is reported.

--impl reference times the CPU oracle (the plain C restatement of the method)
on the host cores, on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

METRIC = "FP4 linear-layer TFLOPS & tokens/s (1 B200); quantizer GB/s; % roofline"
L2_FLUSH_BYTES = 256 << 20


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return dict(hbm_gbs=float(p["hbm_gbs"]), bf16_tflops=float(p["bf16_tflops"]),
                    bf16_tflops_sustained=float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                    sm_max_mhz=float(p.get("sm_max_mhz", 1965.0)), source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0,
                sm_max_mhz=1965.0, source="fallback")


# ------------------------------------------------------------------ ranks
def max_over_ranks(x: float, world: int, device=None) -> float:
    """The largest value of x over all ranks (x itself on one rank).  Uses a
    device tensor under NCCL and a host tensor under gloo."""
    if world <= 1:
        return float(x)
    import torch.distributed as dist
    dev = device if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(work_per_rank_per_step: float, steps: int, max_ms: float,
                       world: int) -> float:
    """Whole-job throughput: the work all ranks did over the slowest rank's
    time (units of work per second)."""
    return world * work_per_rank_per_step * steps / (max_ms * 1e-3)


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"qg_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.f,
                stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                except ValueError:
                    continue
                for name, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(name)
        os.remove(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "samples": len(sm), "reasons": sorted(reasons)}


# ------------------------------------------------------------------ our arm
class Layer:
    """One linear of the workload with its buffers.  The CSR and workspaces are
    sized for the smallest alpha in `size_alphas` (the most clamped entries),
    so the same buffers serve every alpha of a sweep."""

    def __init__(self, qg, wl, li, device, alpha=None, size_alphas=()):
        from workloads import make_layer_inputs
        self.name = wl.layers[li].name
        self.A, self.W = make_layer_inputs(wl, li, device=device)
        self.alpha = wl.alphas[0] if alpha is None else alpha
        M, K = self.A.shape
        N = self.W.shape[1]
        self.M, self.K, self.N = M, K, N
        dt = qg._dt(self.A)
        a_size = min([self.alpha, *size_alphas])
        self.a_size = a_size
        cap = qg.qg_nnz_capacity(M * K, a_size)
        self.codesT = torch.empty((N, K // 2), dtype=torch.uint8, device=device)
        self.t = torch.empty(N, dtype=torch.float32, device=device)
        self.codes = torch.empty((M, K // 2), dtype=torch.uint8, device=device)
        self.s = torch.empty(M, dtype=torch.float32, device=device)
        self.csr = qg.CSR.empty(M, cap, device=device)
        self.T = torch.empty(1, dtype=torch.float32, device=device)
        self.Y = torch.empty((M, N), dtype=torch.float32, device=device)
        self.ws_cols = qg.Workspace(qg.QG_OP_QUANTIZE_COLS, 1, K, N, dt, device=device)
        self.ws_act = qg.Workspace(qg.QG_OP_QUANTIZE_ACT, M, K, 1, dt, a_size, device=device)
        self.ws_spmm = qg.Workspace(qg.QG_OP_SPMM, M, K, N, dt, device=device)
        self.ws_gemm = qg.Workspace(qg.QG_OP_FP4_GEMM, M, K, N, qg.QG_F32, device=device)
        self.ws_lin = None          # allocated by the e2e arm
        self.dt = dt
        self.flops = 2 * M * N * K
        self.a_bytes = M * K * self.A.element_size()
        self.w_bytes = K * N * self.W.element_size()

    def workspaces(self):
        return tuple(w for w in (self.ws_cols, self.ws_act, self.ws_spmm, self.ws_gemm, self.ws_lin)
                     if w is not None)


KERNELS = ("quantize_cols", "quantize_act", "spmm", "fp4_gemm")


def layer_order(qg, L):
    """The order of the layer's four calls, as qg_fp4_linear runs them for
    fp32 Y: with many clamped entries per row the GEMM writes Y and the SpMM
    adds the compensation into it; otherwise the SpMM writes the compensation
    into Y and the GEMM adds its product into it (qg_fp4_gemm_accumulate; in
    place through C = Y when N is not a multiple of 4)."""
    if qg.linear_adds_into_y(L.M, L.K, L.alpha):
        return ("quantize_cols", "quantize_act", "fp4_gemm", "spmm")
    return ("quantize_cols", "quantize_act", "spmm", "fp4_gemm")


def run_step(qg, layers, ev=None):
    """One pass of the hot path over every layer, the calls qg_fp4_linear
    makes for fp32 Y: the weight quantizer, the fused activation quantizer
    (threshold, clamp, dA, codes), then the compensation dA . W and the FP4
    GEMM into Y in the layer's order (layer_order).  With `ev`, record events
    around each of the four calls of each layer (same stream)."""
    def _chk(st, where):
        if st != qg.QG_OK:
            raise qg.QGError(st, where)

    def call(L, name):
        if name == "quantize_cols":
            _chk(qg.qg_quantize_cols(L.W, L.codesT, L.t, L.ws_cols), name)
        elif name == "quantize_act":
            _chk(qg.qg_quantize_act(L.A, L.alpha, L.codes, L.s, L.csr, L.T, L.ws_act), name)
        elif name == "spmm":
            if L.adds:
                _chk(qg.qg_spmm_accumulate(L.csr, L.M, L.W, L.Y, L.ws_spmm), name)
            else:
                _chk(qg.qg_spmm_correction(L.csr, L.M, L.W, L.Y, L.ws_spmm), name)
        elif L.adds:
            _chk(qg.qg_fp4_gemm(L.codes, L.s, L.codesT, L.t, L.M, L.N, L.K, None, L.Y, None,
                                L.ws_gemm), name)
        elif L.N % 4 == 0:
            _chk(qg.qg_fp4_gemm_accumulate(L.codes, L.s, L.codesT, L.t, L.M, L.N, L.K, L.Y,
                                           L.ws_gemm), name)
        else:
            _chk(qg.qg_fp4_gemm(L.codes, L.s, L.codesT, L.t, L.M, L.N, L.K, L.Y, L.Y, None,
                                L.ws_gemm), name)

    for i, L in enumerate(layers):
        order = layer_order(qg, L)
        L.adds = order[2] == "fp4_gemm"
        L.order = order
        if ev is not None:
            ev[i][0].record()
        for j, name in enumerate(order):
            call(L, name)
            if ev is not None:
                ev[i][j + 1].record()


def capture_step(qg, layers):
    """Capture one step (run_step) into a CUDA graph.  Returns (graph, library
    launches in the step), or (None, None) when capture is not available;
    the captured step is replayed once and must leave the workspaces' status
    clean."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    try:
        with torch.cuda.stream(side):
            run_step(qg, layers)         # on the capture stream once before capturing
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        n1 = qg.qg_launch_count()
        with torch.cuda.graph(graph):
            run_step(qg, layers)
        per_step = qg.qg_launch_count() - n1
        graph.replay()
        torch.cuda.synchronize()
        for L in layers:
            for ws in L.workspaces():
                qg.check_status(ws, f"graph {L.name}")
    except Exception as ex:   # capture unsupported here: run eagerly
        print(f"bench: CUDA graph capture unavailable ({type(ex).__name__}); eager launches",
              file=sys.stderr)
        torch.cuda.synchronize()
        return None, None
    return graph, per_step


def _measure(qg, layers, steps, flush, world, device, no_graph):
    """Time `steps` steps of the hot path.  Region 1 (the headline): the
    step's library calls captured once into a CUDA graph and replayed once per
    step, each replay between two events on the stream (eager launches
    without graph support).  Region 2 (the breakdown): the same steps launched
    eagerly with events between the calls, for per-kernel times (those
    intervals also hold the launch gaps the events add).  Returns the step
    times, the per-kernel times per step, the library launches of region 1,
    the clocks sampled over both regions and whether a graph was used."""
    n_l = len(layers)
    graph, launches_per_step = (None, None) if no_graph else capture_step(qg, layers)
    ev_step = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(steps)]
    ev_steps = [[[torch.cuda.Event(enable_timing=True) for _ in range(len(KERNELS) + 1)]
                 for _ in range(n_l)] for _ in range(steps)]
    sampler = ClockSampler(torch.cuda.current_device() if world == 1 else int(os.environ.get("LOCAL_RANK", 0)))
    sampler.start()
    time.sleep(0.3)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    launches0 = qg.qg_launch_count()
    for k in range(steps):
        flush.fill_(k & 0xFF)           # L2 flush outside the step's events
        ev_step[k][0].record()
        if graph is not None:
            graph.replay()
        else:
            run_step(qg, layers)
        ev_step[k][1].record()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    wall = time.perf_counter() - wall0
    launches = (launches_per_step * steps if graph is not None
                else qg.qg_launch_count() - launches0)
    for k in range(steps):              # region 2
        flush.fill_(k & 0xFF)
        run_step(qg, layers, ev_steps[k])
    torch.cuda.synchronize()
    clocks = sampler.stop()
    for L in layers:
        for ws in L.workspaces():
            qg.check_status(ws, f"timed {L.name}")
    used_graph = graph is not None
    del graph
    step_ms = [a.elapsed_time(b) for a, b in ev_step]
    per_kernel = {k: [] for k in KERNELS}
    per_layer = {k: [0.0] * n_l for k in KERNELS}
    for ev in ev_steps:
        for kn in KERNELS:
            t = []
            for i in range(n_l):
                j = layers[i].order.index(kn)
                t.append(ev[i][j].elapsed_time(ev[i][j + 1]))
            per_kernel[kn].append(sum(t))
            for i in range(n_l):
                per_layer[kn][i] += t[i] / steps
    return dict(step_ms=step_ms, per_kernel=per_kernel, per_layer=per_layer,
                launches=int(launches), clocks=clocks, graph=used_graph, wall=wall)


def _mma_loop_peak():
    """The E2M1 rate measured by the library's MMA-only loop (2-SM pairs, the
    GEMM's form for M > 128), from the committed summary, or None."""
    path = os.path.join(ROOT, "profiles", "fp4_mma_peak.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        return float(json.load(f)["pair_tflops"])


def _kernel_rows(layers, per_kernel, steps, peaks, sm_mhz, n_sm):
    """Each kernel's achieved rate against the roofline that bounds it: its
    algorithmic bytes or flops per step (defined below, per kernel) over its
    measured time per step."""
    fp4_peak = 4.0 * peaks["bf16_tflops"]             # burst: a sub-second kernel
    alu_peak = n_sm * 128 * 2 * sm_mhz * 1e6 / 1e12
    rows = {}
    for k in KERNELS:
        kms = sum(per_kernel[k]) / steps
        t = kms * 1e-3
        if k == "fp4_gemm":
            # the GEMM moves the FP4 codes, the scales and Y: written only
            # when it runs first, read and written (by the memory system's
            # reduction, or in place) when the SpMM wrote Y first; its bound is
            # whichever of the tensor-core time and the HBM time is longer
            flops = sum(L.flops for L in layers)
            byts = sum(L.M * L.K / 2 + L.N * L.K / 2 + 4 * (L.M + L.N)
                       + (4 if L.adds else 8) * L.M * L.N for L in layers)
            t_tensor = flops / (fp4_peak * 1e12)
            t_hbm = byts / (peaks["hbm_gbs"] * 1e9)
            if t_tensor >= t_hbm:
                bound, unit, peak, algo = "tensor", "TFLOP/s", fp4_peak, flops / 1e12
            else:
                bound, unit, peak, algo = "hbm", "GB/s", peaks["hbm_gbs"], byts / 1e9
            loop = _mma_loop_peak()
            extra = {"tflops": round(flops / t / 1e12, 1) if t > 0 else 0.0,
                     "frac_of_9pf_datasheet": round(flops / t / 9e15, 4) if t > 0 else 0.0,
                     "frac_of_mma_loop": (round(flops / t / 1e12 / loop, 4)
                                          if t > 0 and loop else None),
                     "ceilings_ms": {"tensor": round(1e3 * t_tensor, 4), "hbm": round(1e3 * t_hbm, 4)}}
        elif k == "spmm":
            # 2 nnz N fp32 FMA flops; every entry gathers its W row segment
            # (nnz N elements) from L2; Y is written (4 M N bytes) or, in the
            # GEMM-first order, read and written by the memory system's adds
            algo = sum(2 * int(L.csr.nnz.item()) * L.N for L in layers) / 1e12
            bound, unit, peak = "alu", "TFLOP/s", alu_peak
            extra = {"w_row_gather_bytes": sum(int(L.csr.nnz.item()) * L.N * L.W.element_size()
                                               for L in layers)}
        elif k == "fp4_gemm_compensated":
            # three ceilings: the FP4 MMAs on the tensor cores (2 M N K), the
            # compensation's fp32 FMAs on the CUDA cores (2 nnz N), and the
            # HBM bytes (codes, scales, the CSR, W read once, Y written); the
            # kernel's roofline time is the largest of the three
            flops = sum(L.flops for L in layers)
            alu_flops = sum(2 * int(L.csr.nnz.item()) * L.N for L in layers)
            byts = sum(L.M * L.K / 2 + L.N * L.K / 2 + 4 * (L.M + L.N) + 4 * (L.M + 1)
                       + 12 * int(L.csr.nnz.item()) + L.w_bytes
                       + L.Y.element_size() * L.M * L.N for L in layers)
            t_tensor = flops / (fp4_peak * 1e12)
            t_alu = alu_flops / (alu_peak * 1e12)
            t_hbm = byts / (peaks["hbm_gbs"] * 1e9)
            worst = max(t_tensor, t_alu, t_hbm)
            if worst == t_tensor:
                bound, unit, peak, algo = "tensor", "TFLOP/s", fp4_peak, flops / 1e12
            elif worst == t_alu:
                bound, unit, peak, algo = "alu", "TFLOP/s", alu_peak, alu_flops / 1e12
            else:
                bound, unit, peak, algo = "hbm", "GB/s", peaks["hbm_gbs"], byts / 1e9
            loop = _mma_loop_peak()
            extra = {"fp4_tflops": round(flops / t / 1e12, 1) if t > 0 else 0.0,
                     "frac_of_9pf_datasheet": round(flops / t / 9e15, 4) if t > 0 else 0.0,
                     "frac_of_mma_loop": (round(flops / t / 1e12 / loop, 4)
                                          if t > 0 and loop else None),
                     "compensation_tflops": round(alu_flops / t / 1e12, 2) if t > 0 else 0.0,
                     "ceilings_ms": {"tensor": round(1e3 * t_tensor, 4),
                                     "alu": round(1e3 * t_alu, 4), "hbm": round(1e3 * t_hbm, 4)},
                     "w_row_gather_bytes": sum(int(L.csr.nnz.item()) * L.N * L.W.element_size()
                                               for L in layers)}
        elif k == "quantize_act":
            algo = sum(2 * L.a_bytes + L.M * L.K / 2 + 4 * L.M + 16 * int(L.csr.nnz.item())
                       + 4 * (L.M + 1) + 8 * L.M for L in layers) / 1e9
            bound, unit, peak = "hbm", "GB/s", peaks["hbm_gbs"]
            extra = {}
        else:
            algo = sum(2 * L.w_bytes + L.K * L.N / 2 + 4 * L.N for L in layers) / 1e9
            bound, unit, peak = "hbm", "GB/s", peaks["hbm_gbs"]
            extra = {}
        achieved = algo / t if kms > 0 else 0.0
        if bound == "hbm" and k != "fp4_gemm":
            # the quantizers' stated target is a fraction of the nominal 8 TB/s
            extra["frac_of_8tbs_nominal"] = round(achieved / 8000.0, 4)
        rows[k] = {"bound": bound, "achieved": round(achieved, 2), "peak": round(peak, 1),
                   "unit": unit, "frac": round(achieved / peak, 4), "ms_per_step": round(kms, 4),
                   **extra}
    return rows, fp4_peak


def our_arm(args, rank, world, device):
    import quantize_gemm_b200 as qg
    from workloads import WORKLOADS
    wl = WORKLOADS[args.workload]
    peaks = _peaks()
    alphas = [args.alpha] if args.alpha is not None else list(wl.alphas)
    idx = range(len(wl.layers)) if args.layer is None else [args.layer]
    layers = [Layer(qg, wl, i, device, alphas[0], size_alphas=alphas) for i in idx]
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    n_sm = torch.cuda.get_device_properties(device).multi_processor_count
    flops_step = sum(L.flops for L in layers)
    tokens_step = wl.M          # tokens through the layers of the step

    def warm():
        for _ in range(args.warmup):
            run_step(qg, layers)
        torch.cuda.synchronize()
        for L in layers:
            for ws in L.workspaces():
                qg.check_status(ws, f"warm-up {L.name}")

    results = []
    for a in alphas:
        for L in layers:
            L.alpha = a
        warm()
        orders = [list(L.order) for L in layers]
        m = _measure(qg, layers, args.steps, flush, world, device, args.no_graph)
        total_ms = max_over_ranks(sum(m["step_ms"]), world, device)
        sm_mhz = m["clocks"].get("sm_mhz") or peaks["sm_max_mhz"]
        rows, fp4_peak = _kernel_rows(layers, m["per_kernel"], args.steps, peaks, sm_mhz, n_sm)
        for k in rows:
            rows[k]["ms_per_layer"] = [round(x, 4) for x in m["per_layer"][k]]
        nnz = [int(L.csr.nnz.item()) for L in layers]
        results.append(dict(alpha=a, m=m, total_ms=total_ms, rows=rows, fp4_peak=fp4_peak,
                            sm_mhz=sm_mhz, nnz=nnz, orders=orders))

    head = results[0]
    m, rows, total_ms = head["m"], head["rows"], head["total_ms"]
    for L in layers:
        L.alpha = head["alpha"]
        L.order = tuple(head["orders"][layers.index(L)])
        L.adds = L.order[2] == "fp4_gemm"
    ms_per_step = total_ms / args.steps
    value = weak_scaling_value(flops_step, args.steps, total_ms, world) / 1e12
    dominant = max(KERNELS, key=lambda k: rows[k]["ms_per_step"])
    traffic = _ncu_traffic(dominant, args.workload)
    roofline = {k: v for k, v in rows[dominant].items() if k in ("bound", "achieved", "peak", "unit", "frac")}
    roofline["kernel"] = dominant
    roofline["traffic"] = traffic
    bound = rows[dominant]["bound"]
    roofline["peak_source"] = (
        f"{peaks['source']}: 4 x bf16 burst {peaks['bf16_tflops']} (FP4:bf16 nominal ratio)"
        if bound == "tensor" else f"{peaks['source']} HBM copy" if bound == "hbm" else
        f"SMs x 128 FMA x 2 x median SM clock {head['sm_mhz']} MHz")
    out = {
        "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "e2m1",
        "data": "synthetic",
        "config": dict(workload_config(wl, layers, head["alpha"], args.layer is not None),
                       l2="flushed (256 MiB write between timed steps)",
                       parallelism=f"replicas x{world}"),
        "tokens_per_s": round(weak_scaling_value(tokens_step, args.steps, total_ms, world), 1),
        "quantizer_gbs": rows["quantize_act"]["achieved"],
        "kernels": rows,
        "roofline": roofline,
        "clocks": m["clocks"],
        "gpu_launches": m["launches"],
        "cuda_graph": m["graph"],
        "nnz_per_layer": head["nnz"],
        "call_order": [list(L.order) for L in layers],
        "breakdown_ms_per_step": round(sum(sum(v) for v in m["per_kernel"].values()) / args.steps, 4),
        "wall_s": round(m["wall"], 3),
    }
    if len(results) > 1:
        out["alpha_sweep"] = [
            {"alpha": r["alpha"], "value": round(weak_scaling_value(flops_step, args.steps, r["total_ms"], world) / 1e12, 3),
             "unit": "TFLOP/s", "ms_per_step": round(r["total_ms"] / args.steps, 4),
             "tokens_per_s": round(weak_scaling_value(tokens_step, args.steps, r["total_ms"], world), 1),
             "nnz_per_layer": r["nnz"], "gpu_launches": r["m"]["launches"],
             "call_order": r["orders"],
             "kernels": {k: {kk: v[kk] for kk in ("ms_per_step", "achieved", "unit", "frac", "bound")}
                         for k, v in r["rows"].items()},
             "clocks": r["m"]["clocks"]}
            for r in results[1:]]
    if not args.no_e2e:
        out["e2e"] = e2e_arm(qg, args, layers, device, world)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(args, wl, layers)
    return out


def e2e_arm(qg, args, layers, device, world):
    """Same metric through the public call qg_fp4_linear with host buffers:
    pinned host A -> device, weight quantization, the layer, Y -> pinned host,
    all inside the timed region.  Uploads run on one copy stream, downloads on
    another, the layers on the compute stream, ordered by events, so the PCIe
    transfers of one layer overlap the computation of its neighbours."""
    for L in layers:
        if L.ws_lin is None:
            L.ws_lin = qg.Workspace(qg.QG_OP_FP4_LINEAR, L.M, L.K, L.N, L.dt, L.a_size, device=device)
    hostA = [L.A.cpu().pin_memory() for L in layers]
    hostY = [torch.empty(L.Y.shape, dtype=L.Y.dtype).pin_memory() for L in layers]
    devA = [torch.empty_like(L.A) for L in layers]
    cs = torch.cuda.current_stream()
    hs = torch.cuda.Stream(device=device)
    ds = torch.cuda.Stream(device=device)
    n = len(layers)
    ev_up = [torch.cuda.Event() for _ in range(n)]
    ev_done = [torch.cuda.Event() for _ in range(n)]
    ev_down = [torch.cuda.Event() for _ in range(n)]
    started = [False]

    def step(t0=None, t1=None):
        if t0 is not None:
            t0.record(cs)
        start = torch.cuda.Event()
        start.record(cs)
        hs.wait_event(start)
        for i in range(n):
            if started[0]:
                hs.wait_event(ev_done[i])       # the last step has finished reading devA[i]
            with torch.cuda.stream(hs):
                devA[i].copy_(hostA[i], non_blocking=True)
            ev_up[i].record(hs)
        for i, L in enumerate(layers):
            cs.wait_event(ev_up[i])
            if started[0]:
                cs.wait_event(ev_down[i])       # the last step's Y[i] has left the device
            st = qg.qg_quantize_cols(L.W, L.codesT, L.t, L.ws_cols)
            if st != qg.QG_OK:
                raise qg.QGError(st, "e2e quantize_cols")
            st = qg.qg_fp4_linear(devA[i], L.codesT, L.t, L.W, L.alpha, L.Y, L.ws_lin)
            if st != qg.QG_OK:
                raise qg.QGError(st, "e2e fp4_linear")
            ev_done[i].record(cs)
            ds.wait_event(ev_done[i])
            with torch.cuda.stream(ds):
                hostY[i].copy_(L.Y, non_blocking=True)
            ev_down[i].record(ds)
        for i in range(n):
            cs.wait_event(ev_down[i])
        started[0] = True
        if t1 is not None:
            t1.record(cs)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    total = 0.0
    e2e_steps = max(10, args.steps // 10)
    for k in range(e2e_steps):
        flush.fill_(k & 0xFF)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        step(a, b)
        torch.cuda.synchronize()
        total += a.elapsed_time(b)
    for L in layers:
        qg.check_status(L.ws_lin, "e2e")
    total = max_over_ranks(total, world, device)
    flops = sum(L.flops for L in layers)
    return {"value": round(weak_scaling_value(flops, e2e_steps, total, world) / 1e12, 3),
            "unit": "TFLOP/s", "steps": e2e_steps,
            "h2d_bytes_per_step": int(sum(L.a_bytes for L in layers)),
            "d2h_bytes_per_step": int(sum(L.Y.numel() * L.Y.element_size() for L in layers)),
            "ms_per_step": round(total / e2e_steps, 4),
            "overlap": "uploads, layers and downloads on three streams ordered by events"}


def _ncu_traffic(kernel, workload):
    """DRAM bytes of one step (the kernel's launches over the workload's
    layers, the unit `achieved` is counted in) from a committed ncu summary,
    when it was taken on the current source of that kernel (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    import hashlib
    with open(path) as f:
        data = json.load(f)
    rec = data.get(f"{kernel}:{workload}")
    if not rec:
        return None
    src = os.path.join(ROOT, rec["source"])
    if not os.path.exists(src):
        return None
    with open(src, "rb") as f:
        sha = hashlib.sha256(f.read()).hexdigest()[:16]
    return rec.get("dram_bytes_per_step") if sha == rec["source_sha256_16"] else None


# ------------------------------------------------------------------ CPU oracle
def _oracle_sample(wl, A_list, W_list, frac, alpha=None, step=0):
    """Time the oracle on a bounded sample of one step and return the seconds
    the whole step would take.  For each layer a fraction `frac` of the work:
    the activation quantizer (threshold, clamp, dA, row codes) on a slice of
    about frac * M rows, the W quantizer on about frac * N columns, Y for about
    frac * M evenly spaced rows; each part's time is scaled by its inverse
    fraction.  `step` rotates the slices through the tensors.  frac = 1 runs
    the quantizers on the full tensors (Y is then sampled by `_Y_ROWS_FULL`)."""
    import oracle
    t_total = 0.0
    alpha = wl.alphas[0] if alpha is None else alpha
    for A, W in zip(A_list, W_list):
        M, K = A.shape
        N = W.shape[1]
        ra = M if frac >= 1 else max(32, min(M, int(round(frac * M))))
        cs = N if frac >= 1 else max(32, min(N, int(round(frac * N))))
        ry = _Y_ROWS_FULL if frac >= 1 else max(1, min(M, int(round(frac * M))))
        r0 = (step * ra) % (M - ra + 1)
        c0 = (step * cs) % (N - cs + 1)
        A_s = A[r0:r0 + ra]
        W_s = W if cs == N else np.ascontiguousarray(W[:, c0:c0 + cs])
        t0 = time.perf_counter()
        act = oracle.quantize_act(A_s, alpha)
        t1 = time.perf_counter()
        oracle.quantize_cols(W_s)
        t2 = time.perf_counter()
        # Y needs the codes of all N columns; their time is the W quantizer's,
        # already sampled above, so the full-column codes are made untimed.
        oT, ot = _codes_cache(W)
        rows = (np.linspace(0, ra - 1, ry).astype(np.int64) + step) % ra
        t3 = time.perf_counter()
        acc = oracle.gemm_acc(act["codes"], oT, K, rows=rows)
        oracle.linear_y(acc, act["scales"], ot, act["row_ptr"], act["col"], act["val"], W, rows=rows)
        t4 = time.perf_counter()
        t_total += (t1 - t0) * (M / ra) + (t2 - t1) * (N / cs) + (t4 - t3) * (M / ry)
    return t_total


_Y_ROWS_FULL = 16
_CODES = {}


def _codes_cache(W):
    """The oracle's column codes of W, computed once per weight."""
    import oracle
    key = id(W)
    if key not in _CODES:
        _CODES[key] = oracle.quantize_cols(W)
    return _CODES[key]


CPU_BASELINE_BUDGET_S = 15.0   # host seconds the cpu_baseline sample aims for


def cpu_baseline(args, wl, layers):
    """The oracle as it stands, on the host cores, on a bounded sample of one
    step of the workload: a probe sample sets the fraction f of each layer's
    work (rows of A for the activation quantizer and for Y, columns of W for
    the weight quantizer) that takes about CPU_BASELINE_BUDGET_S seconds; each
    part's time is scaled by its inverse fraction to the whole step."""
    import oracle
    A_list = [oracle.as_f32(L.A.cpu()) for L in layers]
    W_list = [oracle.as_f32(L.W.cpu()) for L in layers]
    alpha = layers[0].alpha
    for W in W_list:
        _codes_cache(W)
    t_probe = _oracle_sample(wl, A_list, W_list, 1.0 / 1024, alpha)
    frac = min(1.0, CPU_BASELINE_BUDGET_S / max(t_probe, 1e-9))
    w0 = time.perf_counter()
    t_est = _oracle_sample(wl, A_list, W_list, frac, alpha)
    wall = time.perf_counter() - w0
    flops = sum(L.flops for L in layers)
    if frac >= 1:
        sample = (f"one step of {wl.name}: quantizers (threshold, clamp, dA, row and column "
                  f"codes) on the full tensors; Y for {_Y_ROWS_FULL} evenly spaced rows per "
                  f"layer, its time scaled by M/{_Y_ROWS_FULL}")
    else:
        sample = (f"one step of {wl.name}, alpha {alpha}: on every layer a fraction {frac:.3g} "
                  f"of the work (activation quantizer, threshold included, on a slice of "
                  f">= 32 rows; W quantizer on >= 32 columns; Y for >= 1 row), each part's "
                  f"time scaled by its inverse fraction; {wall:.1f} s of host time")
    return {"value": round(flops / t_est / 1e12, 6), "unit": "TFLOP/s",
            "cores": oracle.num_threads(), "kind": "oracle", "sample": sample,
            "sample_fraction": round(frac, 6), "sample_wall_s": round(wall, 2),
            "seconds_per_step_estimate": round(t_est, 3)}


def workload_config(wl, layers, alpha, one_layer=False):
    """The `config` keys both arms share: the workload, its shapes, alpha and
    the input and output dtypes."""
    return {"workload": f"{wl.name}:{layers[0].name}" if one_layer else wl.name,
            "description": wl.description, "M": wl.M,
            "layers": [[L.name, L.K, L.N] for L in layers], "alpha": alpha,
            "input_dtype": wl.dtype, "y_dtype": "f32"}


REFERENCE_BUDGET_S = 150.0   # wall time the reference arm's warm-up + timed steps aim for


def reference_arm(args, rank, world):
    """The CPU oracle as the reference arm (rank 0 only).  Every step times the
    oracle on a sample of the step whose size is set so that the W warm-up and
    K timed steps together take about REFERENCE_BUDGET_S seconds; the value is
    the step's FLOPs over the step time the samples stand for."""
    from workloads import WORKLOADS, make_layer_inputs
    import oracle
    wl = WORKLOADS[args.workload]
    idx = list(range(len(wl.layers))) if args.layer is None else [args.layer]
    A_list, W_list = [], []
    for i in idx:
        A, W = make_layer_inputs(wl, i, device="cpu")
        A_list.append(oracle.as_f32(A))
        W_list.append(oracle.as_f32(W))
    for W in W_list:
        _codes_cache(W)
    # calibrate: one small sample gives the full step's estimated time
    probe = 1.0 / 256
    t_step = _oracle_sample(wl, A_list, W_list, probe, args.alpha)
    n_runs = max(1, args.steps + args.warmup)
    frac = min(1.0, REFERENCE_BUDGET_S / n_runs / max(t_step, 1e-9))
    for s in range(args.warmup):
        _oracle_sample(wl, A_list, W_list, frac, args.alpha, step=s)
    total = 0.0
    for s in range(args.steps):
        total += _oracle_sample(wl, A_list, W_list, frac, args.alpha, step=args.warmup + s)
    flops = sum(2 * wl.M * wl.layers[i].K * wl.layers[i].N for i in idx)
    value = flops * args.steps / total / 1e12
    cores = oracle.num_threads()
    if frac >= 1:
        sample = (f"each step: quantizers on the full tensors of every {wl.name} layer, Y for "
                  f"{_Y_ROWS_FULL} evenly spaced rows per layer with its time scaled by "
                  f"M/{_Y_ROWS_FULL}")
    else:
        sample = (f"each step: on every {wl.name} layer, a fraction {frac:.3g} of the work "
                  f"(activation quantizer on a slice of >= 32 rows, W quantizer on >= 32 "
                  f"columns, Y for >= 1 row; slices rotate across steps), each part's time "
                  f"scaled by its inverse fraction; sized so the {args.warmup} + {args.steps} "
                  f"steps take about {REFERENCE_BUDGET_S:.0f} s")
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * total / args.steps, 3),
        "ms_per_step_kind": ("estimate: each step times the oracle on a sample of the step and "
                             "scales each part's time by its inverse sample fraction"
                             if frac < 1 else "measured quantizers; Y rows sampled and scaled"),
        "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(workload_config(wl, [wl.layers[i] for i in idx],
                                       wl.alphas[0] if args.alpha is None else args.alpha,
                                       args.layer is not None),
                       parallelism="rank 0 only, on the host cores"),
        "cpu_baseline": {"kind": "oracle", "cores": cores, "sample": sample,
                         "value": round(value, 6), "unit": "TFLOP/s"},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def quantizer_sweep(device, reps=20, warm=5):
    """The quantizers alone over A = M x 4096 bf16, Student-t(3), M = 256 * 2^j
    (1M .. 256M elements), alpha = 0.99; quantize_cols on a 4096 x M weight of
    the same element count.  Median of `reps` CUDA-event timings, L2 flushed
    (256 MiB write) before each; GB/s from algorithmic bytes."""
    import quantize_gemm_b200 as qg
    from workloads import make_matrix
    peaks = _peaks()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)

    def timed(fn):
        for _ in range(warm):
            fn()
        ts = []
        for _ in range(reps):
            flush.fill_(1)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        ts.sort()
        return ts[len(ts) // 2]

    K, alpha = 4096, 0.99
    for j in range(9):
        M = 256 * 2 ** j
        n = M * K
        A = make_matrix((M, K), ("student_t", 3), seed=5000 + j, device=device, dtype=torch.bfloat16)
        codes = torch.empty((M, K // 2), dtype=torch.uint8, device=device)
        s = torch.empty(M, dtype=torch.float32, device=device)
        ws_r = qg.Workspace(qg.QG_OP_QUANTIZE_ROWS, M, K, 1, qg.QG_BF16, device=device)
        t_rows = timed(lambda: qg.qg_quantize_rows(A, codes, s, ws_r))
        ws_a = qg.Workspace(qg.QG_OP_QUANTIZE_ACT, M, K, 1, qg.QG_BF16, alpha, device=device)
        csr = qg.CSR.empty(M, qg.qg_nnz_capacity(n, alpha), device=device)
        T = torch.empty(1, dtype=torch.float32, device=device)
        t_act = timed(lambda: qg.qg_quantize_act(A, alpha, codes, s, csr, T, ws_a))
        qg.check_status(ws_a, "sweep quantize_act")
        nnz = int(csr.nnz.item())
        del A, csr, ws_a, ws_r
        W = make_matrix((K, M), ("normal",), seed=6000 + j, device=device, dtype=torch.bfloat16,
                        scale=0.02)
        codesT = torch.empty((M, K // 2), dtype=torch.uint8, device=device)
        tw = torch.empty(M, dtype=torch.float32, device=device)
        ws_c = qg.Workspace(qg.QG_OP_QUANTIZE_COLS, 1, K, M, qg.QG_BF16, device=device)
        t_cols = timed(lambda: qg.qg_quantize_cols(W, codesT, tw, ws_c))
        qg.check_status(ws_c, "sweep quantize_cols")
        del W, ws_c, codesT, codes
        torch.cuda.empty_cache()
        by = {"quantize_rows": 2 * n + n / 2 + 4 * M,
              "quantize_act": 2 * 2 * n + n / 2 + 4 * M + 16 * nnz + 4 * (M + 1) + 8 * M,
              "quantize_cols": 2 * 2 * n + n / 2 + 4 * M}
        line = {"sweep": "quantizers", "elements": n, "M": M, "K": K, "alpha": alpha, "nnz": nnz,
                "dtype": "bf16", "l2": "flushed before each rep", "reps": reps}
        for k, t in (("quantize_rows", t_rows), ("quantize_act", t_act), ("quantize_cols", t_cols)):
            gbs = by[k] / (t * 1e-3) / 1e9
            line[k] = {"ms": round(t, 4), "GB/s": round(gbs, 1),
                       "frac_measured": round(gbs / peaks["hbm_gbs"], 4),
                       "frac_8TBs": round(gbs / 8000.0, 4)}
        print(json.dumps(line), flush=True)


def grads_sweep(device, workload, reps=20, warm=5):
    """Forward layer, dgrad and wgrad of every linear of a workload, each
    timed alone (median of `reps` CUDA-event timings, L2 flushed before each),
    with the FP4 GEMM of the same shape timed on its own beside it.  One JSON
    line per linear; TFLOP/s counts 2*M*K*N per product."""
    import quantize_gemm_b200 as qg
    from workloads import WORKLOADS, make_layer_inputs, make_matrix
    peaks = _peaks()
    fp4_peak = 4.0 * peaks["bf16_tflops_sustained"]
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    wl = WORKLOADS[workload]

    def timed(fn):
        for _ in range(warm):
            fn()
        ts = []
        for _ in range(reps):
            flush.fill_(1)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        ts.sort()
        return ts[len(ts) // 2]

    for li, layer in enumerate(wl.layers):
        A, W = make_layer_inputs(wl, li, device=device)
        M, K = A.shape
        N = W.shape[1]
        dY = make_matrix((M, N), seed=9000 + li, device=device, dtype=A.dtype, scale=1e-3)
        alpha = wl.alphas[0]
        codesT, t = qg.quantize_cols(W)
        ws_f = qg.Workspace(qg.QG_OP_FP4_LINEAR, M, K, N, qg._dt(A), alpha, device=device)
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
        t_fwd = timed(lambda: qg.qg_fp4_linear(A, codesT, t, W, alpha, Y, ws_f))
        qg.check_status(ws_f, "grads forward")
        del ws_f, Y
        ws_d = qg.Workspace(qg.QG_OP_FP4_DGRAD, M, K, N, qg.QG_F32, device=device)
        dA = torch.empty((M, K), dtype=torch.bfloat16, device=device)
        t_dgrad = timed(lambda: qg.qg_fp4_dgrad(dY, W, dA, ws_d))
        qg.check_status(ws_d, "grads dgrad")
        del ws_d, dA
        ws_w = qg.Workspace(qg.QG_OP_FP4_WGRAD, M, K, N, qg.QG_F32, device=device)
        dW = torch.empty((K, N), dtype=torch.bfloat16, device=device)
        t_wgrad = timed(lambda: qg.qg_fp4_wgrad(A, dY, dW, ws_w))
        qg.check_status(ws_w, "grads wgrad")
        del ws_w, dW
        # the GEMMs alone on codes of the same shapes
        gemm_ms = {}
        for name, (m, n, k) in (("dgrad", (M, K, N)), ("wgrad", (K, N, M))):
            cA = torch.randint(0, 256, (m, k // 2), dtype=torch.uint8, device=device)
            cB = torch.randint(0, 256, (n, k // 2), dtype=torch.uint8, device=device)
            sa = torch.full((m,), 1e-3, device=device)
            sb = torch.full((n,), 1e-3, device=device)
            out = torch.empty((m, n), dtype=torch.bfloat16, device=device)
            ws_g = qg.Workspace(qg.QG_OP_FP4_GEMM, m, k, n, qg.QG_F32, device=device)
            gemm_ms[name] = timed(lambda: qg.qg_fp4_gemm(cA, sa, cB, sb, m, n, k, None, out, None,
                                                         ws_g))
            qg.check_status(ws_g, "grads gemm")
            del cA, cB, out, ws_g
        torch.cuda.empty_cache()
        fl = 2.0 * M * K * N
        line = {"sweep": "grads", "workload": wl.name, "layer": layer.name, "M": M, "K": K,
                "N": N, "dtype": wl.dtype, "out": "bf16", "l2": "flushed before each rep",
                "reps": reps, "fp4_peak_tflops": fp4_peak}
        for k, tm in (("forward", t_fwd), ("dgrad", t_dgrad), ("wgrad", t_wgrad),
                      ("dgrad_gemm_only", gemm_ms["dgrad"]), ("wgrad_gemm_only", gemm_ms["wgrad"])):
            tf = fl / (tm * 1e-3) / 1e12
            line[k] = {"ms": round(tm, 4), "TFLOP/s": round(tf, 1),
                       "frac_measured": round(tf / fp4_peak, 4)}
        print(json.dumps(line), flush=True)
        del A, W, dY, codesT, t


def mx_sweep(device, workload, reps=20, warm=5):
    """MXFP4 variant on every linear of a workload: the block row quantizer
    on A, the block column quantizer on W and the block-scaled GEMM (fp32 Y),
    each timed alone (median of `reps`, L2 flushed before each), beside the
    per-row/per-column FP4 GEMM of the same shape.  One JSON line per linear."""
    import quantize_gemm_b200 as qg
    from workloads import WORKLOADS, make_layer_inputs
    peaks = _peaks()
    fp4_peak = 4.0 * peaks["bf16_tflops_sustained"]
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    wl = WORKLOADS[workload]

    def timed(fn):
        for _ in range(warm):
            fn()
        ts = []
        for _ in range(reps):
            flush.fill_(1)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        ts.sort()
        return ts[len(ts) // 2]

    for li, layer in enumerate(wl.layers):
        A, W = make_layer_inputs(wl, li, device=device)
        M, K = A.shape
        N = W.shape[1]
        ws_q = qg.Workspace(qg.QG_OP_QUANTIZE_ROWS, M, K, 1, qg._dt(A), device=device)
        codes = torch.empty((M, K // 2), dtype=torch.uint8, device=device)
        sa = torch.empty(qg.qg_mx_scale_bytes(M, K), dtype=torch.uint8, device=device)
        codesT = torch.empty((N, K // 2), dtype=torch.uint8, device=device)
        sw = torch.empty(qg.qg_mx_scale_bytes(N, K), dtype=torch.uint8, device=device)
        t_rows = timed(lambda: qg.qg_mx_quantize_rows(A, codes, sa, ws_q))
        t_cols = timed(lambda: qg.qg_mx_quantize_cols(W, codesT, sw, ws_q))
        qg.check_status(ws_q, "mx quantizers")
        Y = torch.empty((M, N), dtype=torch.float32, device=device)
        ws_g = qg.Workspace(qg.QG_OP_FP4_GEMM, M, K, N, qg.QG_F32, device=device)
        t_mx = timed(lambda: qg.qg_mx_gemm(codes, sa, codesT, sw, M, N, K, None, Y, None, ws_g))
        s_row = torch.full((M,), 1e-3, device=device)
        s_col = torch.full((N,), 1e-3, device=device)
        t_fp4 = timed(lambda: qg.qg_fp4_gemm(codes, s_row, codesT, s_col, M, N, K, None, Y, None,
                                             ws_g))
        qg.check_status(ws_g, "mx gemm")
        fl = 2.0 * M * K * N
        b = qg._dt(A) == qg.QG_BF16 and 2 or 4
        line = {"sweep": "mx", "workload": wl.name, "layer": layer.name, "M": M, "K": K, "N": N,
                "dtype": wl.dtype, "y": "f32", "l2": "flushed before each rep", "reps": reps,
                "fp4_peak_tflops": fp4_peak, "hbm_gbs": peaks["hbm_gbs"]}
        for k, tm, by in (("mx_quantize_rows", t_rows, b * M * K + M * K / 2 + M * K / 32),
                          ("mx_quantize_cols", t_cols, b * K * N + K * N / 2 + K * N / 32)):
            gbs = by / (tm * 1e-3) / 1e9
            line[k] = {"ms": round(tm, 4), "GB/s": round(gbs, 1),
                       "frac_measured": round(gbs / peaks["hbm_gbs"], 4)}
        for k, tm in (("mx_gemm", t_mx), ("fp4_gemm_row_col_scales", t_fp4)):
            tf = fl / (tm * 1e-3) / 1e12
            line[k] = {"ms": round(tm, 4), "TFLOP/s": round(tf, 1),
                       "frac_measured": round(tf / fp4_peak, 4)}
        print(json.dumps(line), flush=True)
        del A, W, codes, codesT, sa, sw, Y, ws_q, ws_g
        torch.cuda.empty_cache()


def compensated_sweep(device, workload, alpha=None, reps=10, warm=3):
    """The compensated GEMM (dA . W computed inside the GEMM kernel) beside the
    two-kernel form (the SpMM writing the compensation into Y, then the GEMM
    adding the product in place), and the whole layer call (qg_fp4_linear,
    activation quantizer included) with fp32 Y and with bf16 Y (row chunks
    through the layer's fp32 scratch), on every linear of a workload; median
    of `reps` CUDA-event timings, L2 flushed before each.  One JSON line per
    linear."""
    import quantize_gemm_b200 as qg
    from workloads import WORKLOADS, make_layer_inputs
    wl = WORKLOADS[workload]
    alpha = wl.alphas[0] if alpha is None else alpha
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)

    def timed(fn):
        for _ in range(warm):
            fn()
        ts = []
        for _ in range(reps):
            flush.fill_(1)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        ts.sort()
        return ts[len(ts) // 2]

    for li, layer in enumerate(wl.layers):
        A, W = make_layer_inputs(wl, li, device=device)
        M, K = A.shape
        N = W.shape[1]
        codes, s, csr, _ = qg.quantize_act(A, alpha)
        codesT, t = qg.quantize_cols(W)
        Y = torch.empty((M, N), dtype=torch.float32, device=device)
        ws_c = qg.Workspace(qg.QG_OP_FP4_GEMM_COMPENSATED, M, K, N, qg.QG_F32, device=device)
        ws_s = qg.Workspace(qg.QG_OP_SPMM, M, K, N, qg._dt(W), device=device)
        ws_g = qg.Workspace(qg.QG_OP_FP4_GEMM, M, K, N, qg.QG_F32, device=device)
        t_comp = timed(lambda: qg.qg_fp4_gemm_compensated(codes, s, codesT, t, M, N, K, csr, W, Y,
                                                          ws_c))
        t_spmm = timed(lambda: qg.qg_spmm_correction(csr, M, W, Y, ws_s))
        t_gemm = timed(lambda: qg.qg_fp4_gemm(codes, s, codesT, t, M, N, K, Y, Y, None, ws_g))
        Yb = torch.empty((M, N), dtype=torch.bfloat16, device=device)
        ws_l = qg.Workspace(qg.QG_OP_FP4_LINEAR, M, K, N, qg._dt(A), alpha, device=device)
        ws_a = qg.Workspace(qg.QG_OP_QUANTIZE_ACT, M, K, 1, qg._dt(A), alpha, device=device)
        t_lf = timed(lambda: qg.qg_fp4_linear(A, codesT, t, W, alpha, Y, ws_l))
        t_lb = timed(lambda: qg.qg_fp4_linear(A, codesT, t, W, alpha, Yb, ws_l))
        t_act = timed(lambda: qg.quantize_act(A, alpha, ws=ws_a))
        for ws in (ws_c, ws_s, ws_g, ws_l, ws_a):
            qg.check_status(ws, "compensated sweep")
        nnz = int(csr.nnz.item())
        chunk = max(256, (128 << 20) // (4 * N) // 256 * 256)
        print(json.dumps({"sweep": "compensated", "workload": wl.name, "layer": layer.name,
                          "M": M, "K": K, "N": N, "alpha": alpha, "nnz": nnz,
                          "compensated_gemm_ms": round(t_comp, 4),
                          "spmm_ms": round(t_spmm, 4), "gemm_in_place_ms": round(t_gemm, 4),
                          "two_kernel_ms": round(t_spmm + t_gemm, 4),
                          "compensation_tflops_fused": round(2 * nnz * N / (t_comp * 1e-3) / 1e12, 2),
                          "layer_fp32_y_ms": round(t_lf, 4), "layer_bf16_y_ms": round(t_lb, 4),
                          "act_quantizer_ms": round(t_act, 4),
                          "bf16_y_chunk_rows": min(chunk, M),
                          "l2": "flushed before each rep", "reps": reps}), flush=True)
        del A, W, codes, codesT, Y, Yb, ws_c, ws_s, ws_g, ws_l, ws_a
        torch.cuda.empty_cache()


def fp4_peak_sweep(device, reps=10, warm=3, iters=1 << 16):
    """The tensor pipe's E2M1 rate from the library's MMA-only loop
    (qg_fp4_mma_loop: operands in shared memory, the GEMM's MMA shape, no
    global traffic), one CTA per SM and 2-SM pairs; median of `reps` CUDA-event
    timings on the launching stream, clocks sampled meanwhile.  One JSON line
    per form, with the ratio to the FP4 denominator the other lines use
    (4 x the measured sustained bf16 rate)."""
    import quantize_gemm_b200 as qg
    peaks = _peaks()
    fp4_denominator = 4.0 * peaks["bf16_tflops_sustained"]
    ws = qg.Workspace(qg.QG_OP_FP4_GEMM, 1, 32, 1, qg.QG_F32, device=device)
    stream = torch.cuda.current_stream(device)
    for pair in (False, True):
        # one launch first, its status read before any further launch: a form
        # whose first launch flags an error is reported and not launched again
        qg.fp4_mma_loop(iters, pair, ws, stream=stream)
        st = ws.sync_status(stream)
        if st != qg.QG_OK:
            print(json.dumps({"sweep": "fp4_peak", "pair": pair, "error": qg.qg_status_string(st)}),
                  flush=True)
            continue
        for _ in range(warm - 1):
            qg.fp4_mma_loop(iters, pair, ws, stream=stream)
        clocks = ClockSampler(device.index or 0)
        clocks.start()
        ts, flops = [], 0.0
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            flops = qg.fp4_mma_loop(iters, pair, ws, stream=stream)
            b.record(stream)
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        clk = clocks.stop()
        qg.check_status(ws, "fp4 mma loop")
        ts.sort()
        ms = ts[len(ts) // 2]
        tf = flops / (ms * 1e-3) / 1e12
        line = {"sweep": "fp4_peak", "form": "2-SM pairs (cta_group::2)" if pair else "one CTA per SM",
                "mma": "256 x 224 x 64" if pair else "128 x 224 x 64", "iters": iters,
                "reps": reps, "ms": round(ms, 4), "TFLOP/s": round(tf, 1),
                "ratio_to_4x_bf16_sustained": round(tf / fp4_denominator, 4),
                "fp4_denominator_tflops": fp4_denominator, "clocks": clk}
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="block16k")
    ap.add_argument("--layer", type=int, default=None,
                    help="run one linear of the workload (index), e.g. for profiling")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch the timed steps eagerly instead of replaying a captured CUDA graph")
    ap.add_argument("--alpha", type=float, default=None,
                    help="quantile of the clamp (default: every alpha of the workload, the "
                         "first as the headline, the others in alpha_sweep)")
    ap.add_argument("--quantizer-sweep", action="store_true",
                    help="time the three quantizers over 1M..256M bf16 elements (one JSON line "
                         "per size) instead of the layer stream")
    ap.add_argument("--mx", action="store_true",
                    help="time the MXFP4 block-scaled quantizers and GEMM on each linear of "
                         "--workload (one JSON line per linear) instead of the layer stream")
    ap.add_argument("--fp4-peak", action="store_true",
                    help="time the library's MMA-only tensor-pipe loop (E2M1 rate of the tensor "
                         "cores, solo and 2-SM pairs) instead of the layer stream")
    ap.add_argument("--compensated", action="store_true",
                    help="time the compensated GEMM (dA . W inside the GEMM kernel) beside the "
                         "SpMM + in-place GEMM pair on each linear of --workload (one JSON line "
                         "per linear) instead of the layer stream")
    ap.add_argument("--grads", action="store_true",
                    help="time forward, dgrad and wgrad of each linear of --workload (one JSON "
                         "line per linear) instead of the layer stream")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return
        print(json.dumps(reference_arm(args, rank, world)), flush=True)
        return

    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    import __graft_entry__
    if rank == 0:
        __graft_entry__.build()
    if args.quantizer_sweep or args.grads or args.mx or args.fp4_peak or args.compensated:
        if rank == 0:
            if args.quantizer_sweep:
                quantizer_sweep(device)
            elif args.compensated:
                compensated_sweep(device, args.workload, args.alpha)
            elif args.fp4_peak:
                fp4_peak_sweep(device)
            elif args.mx:
                mx_sweep(device, args.workload)
            else:
                grads_sweep(device, args.workload)
        return
    if world > 1:
        torch.distributed.barrier()
    out = our_arm(args, rank, world, device)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
