"""Benchmark of the rotated W4A4 linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step is one pass of the whole path over one batch through the public
call convrot_linear: the fused prep kernel (rotation, rowwise absmax INT4
quantisation, packing) and the tcgen05 GEMM with its scale/bias/bf16
epilogue (two kernels per linear layer; for 1-4 tokens one kernel that does
both).  Weights are prepared once before
timing (the offline step).  Caches stay cold without a flush kernel: the
steps cycle through enough full copies of the step's data (activations,
workspace, weights, outputs) that the copies together exceed twice the L2
size.  Each step is one CUDA graph replay; K replays run back to back between
two CUDA events on the launching stream.  Two more passes of K replays time
the prep kernel alone and the GEMM alone for the roofline.  The end-to-end
figure calls convrot_linear on pinned host buffers with the copies inside the
timed interval (L2 flushed before each of those steps).  Under torchrun every
rank runs its own batch (weak scaling, no collective on the data path); the
reported time is the maximum over ranks.

Prints one JSON line (rank 0).  ``--impl reference`` times the CPU oracle
instead, on bounded samples of the same workload, on the host cores.

``--variant w4a16`` measures the W4A16 variant the same way instead (public
call convrot_w4a16_linear: the rotation kernel writing bf16, then the bf16 x
INT4 tcgen05 GEMM), reported in bf16 tensor TFLOP/s.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from rotated_w4a4_quantized_b200 import workloads as wl  # noqa: E402

METRIC = "W4A4 linear end-to-end TOPS and % of INT8 tensor peak; prep kernel HBM GB/s"
L2_FLUSH_BYTES = 256 << 20
# Bytes a prep launch must move per row: 2K read (bf16), K/2 + 4 written.
PREP_BYTES_PER_ROW = lambda K: 2 * K + K // 2 + 4  # noqa: E731
# GEMM algorithmic bytes: packed codes of both operands, both scale vectors,
# bias, bf16 output
GEMM_BYTES = lambda M, N, K: M * K // 2 + N * K // 2 + 4 * (M + N) + 2 * N + 2 * M * N  # noqa: E731
SKINNY_MAX_M = 128   # the GEMM's few-token form (weight stream, HBM-bound) up to here
# whole-layer algorithmic bytes when the layer runs as one kernel
LAYER_BYTES = lambda M, N, K: 2 * M * K + N * K // 2 + 4 * N + 2 * N + 2 * M * N  # noqa: E731
INT8_PER_BF16 = 2.0   # nominal dense ratio (4.5 / 2.25 PFLOP/s)
METRIC_W4A16 = "W4A16 linear end-to-end TFLOP/s (bf16 x INT4 tensor ops); rotation kernel HBM GB/s"
# W4A16 algorithmic bytes: the rotation reads x and writes xr (bf16 each);
# the GEMM reads xr, the packed weights, scales and bias and writes y
ROT16_BYTES = lambda M, K: 4 * M * K  # noqa: E731
GEMM16_BYTES = lambda M, N, K: 2 * M * K + N * K // 2 + 4 * N + 2 * N + 2 * M * N  # noqa: E731
METRIC_NVFP4 = ("NVFP4 linear end-to-end TFLOP/s (E2M1 x E2M1 block-scaled tensor ops); "
                "quantisation kernel HBM GB/s")
FP4_PER_BF16 = 4.0    # nominal dense ratio (9 / 2.25 PFLOP/s)
# NVFP4 algorithmic bytes: the quantisation reads x (bf16) and writes codes,
# block scales and row scales; the GEMM reads both operands' codes and
# scales, the bias, and writes y
FP4_QUANT_BYTES = lambda M, K: 2 * M * K + M * K // 2 + M * K // 16 + 4 * M  # noqa: E731
FP4_GEMM_BYTES = lambda M, N, K: (M + N) * (K // 2 + K // 16 + 4) + 2 * N + 2 * M * N  # noqa: E731


MIN_KERNEL_MS = 50.0          # device time of each per-kernel timing pass, at least
NOMINAL_INT8_TOPS = 4500.0    # datasheet dense int8 (half of the 2:4-sparse figure)


def int8_ceiling(dev, n=8192):
    """The achieved int8 tensor-core ceiling of this GPU: torch._int_mm
    (cuBLASLt s8 x s8 -> s32, both operands K-major) on n x n x n, best of 10
    back-to-back launches timed with CUDA events after warm-up.  None where
    the call is not available."""
    try:
        a = torch.randint(-7, 8, (n, n), dtype=torch.int8, device=dev)
        b = torch.randint(-7, 8, (n, n), dtype=torch.int8, device=dev).t()
        for _ in range(3):
            c = torch._int_mm(a, b)
        torch.cuda.synchronize()
        best = float("inf")
        for _ in range(10):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            c = torch._int_mm(a, b)
            e1.record()
            e1.synchronize()
            best = min(best, e0.elapsed_time(e1))
        del a, b, c
        torch.cuda.empty_cache()
        return {"tops": round(2 * n ** 3 / (best * 1e-3) / 1e12, 1), "shape": f"{n}^3",
                "how": "torch._int_mm (cuBLASLt s8xs8->s32), best of 10, CUDA events"}
    except (RuntimeError, TypeError) as e:
        return {"tops": None, "error": str(e).splitlines()[0][:200]}


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm": float(p["hbm_gbs"]), "bf16": float(p["bf16_tflops"]),
                "bf16_sustained": float(p["bf16_tflops_sustained"]), "src": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "src": "fallback"}


# the sources libconvrot.so (the W4A4 kernels) is compiled from
W4A4_SOURCES = ("convrot.cu", "decode.cuh", "gemm.cuh", "prep.cuh", "ptx.cuh", "skinny.cuh")


def _src_hash():
    """Hash of the W4A4 kernel sources: the committed per-launch DRAM traffic
    of those kernels holds while it is unchanged."""
    h = hashlib.sha256()
    d = os.path.join(ROOT, "rotated_w4a4_quantized_b200", "csrc")
    for name in sorted(W4A4_SOURCES):
        with open(os.path.join(d, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def _traffic(workload, kernel):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel sources; else None."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return None
    if t.get("src_hash") != _src_hash():
        return None
    return t.get("per_launch_bytes", {}).get(workload, {}).get(kernel)


class ClockSampler:
    """nvidia-smi samples of one GPU while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: str):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            # wait (up to 3 s) until the sampler runs, so the window is covered
            t0 = time.time()
            while not self.lines and time.time() - t0 < 3.0 and self.proc.poll() is None:
                time.sleep(0.01)
        except OSError:
            self.proc = None
        self.first = len(self.lines)
        return self

    def mark_end(self):
        """Call when the timed work is done; later samples are not used."""
        time.sleep(0.03)             # let the sample covering the end arrive
        self.last = len(self.lines)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.t.join(timeout=2)

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        lo = max(0, getattr(self, "first", 0) - 1)
        hi = getattr(self, "last", len(self.lines))
        for line in self.lines[lo:hi]:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != 6:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[2:]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def _dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def aggregate(local_ms: float, local_ops: float, device=None):
    """(max time over ranks, total ops over ranks); control plane only."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return local_ms, local_ops
    t = torch.tensor([local_ms], dtype=torch.float64, device=device)
    o = torch.tensor([local_ops], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(o, op=dist.ReduceOp.SUM)
    return float(t.item()), float(o.item())


# ---------------------------------------------------------------------------
# the GPU arm
# ---------------------------------------------------------------------------

def run_gpu(args):
    import torch.distributed as dist

    import rotated_w4a4_quantized_b200 as cr
    from rotated_w4a4_quantized_b200 import build
    build.build()

    world, rank, local = _dist()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    name = args.workload
    spec = wl.WORKLOADS[name]
    layers = wl.make_workload(name, seed=spec.seed + rank)
    stream = torch.cuda.current_stream()
    nl = len(layers)

    # offline step: prepare the weights once
    prepared = []
    for lt in layers:
        w = lt.w.to(dev)
        qw, sw = cr.convrot_quantize_weight(w, lt.spec.group)
        b = None if lt.b is None else lt.b.to(dev)
        del w
        prepared.append((lt.spec, qw, sw, b))
    x0 = layers[0].x.to(dev)

    # Cold caches without a flush kernel: the steps cycle through R full copies
    # of everything a step touches (activations, workspace, weights, outputs),
    # with R copies together at least twice the L2 size, so no step finds its
    # data in L2 from an earlier one.
    # (the workspace's codes and scales; its split area is touched only by
    # the partial sums of one wave, a small share of a step)
    step_bytes = sum(sp.M * sp.K * 2 + sp.M * (sp.K // 2 + 4)
                     + sp.N * (sp.K // 2 + 6) + sp.M * sp.N * 2 for sp, *_ in prepared)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    R = 1 if step_bytes >= 2 * l2 else min(64, -(-2 * l2 // step_bytes))

    class Copy:
        pass

    copies = []
    for r in range(R):
        c = Copy()
        c.w = [(sp, qw.clone(), sw.clone(), None if b is None else b.clone())
               for sp, qw, sw, b in prepared]
        c.acts = [x0.clone()]
        c.ws, c.lws, c.outs = [], [], []
        for i, (sp, *_) in enumerate(prepared):
            c.ws.append((torch.empty(sp.M, sp.K // 2, dtype=torch.uint8, device=dev),
                         torch.empty(sp.M, dtype=torch.float32, device=dev)))
            c.lws.append(torch.empty(max(1, cr.convrot_linear_workspace_size(sp.M, sp.K)),
                                     dtype=torch.uint8, device=dev))
            c.outs.append(torch.empty(sp.M, sp.N, dtype=torch.bfloat16, device=dev))
            if i + 1 < nl:
                c.acts.append(c.outs[i])   # chained layers: next input is this output
        copies.append(c)

    def step(c):
        # the public whole-layer call: prep kernel + GEMM kernel per layer
        for i, (sp, qw, sw, b) in enumerate(c.w):
            cr.convrot_linear(c.acts[i], qw, sw, b, sp.group, c.lws[i], c.outs[i])

    def prep_only(c, i):
        sp, qw, sw, b = c.w[i]
        cr.convrot_prepare_act(c.acts[i], sp.group, c.ws[i][0], c.ws[i][1])

    # the GEMM alone with a split area, so it runs the split-K plan of the
    # whole-layer call (steps on one stream may share one area)
    areas = [cr.new_split_area(dev) for _ in prepared]

    def gemm_only(c, i):
        sp, qw, sw, b = c.w[i]
        cr.convrot_linear_prepared_split(c.ws[i][0], c.ws[i][1], qw, sw, b, sp.K, areas[i],
                                         out=c.outs[i])

    for k in range(max(args.warmup, R)):
        step(copies[k % R])
        for i in range(nl):
            prep_only(copies[k % R], i)
            gemm_only(copies[k % R], i)
    torch.cuda.synchronize()
    if cr.convrot_check_device_error() != 0:
        raise RuntimeError("device error during warm-up")

    # CUDA graphs per program (whole step, prep only, GEMM only): one graph
    # per copy, and one graph that runs every copy once in turn (R steps), so
    # a replay launches R steps and host launch cost stays out of the device
    # timing even for layers that take a few microseconds.
    def capture(fn, *a):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn(*a)
        return g

    def capture_all(fn, *a):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for c in copies:
                fn(c, *a)
        return g

    progs = {"step": (step, ())}
    for i in range(nl):
        progs[("prep", i)] = (prep_only, (i,))
        progs[("gemm", i)] = (gemm_only, (i,))
    graphs = {k: ([capture(fn, c, *a) for c in copies], capture_all(fn, *a))
              for k, (fn, a) in progs.items()}
    for one, every in graphs.values():
        for g in one + [every]:
            g.replay()
    torch.cuda.synchronize()

    def timed(key, steps):
        """Device time of exactly `steps` back-to-back steps of one program."""
        one, every = graphs[key]
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(steps // R):
            every.replay()
        for k in range(steps % R):
            one[k].replay()
        b.record()
        b.synchronize()
        return a.elapsed_time(b)

    # timed region: K whole steps
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        gpu_id = str(local)
    with ClockSampler(gpu_id) as clocks:
        local_ms = timed("step", args.steps)
        torch.cuda.synchronize()
        clocks.mark_end()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    status = cr.convrot_check_device_error()
    if status != 0:
        raise RuntimeError(f"device error status {status} in the timed region")

    # per-kernel durations: back-to-back launches of one kernel of one layer,
    # at least K of them and at least MIN_KERNEL_MS of device time, so that
    # short kernels are not timed over a fraction of a millisecond
    def timed_kernel(key):
        n = args.steps
        t = timed(key, n)
        if t < MIN_KERNEL_MS:
            n = int(math.ceil(n * MIN_KERNEL_MS * 1.05 / max(t, 1e-3)))
            t = timed(key, n)
        return t / n, n

    prep_pass = [timed_kernel(("prep", i)) for i in range(nl)]
    gemm_pass = [timed_kernel(("gemm", i)) for i in range(nl)]
    prep_ms = [[avg] * args.steps for avg, _ in prep_pass]
    gemm_ms = [[avg] * args.steps for avg, _ in gemm_pass]
    ceiling = int8_ceiling(dev) if any(sp.M > SKINNY_MAX_M for sp, *_ in prepared) else None
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)   # e2e pass only
    ops_step = spec.ops
    t_max, ops_total = aggregate(local_ms, ops_step * args.steps, dev)
    value = ops_total / (t_max * 1e-3) / 1e12                      # TOPS, whole job
    tokens_s = spec.tokens * world * args.steps / (t_max * 1e-3)

    peaks = _peaks()
    int8_peak = peaks["bf16"] * INT8_PER_BF16
    gemm_avg = [statistics.fmean(g) for g in gemm_ms]
    prep_avg = [statistics.fmean(p) for p in prep_ms]
    gemm_tops = [2 * sp.M * sp.N * sp.K / (g * 1e-3) / 1e12 for (sp, *_), g in zip(prepared, gemm_avg)]
    prep_gbs = [sp.M * PREP_BYTES_PER_ROW(sp.K) / (p * 1e-3) / 1e9 for (sp, *_), p in zip(prepared, prep_avg)]
    gemm_total, prep_total = sum(map(sum, gemm_ms)), sum(map(sum, prep_ms))
    single = [cr.convrot_linear_single_kernel(sp.M, sp.K, sp.group) for sp, *_ in prepared]
    if all(single):
        # the whole step is one decode kernel per layer (token preparation
        # fused into a CUDA-core GEMV): its algorithmic bytes over the step time
        byts = sum(LAYER_BYTES(sp.M, sp.N, sp.K) for sp, *_ in prepared)
        gbs = byts * args.steps / (t_max * 1e-3) / 1e9
        roof = {"kernel": "decode_kernel", "bound": "hbm", "achieved": round(gbs, 1),
                "peak": peaks["hbm"], "unit": "GB/s", "frac": round(gbs / peaks["hbm"], 4),
                "traffic": _traffic(name, "decode_kernel"),
                "note": "whole layer in one kernel; algorithmic bytes 2MK (x) + NK/2 + 4N + 2N "
                        f"+ 2MN (y) per step; HBM peak {peaks['src']}"}
    elif gemm_total >= prep_total:
        i = max(range(nl), key=lambda j: sum(gemm_ms[j]))
        sp = prepared[i][0]
        if sp.M <= SKINNY_MAX_M:
            gbs = GEMM_BYTES(sp.M, sp.N, sp.K) / (gemm_avg[i] * 1e-3) / 1e9
            roof = {"kernel": "skinny_kernel", "bound": "hbm", "achieved": round(gbs, 1),
                    "peak": peaks["hbm"], "unit": "GB/s", "frac": round(gbs / peaks["hbm"], 4),
                    "traffic": _traffic(name, "skinny_kernel"),
                    "note": "algorithmic bytes M K/2 + N K/2 + 4(M+N) + 2N + 2MN (the packed "
                            f"weight stream dominates); HBM peak {peaks['src']}"}
        else:
            roof = {"kernel": "gemm_kernel", "bound": "tensor", "achieved": round(gemm_tops[i], 2),
                    "peak": round(int8_peak, 1), "unit": "TFLOP/s",
                    "frac": round(gemm_tops[i] / int8_peak, 4),
                    "traffic": _traffic(name, "gemm_kernel"),
                    "frac_of_nominal_int8": round(gemm_tops[i] / NOMINAL_INT8_TOPS, 4),
                    "frac_of_int_mm": (round(gemm_tops[i] / ceiling["tops"], 4)
                                       if ceiling and ceiling.get("tops") else None),
                    "note": "integer tensor ops (2 per multiply-add); peak = measured bf16 burst "
                            f"x {INT8_PER_BF16} nominal int8/bf16 ratio ({peaks['src']}); also "
                            f"against the {NOMINAL_INT8_TOPS:.0f} TOPS nominal dense int8 peak "
                            "and against torch._int_mm (cuBLASLt int8) measured in this run"}
    else:
        i = max(range(nl), key=lambda j: sum(prep_ms[j]))
        roof = {"kernel": "prep_kernel", "bound": "hbm", "achieved": round(prep_gbs[i], 1),
                "peak": peaks["hbm"], "unit": "GB/s", "frac": round(prep_gbs[i] / peaks["hbm"], 4),
                "traffic": _traffic(name, "prep_kernel"),
                "note": f"HBM peak {peaks['src']}"}

    # end to end through the public call, host buffers, copies inside the interval
    e2e = run_e2e(cr, prepared, spec, dev, stream, flush, args)
    t_e2e, ops_e2e = aggregate(e2e["ms"], ops_step * e2e["steps"], dev)

    launches = sum(1 if s1 else 2 for s1 in single) * args.steps
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "TOPS", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(t_max / args.steps, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "s8",
        "data": "synthetic (seeded bf16, shapes and distributions of the workload; no weights)",
        "config": {"workload": name, "layers": [f"{l.M}x{l.K}->{l.N} g{l.group}" for l in spec.layers],
                   "tokens_per_rank": spec.tokens,
                   "l2": f"cold: steps cycle through {R} copies of all step data "
                         f"({R * step_bytes / 2**20:.0f} MiB >= 2 x L2)",
                   "launch": f"CUDA graphs of {R} steps (each copy once), replayed back to back",
                   "parallelism": f"dp{world}"},
        "tokens_per_s": round(tokens_s, 1),
        "int8_peak_frac_path": round(value / world / int8_peak, 4),
        "gemm_tops": [round(v, 2) for v in gemm_tops],
        "gemm_gbs": [round(GEMM_BYTES(sp.M, sp.N, sp.K) / (g * 1e-3) / 1e9, 1)
                     for (sp, *_), g in zip(prepared, gemm_avg)],
        "prep_gbs": [round(v, 1) for v in prep_gbs],
        "prep_hbm_frac": [round(v / peaks["hbm"], 4) for v in prep_gbs],
        "roofline": roof,
        "e2e": {"value": round(ops_e2e / (t_e2e * 1e-3) / 1e12, 3), "unit": "TOPS",
                "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                "call": f"HostPipeline: pinned host buffers, {e2e['chunks']} row chunks, "
                        "copies overlapped with convrot_linear on three streams",
                "link": e2e["link"]},
        "gpu_launches": launches,
        "kernel_passes": {"prep_launches": [n for _, n in prep_pass],
                          "gemm_launches": [n for _, n in gemm_pass],
                          "min_device_ms": MIN_KERNEL_MS},
        "int8_ceiling": ceiling,
        "clocks": clocks.summary(),
    }
    if rank == 0:
        line["cpu_baseline"] = cpu_baseline(name, args.cpu_seconds) if world == 1 and not args.no_cpu else None
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


class W4A16Variant:
    """bf16 activations x the W4A4 packed weights (include/convrot_w4a16.h)."""
    name, metric, dtype = "w4a16", METRIC_W4A16, "bf16"
    peak_ratio, peak_note = 1.0, "measured bf16 burst"
    prep_kernel = "rotate_bf16_kernel"
    prep_bytes = staticmethod(ROT16_BYTES)

    @staticmethod
    def gemm_kernel_for(sp):
        # up to 64 tokens the few-token form with the weights widened into TMEM
        return "w4a16_skinny_kernel" if sp.M <= 64 else "w4a16_gemm_kernel"

    gemm_bytes = staticmethod(GEMM16_BYTES)
    prep_desc = "algorithmic bytes 4MK"
    gemm_desc = "2MK (xr) + NK/2 + 4N + 2N + 2MN"

    @staticmethod
    def weights(cr, w, group):
        return cr.convrot_quantize_weight(w, group)

    @staticmethod
    def buffers(cr, sp, dev):
        ws = torch.empty(cr.convrot_w4a16_workspace_size(sp.M, sp.K), dtype=torch.uint8, device=dev)
        return {"ws": ws, "xr": ws[:sp.M * sp.K * 2].view(torch.bfloat16).view(sp.M, sp.K)}

    @staticmethod
    def step(cr, x, wt, b, sp, bufs, out):
        cr.convrot_w4a16_linear(x, *wt, b, sp.group, bufs["ws"], out)

    @staticmethod
    def prep(cr, x, sp, bufs):
        cr.convrot_w4a16_prepare_act(x, sp.group, out=bufs["xr"])

    @staticmethod
    def gemm(cr, wt, b, sp, bufs, out):
        cr.convrot_w4a16_linear_prepared(bufs["xr"], *wt, b, out=out)

    @staticmethod
    def check(cr):
        return cr.convrot_w4a16_check_device_error()


class NVFP4Variant:
    """E2M1 activations and weights with E4M3 block scales (include/convrot_nvfp4.h)."""
    name, metric, dtype = "nvfp4", METRIC_NVFP4, "e2m1"
    peak_ratio = FP4_PER_BF16
    peak_note = f"measured bf16 burst x {FP4_PER_BF16} nominal fp4/bf16 ratio"
    prep_kernel = "quant_kernel"
    prep_bytes = staticmethod(FP4_QUANT_BYTES)

    @staticmethod
    def gemm_kernel_for(sp):
        return "nvfp4_gemm_kernel"

    gemm_bytes = staticmethod(FP4_GEMM_BYTES)
    prep_desc = "algorithmic bytes 2MK + MK/2 + MK/16 + 4M"
    gemm_desc = "(M+N)(K/2 + K/16 + 4) + 2N + 2MN"

    @staticmethod
    def weights(cr, w, group):
        return cr.convrot_nvfp4_quantize(w, group)

    @staticmethod
    def buffers(cr, sp, dev):
        M, K = sp.M, sp.K
        ws = torch.empty(cr.convrot_nvfp4_workspace_size(M, K), dtype=torch.uint8, device=dev)
        r256 = lambda v: (v + 255) // 256 * 256  # noqa: E731
        nsf = cr.convrot_nvfp4_scale_bytes(M, K)
        o1 = r256(M * K // 2)
        o2 = o1 + r256(nsf)
        return {"ws": ws, "q": ws[:M * K // 2].view(M, K // 2), "sf": ws[o1:o1 + nsf],
                "s": ws[o2:o2 + 4 * M].view(torch.float32)}

    @staticmethod
    def step(cr, x, wt, b, sp, bufs, out):
        cr.convrot_nvfp4_linear(x, *wt, b, sp.group, bufs["ws"], out)

    @staticmethod
    def prep(cr, x, sp, bufs):
        cr.convrot_nvfp4_quantize(x, sp.group, bufs["q"], bufs["sf"], bufs["s"])

    @staticmethod
    def gemm(cr, wt, b, sp, bufs, out):
        cr.convrot_nvfp4_linear_prepared(bufs["q"], bufs["sf"], bufs["s"], *wt, b, sp.K, out=out)

    @staticmethod
    def check(cr):
        return cr.convrot_nvfp4_check_device_error()


VARIANTS = {"w4a16": W4A16Variant, "nvfp4": NVFP4Variant}


def run_gpu_variant(args, V):
    """A variant on the bf16 tensor path (W4A16, NVFP4): the same timing
    scheme as run_gpu (cold L2 through rotating copies, CUDA graphs, K
    back-to-back steps between two events, max over ranks), through the
    variant's public whole-layer call."""
    import torch.distributed as dist

    import rotated_w4a4_quantized_b200 as cr
    from rotated_w4a4_quantized_b200 import build
    build.build()

    world, rank, local = _dist()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    name = args.workload
    spec = wl.WORKLOADS[name]
    layers = wl.make_workload(name, seed=spec.seed + rank)
    nl = len(layers)
    prepared = []
    for lt in layers:
        w = lt.w.to(dev)
        wt = V.weights(cr, w, lt.spec.group)             # offline step
        b = None if lt.b is None else lt.b.to(dev)
        del w
        prepared.append((lt.spec, wt, b))
    x0 = layers[0].x.to(dev)

    step_bytes = sum(V.prep_bytes(sp.M, sp.K) + V.gemm_bytes(sp.M, sp.N, sp.K) for sp, *_ in prepared)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    R = 1 if step_bytes >= 2 * l2 else min(64, -(-2 * l2 // step_bytes))

    class Copy:
        pass

    copies = []
    for r in range(R):
        c = Copy()
        c.w = [(sp, tuple(t.clone() for t in wt), None if b is None else b.clone())
               for sp, wt, b in prepared]
        c.acts, c.bufs, c.outs = [x0.clone()], [], []
        for i, (sp, *_) in enumerate(prepared):
            c.bufs.append(V.buffers(cr, sp, dev))
            c.outs.append(torch.empty(sp.M, sp.N, dtype=torch.bfloat16, device=dev))
            if i + 1 < nl:
                c.acts.append(c.outs[i])
        copies.append(c)

    def step(c):
        for i, (sp, wt, b) in enumerate(c.w):
            V.step(cr, c.acts[i], wt, b, sp, c.bufs[i], c.outs[i])

    def prep_only(c, i):
        V.prep(cr, c.acts[i], c.w[i][0], c.bufs[i])

    def gemm_only(c, i):
        sp, wt, b = c.w[i]
        V.gemm(cr, wt, b, sp, c.bufs[i], c.outs[i])

    for k in range(max(args.warmup, R)):
        step(copies[k % R])
        for i in range(nl):
            prep_only(copies[k % R], i)
            gemm_only(copies[k % R], i)
    torch.cuda.synchronize()
    if V.check(cr) != 0:
        raise RuntimeError("device error during warm-up")

    def capture(fn, *a):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn(*a)
        return g

    def capture_all(fn, *a):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for c in copies:
                fn(c, *a)
        return g

    progs = {"step": (step, ())}
    for i in range(nl):
        progs[("prep", i)] = (prep_only, (i,))
        progs[("gemm", i)] = (gemm_only, (i,))
    graphs = {key: ([capture(fn, c, *a) for c in copies], capture_all(fn, *a))
              for key, (fn, a) in progs.items()}
    for one, every in graphs.values():
        for g in one + [every]:
            g.replay()
    torch.cuda.synchronize()

    def timed(key, steps):
        one, every = graphs[key]
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(steps // R):
            every.replay()
        for j in range(steps % R):
            one[j].replay()
        b.record()
        b.synchronize()
        return a.elapsed_time(b)

    def timed_kernel(key):
        n = args.steps
        t = timed(key, n)
        if t < MIN_KERNEL_MS:
            n = int(math.ceil(n * MIN_KERNEL_MS * 1.05 / max(t, 1e-3)))
            t = timed(key, n)
        return t / n

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        gpu_id = str(local)
    with ClockSampler(gpu_id) as clocks:
        local_ms = timed("step", args.steps)
        torch.cuda.synchronize()
        clocks.mark_end()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    status = V.check(cr)
    if status != 0:
        raise RuntimeError(f"device error status {status} in the timed region")

    prep_avg = [timed_kernel(("prep", i)) for i in range(nl)]
    gemm_avg = [timed_kernel(("gemm", i)) for i in range(nl)]
    flops_step = spec.ops                       # 2 M N K per layer
    t_max, flops_total = aggregate(local_ms, flops_step * args.steps, dev)
    value = flops_total / (t_max * 1e-3) / 1e12
    tokens_s = spec.tokens * world * args.steps / (t_max * 1e-3)

    peaks = _peaks()
    tensor_peak = peaks["bf16"] * V.peak_ratio
    gemm_tf = [2 * sp.M * sp.N * sp.K / (g * 1e-3) / 1e12 for (sp, *_), g in zip(prepared, gemm_avg)]
    gemm_gbs = [V.gemm_bytes(sp.M, sp.N, sp.K) / (g * 1e-3) / 1e9
                for (sp, *_), g in zip(prepared, gemm_avg)]
    prep_gbs = [V.prep_bytes(sp.M, sp.K) / (r * 1e-3) / 1e9 for (sp, *_), r in zip(prepared, prep_avg)]
    if sum(gemm_avg) >= sum(prep_avg):
        i = max(range(nl), key=lambda j: gemm_avg[j])
        sp = prepared[i][0]
        # the bound of this shape: the larger of its tensor time and its byte time
        t_tensor = 2 * sp.M * sp.N * sp.K / (tensor_peak * 1e12)
        t_bytes = V.gemm_bytes(sp.M, sp.N, sp.K) / (peaks["hbm"] * 1e9)
        if t_tensor >= t_bytes:
            roof = {"kernel": V.gemm_kernel_for(sp), "bound": "tensor", "achieved": round(gemm_tf[i], 2),
                    "peak": round(tensor_peak, 1), "unit": "TFLOP/s",
                    "frac": round(gemm_tf[i] / tensor_peak, 4), "traffic": None,
                    "note": f"tensor ops (2 per multiply-add); peak = {V.peak_note} ({peaks['src']})"}
        else:
            roof = {"kernel": V.gemm_kernel_for(sp), "bound": "hbm", "achieved": round(gemm_gbs[i], 1),
                    "peak": peaks["hbm"], "unit": "GB/s", "frac": round(gemm_gbs[i] / peaks["hbm"], 4),
                    "traffic": None,
                    "note": f"algorithmic bytes {V.gemm_desc}; HBM peak {peaks['src']}"}
    else:
        i = max(range(nl), key=lambda j: prep_avg[j])
        roof = {"kernel": V.prep_kernel, "bound": "hbm", "achieved": round(prep_gbs[i], 1),
                "peak": peaks["hbm"], "unit": "GB/s", "frac": round(prep_gbs[i] / peaks["hbm"], 4),
                "traffic": None, "note": f"{V.prep_desc}; HBM peak {peaks['src']}"}

    # end to end: pinned host x in, pinned host y out, copies inside the interval
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    x_host = layers[0].x.pin_memory()
    y_host = torch.empty(prepared[-1][0].M, prepared[-1][0].N, dtype=torch.bfloat16).pin_memory()
    c = copies[0]
    e2e_steps = max(3, min(args.steps, 200))

    def e2e_step():
        c.acts[0].copy_(x_host, non_blocking=True)
        step(c)
        y_host.copy_(c.outs[-1], non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(e2e_steps)]
    for a, b in ev:
        flush.zero_()
        a.record(stream)
        e2e_step()
        b.record(stream)
    torch.cuda.synchronize()
    e2e_ms = sum(a.elapsed_time(b) for a, b in ev)
    t_e2e, fl_e2e = aggregate(e2e_ms, flops_step * e2e_steps, dev)

    line = {
        "metric": V.metric, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(t_max / args.steps, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": V.dtype,
        "data": "synthetic (seeded bf16, shapes and distributions of the workload; no weights)",
        "config": {"workload": name, "variant": V.name,
                   "layers": [f"{l.M}x{l.K}->{l.N} g{l.group}" for l in spec.layers],
                   "tokens_per_rank": spec.tokens,
                   "l2": f"cold: steps cycle through {R} copies of all step data "
                         f"({R * step_bytes / 2**20:.0f} MiB >= 2 x L2)",
                   "launch": f"CUDA graphs of {R} steps (each copy once), replayed back to back",
                   "parallelism": f"dp{world}"},
        "tokens_per_s": round(tokens_s, 1),
        "tensor_peak_frac_path": round(value / world / tensor_peak, 4),
        "gemm_tflops": [round(v, 2) for v in gemm_tf],
        "gemm_gbs": [round(v, 1) for v in gemm_gbs],
        "prep_gbs": [round(v, 1) for v in prep_gbs],
        "prep_hbm_frac": [round(v / peaks["hbm"], 4) for v in prep_gbs],
        "roofline": roof,
        "e2e": {"value": round(fl_e2e / (t_e2e * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
                "h2d_bytes_per_step": prepared[0][0].M * prepared[0][0].K * 2,
                "d2h_bytes_per_step": prepared[-1][0].M * prepared[-1][0].N * 2,
                "call": f"pinned host x -> device, the {V.name} whole-layer call per layer, y -> "
                        "pinned host, one stream, L2 flushed before each step"},
        "gpu_launches": 2 * nl * args.steps,
        "clocks": clocks.summary(),
    }
    if rank == 0:
        line["cpu_baseline"] = (cpu_baseline(name, args.cpu_seconds, V.name)
                                if world == 1 and not args.no_cpu else None)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def link_bandwidth(x_host, y_host, dev, reps=5):
    """Pinned host <-> device copy bandwidth of this step's byte counts: H2D
    alone, D2H alone, and both at once on two streams (GB/s, best of
    `reps`, CUDA events): the bound the end-to-end figure is judged against."""
    xd = torch.empty_like(x_host, device=dev)
    yd = torch.empty_like(y_host, device=dev)
    s1, s2 = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)

    def best(fn):
        t = float("inf")
        for _ in range(reps):
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            b.synchronize()
            t = min(t, a.elapsed_time(b))
        return t

    def both():
        cur = torch.cuda.current_stream()
        e = torch.cuda.Event()
        e.record(cur)
        s1.wait_event(e)
        s2.wait_event(e)
        with torch.cuda.stream(s1):
            xd.copy_(x_host, non_blocking=True)
        with torch.cuda.stream(s2):
            y_host.copy_(yd, non_blocking=True)
        cur.wait_stream(s1)
        cur.wait_stream(s2)

    t_in = best(lambda: xd.copy_(x_host, non_blocking=True))
    t_out = best(lambda: y_host.copy_(yd, non_blocking=True))
    t_both = best(both)
    bi, bo = x_host.numel() * x_host.element_size(), y_host.numel() * y_host.element_size()
    return {"h2d_gbs": round(bi / (t_in * 1e-3) / 1e9, 1), "d2h_gbs": round(bo / (t_out * 1e-3) / 1e9, 1),
            "both_gbs": round((bi + bo) / (t_both * 1e-3) / 1e9, 1),
            "bound_ms": round(max(t_in, t_out, t_both), 4)}


def run_e2e(cr, prepared, spec, dev, stream, flush, args):
    """The public host-buffer path: pinned x in, pinned y out, through
    HostPipeline (row chunks; H2D, convrot_linear per layer and D2H overlap
    on three streams), all inside each step's event interval."""
    sp0 = prepared[0][0]
    x_host = wl.make_workload(args.workload)[0].x.pin_memory()
    y_host = torch.empty(prepared[-1][0].M, prepared[-1][0].N, dtype=torch.bfloat16).pin_memory()
    # chunks of at least 256 rows, up to 8: on the 8192-token layer 8 chunks
    # measured 3.36 ms per step against 3.49 (4), 3.41 (12) and 3.47 (16), on
    # QKV 1.68 ms against 1.75 (4) and 1.74 (16): pipeline fill and drain are
    # one chunk's copy each, and every chunk adds its own copy and launch
    # overheads; one chunk would not overlap at all
    pipe = cr.HostPipeline(sp0.M, sp0.K, [(qw, sw, b, sp.group) for sp, qw, sw, b in prepared],
                           chunks=max(1, min(8, sp0.M // 256)), device=dev)
    steps = max(3, min(args.steps, 200))
    for _ in range(3):
        pipe(x_host, y_host, stream)
    torch.cuda.synchronize()
    # Steps are enqueued ahead (no per-step synchronisation), so the interval
    # of each step holds its copies and kernels, not host enqueue gaps.
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for a, b in ev:
        flush.zero_()
        a.record(stream)
        pipe(x_host, y_host, stream)
        b.record(stream)
    torch.cuda.synchronize()
    total = sum(a.elapsed_time(b) for a, b in ev)
    link = link_bandwidth(x_host, y_host, dev)
    link["e2e_over_bound"] = round(total / steps / link["bound_ms"], 3)
    return {"ms": total, "steps": steps, "h2d": sp0.M * sp0.K * 2,
            "d2h": prepared[-1][0].M * prepared[-1][0].N * 2, "chunks": len(pipe.ranges),
            "link": link}


class OracleSampler:
    """The oracle's per-call work on a sample of token rows: prepare those
    activation rows, integer GEMM against the prepared weights, epilogue
    (W4A16: rotate and round those rows, fp64 GEMM, epilogue; NVFP4: rotate
    and quantise those rows to NVFP4, fp64 block-scaled GEMM, epilogue).
    Weight preparation is offline (done once here, untimed), as on the GPU."""

    def __init__(self, name, variant="w4a4"):
        self.variant = variant
        import oracle as O
        O.build()
        self.O = O
        self.spec = wl.WORKLOADS[name]
        l0 = wl.make_workload(name)[0]
        self.sp = l0.spec
        if variant == "nvfp4":
            self.pw, self.sfw, self.sw = O.nvfp4_prepare_rows(wl.bf16_bits(l0.w), self.sp.group)
        else:
            self.pw, self.sw = O.prepare_rows(wl.bf16_bits(l0.w), self.sp.group)
        self.bb = None if l0.b is None else wl.bf16_bits(l0.b)
        self.xb = wl.bf16_bits(l0.x)
        self.cores = O.num_threads()
        self.layer = f"{self.sp.M}x{self.sp.K}->{self.sp.N} g{self.sp.group}"

    def run(self, rows):
        O, sp = self.O, self.sp
        t0 = time.perf_counter()
        if self.variant == "w4a16":
            O.w4a16_linear(self.xb[:rows], self.pw, self.sw, self.bb, sp.group)
        elif self.variant == "nvfp4":
            px, sfx, sx = O.nvfp4_prepare_rows(self.xb[:rows], sp.group)
            acc, _, _ = O.nvfp4_gemm(px, sfx, self.pw, self.sfw, sp.K)
            O.nvfp4_epilogue(acc, sx, self.sw, self.bb)
        else:
            px, sx = O.prepare_rows(self.xb[:rows], sp.group)
            O.epilogue(O.gemm(px, self.pw, sp.K), sx, self.sw, self.bb)
        return time.perf_counter() - t0

    def calibrate(self, seconds):
        """Rows such that one run takes about `seconds` (at least 1 row)."""
        rows, t = 1, self.run(1)
        while t < seconds / 8 and rows < self.sp.M:
            rows = min(self.sp.M, rows * 4)
            t = self.run(rows)
        if t < seconds and rows < self.sp.M:
            rows = min(self.sp.M, max(rows, int(rows * seconds / max(t, 1e-6))))
        return rows

    def ops(self, rows):
        return 2 * rows * self.sp.N * self.sp.K


# what the oracle computes per sampled row, by variant
VARIANT_WORK = {"w4a16": "rotation + bf16 rounding + fp64 GEMM + epilogue",
                "nvfp4": "rotation + NVFP4 quantisation + fp64 block-scaled GEMM + epilogue"}

# workloads whose baseline also gets a one-thread figure
ONE_THREAD_BASELINE = ("small_g256", "outlier_g64")


def cpu_baseline(name, seconds, variant="w4a4"):
    s = OracleSampler(name, variant)
    rows = s.calibrate(seconds)
    t = s.run(rows)
    what = VARIANT_WORK.get(variant, "prep + int64 GEMM + epilogue")
    out = {"value": round(s.ops(rows) / t / 1e12, 9),
           "unit": "TOPS" if variant == "w4a4" else "TFLOP/s", "cores": s.cores,
           "kind": "oracle",
           "sample": f"{rows} of {s.sp.M} token rows of layer {s.layer} ({what}, weights "
                     f"prepared offline), {t:.1f} s"}
    if name in ONE_THREAD_BASELINE and variant == "w4a4":
        s.O.set_num_threads(1)
        try:
            rows1 = s.calibrate(seconds / 4)
            t1 = s.run(rows1)
        finally:
            s.O.set_num_threads(s.cores)
        out["value_1thread"] = round(s.ops(rows1) / t1 / 1e12, 9)
        out["sample_1thread"] = f"{rows1} token rows on one thread, {t1:.1f} s"
    return out


def run_reference(args):
    world, rank, _ = _dist()
    if rank != 0:
        return
    name = args.workload
    V = VARIANTS.get(args.variant)
    s = OracleSampler(name, args.variant)
    # the whole run (warm-up + steps) stays within about --cpu-seconds x 8
    per_step = args.cpu_seconds * 8 / (args.steps + args.warmup)
    rows = s.calibrate(per_step)
    total = 0.0
    for k in range(args.warmup + args.steps):
        t = s.run(rows)
        if k >= args.warmup:
            total += t
    value = s.ops(rows) * args.steps / total / 1e12
    spec = wl.WORKLOADS[name]
    unit = "TOPS" if V is None else "TFLOP/s"
    what = VARIANT_WORK.get(args.variant, "prep + int64 GEMM + epilogue")
    line = {
        "impl": "reference", "metric": METRIC if V is None else V.metric, "value": round(value, 9),
        "unit": unit, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * total / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "s8" if V is None else V.dtype,
        "data": "synthetic (seeded bf16, same workload)",
        "config": {"workload": name, "layers": [f"{l.M}x{l.K}->{l.N} g{l.group}" for l in spec.layers],
                   "tokens_per_rank": spec.tokens, "parallelism": "cpu"},
        "cpu_baseline": {"value": round(value, 9), "unit": unit, "cores": s.cores, "kind": "oracle",
                         "sample": f"each step: {rows} of {s.sp.M} token rows of layer {s.layer} "
                                   f"({what}, weights prepared offline)"},
        "e2e": {"value": round(value, 9), "unit": unit, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def rank_plan(gpus: int, env) -> str:
    """'run' when this process is one of the requested ranks, 'spawn' when
    --gpus asks for more ranks than a process group provides (none was set
    up: start them).  A process group of another size is an error."""
    if gpus < 1:
        raise SystemExit(f"--gpus must be >= 1, got {gpus}")
    world = env.get("WORLD_SIZE")
    if world is None or world == "":
        return "spawn" if gpus > 1 else "run"
    if int(world) != gpus:
        raise SystemExit(f"--gpus {gpus} but WORLD_SIZE={world}: launch one rank per GPU "
                         f"(torchrun --nproc-per-node {gpus}) or drop --gpus")
    return "run"


def spawn_cmd(gpus: int, argv, port: int):
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
            f"--nproc-per-node={gpus}", "--master-addr", "127.0.0.1", f"--master-port={port}",
            os.path.abspath(__file__), *argv]


def spawn_ranks(gpus: int, argv) -> int:
    """Start `gpus` ranks of this script under torchrun on 127.0.0.1; rank 0
    prints the JSON line.  Returns their exit status."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    return subprocess.call(spawn_cmd(gpus, argv, port))


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default=wl.DEFAULT_BENCH, choices=sorted(wl.WORKLOADS))
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="CPU time budget of the oracle baseline")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU baseline")
    ap.add_argument("--variant", default="w4a4", choices=["w4a4", "w4a16", "nvfp4"],
                    help="w4a16: the bf16-activation variant (include/convrot_w4a16.h); "
                         "nvfp4: the NVFP4 variant (include/convrot_nvfp4.h)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    plan = rank_plan(args.gpus, os.environ)
    if plan == "spawn":
        sys.exit(spawn_ranks(args.gpus, sys.argv[1:] if argv is None else list(argv)))
    if args.impl == "reference":
        run_reference(args)
    elif args.variant in VARIANTS:
        run_gpu_variant(args, VARIANTS[args.variant])
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
