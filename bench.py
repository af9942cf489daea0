#!/usr/bin/env python3
"""Benchmark of the quantized decoder projection on B200.

Default workload (one "step"): M = 1 decode through one Llama-3.1-8B layer's
seven projections (q 4096x4096, k/v 1024x4096, o 4096x4096, gate/up
14336x4096, down 4096x14336) in W8A8 int8 and in FP8 E4M3 per-row, i.e. 14
GEMV launches (activation quantization fused) per step.  Metric: HBM GB/s of
algorithmic bytes (weights + scales + x + y) per second, whole job.

Legs:
  value     device time of K steps, each step one CUDA graph replay of the 14
            launches (the pages decode under CUDA graphs); inputs resident in
            HBM; 436 MB of weights per step, larger than L2, so every step
            streams from HBM.
  e2e       the same metric through the public API (``forward``) with the
            step's tokens copied host->device from pinned memory and the
            outputs read back device->host every step (captured in a graph,
            host synchronised per step).
  roofline  the GEMV kernel's algorithmic bytes per launch / its average
            launch duration (step time / launches, CUDA events), against the
            measured HBM copy bandwidth.
  cpu_baseline  the CPU oracle (test infrastructure) on the same workload,
            host cores, a bounded sample; reported, not the target.

``--impl reference`` times the CPU oracle alone on the same metric (rank 0
only).  Multi-GPU (torchrun): replicas, each rank runs the same step on its
own GPU; timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "quantized linear: M=1 GEMV HBM GB/s; M≥512 int8/FP8 TOPS; % of B200 roofline"
WORKLOAD = ("decode GEMV M=1: one Llama-3.1-8B layer's 7 projections "
            "(q,k,v,o,gate,up,down) in W8A8 int8 and in FP8 E4M3 per-row, per-token dynamic "
            "activation quantization fused")
HBM_FALLBACK_GBS = 6650.0


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["qlinear", "reference"], default="qlinear")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="CPU time budget of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=None)
    return ap.parse_args()


def algorithmic_bytes(scheme: int, N: int, K: int, M: int = 1) -> int:
    """Bytes the method must move for one product: weights, weight scales,
    bf16 activations in, bf16 outputs out."""
    sw = 4 * (N // 128) * (K // 128) if scheme == 2 else 4 * N
    return N * K + sw + 2 * M * K + 2 * M * N


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return json.load(f), "measured"
    except (OSError, ValueError):
        return {"hbm_gbs": HBM_FALLBACK_GBS, "bf16_tflops": 1590.0,
                "bf16_tflops_sustained": 1400.0}, "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while running."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,utilization.gpu,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.idx = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        if self.idx is None:
            return self
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.idx), "-lms", "50"], stdout=subprocess.PIPE,
                stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return self
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=5)
        sm, smax, reasons, util_sm = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                s, m, util = float(parts[0]), float(parts[1]), float(parts[3])
            except ValueError:
                continue
            sm.append(s)
            smax.append(m)
            if util > 0:
                util_sm.append(s)
                for n, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        load = util_sm or sm
        return {"sm_mhz": statistics.median(load) if load else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm), "samples_under_load": len(util_sm)}


def nvsmi_index(torch, dev: int):
    try:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
        out = subprocess.run(["nvidia-smi", "--query-gpu=index,uuid", "--format=csv,noheader"],
                             capture_output=True, text=True, timeout=20).stdout
        for ln in out.splitlines():
            i, u = [p.strip() for p in ln.split(",")]
            if u.replace("GPU-", "") == uuid.replace("GPU-", ""):
                return int(i)
    except Exception:
        pass
    return None


# ------------------------------------------------------------------ workload
def build_decode(torch, ql, synthetic, device, tokens=2):
    """Quantized weights (on the GPU, by the library's own quantizer) and a
    small rotation of input tokens for each projection."""
    work = []
    for name, N, K in synthetic.LLAMA31_8B:
        w = synthetic.make_w_device(N, K, seed=0, tag=f"llama31_8b.{name}", device=device)
        xs = synthetic.make_x_device(tokens, K, seed=0, tag=f"llama31_8b.{name}.x",
                                     outliers=synthetic.outlier_count(K), device=device)
        for scheme in (ql.W8A8_INT8_ROW, ql.FP8_E4M3_ROW):
            wq, sw = ql.quantize_weight(scheme, w)
            work.append(dict(name=name, scheme=scheme, N=N, K=K, wq=wq, sw=sw, xs=xs,
                             bytes=algorithmic_bytes(scheme, N, K)))
        del w
    torch.cuda.synchronize()
    return work


def capture_step_graphs(torch, ql, work, tokens, stream):
    """One CUDA graph per token slot, each holding the step's 14 GEMV launches."""
    for item in work:
        item["ys"] = [torch.empty((1, item["N"]), dtype=torch.bfloat16, device="cuda")
                      for _ in range(tokens)]
    # warm the launch path (device info, shared-memory attribute) before capture
    with torch.cuda.stream(stream):
        for item in work:
            ql.gemv(item["scheme"], item["xs"][0:1], item["wq"], item["sw"], y=item["ys"][0])
    stream.synchronize()
    graphs = []
    for t in range(tokens):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for item in work:
                ql.gemv(item["scheme"], item["xs"][t:t + 1], item["wq"], item["sw"], y=item["ys"][t])
        graphs.append(g)
    return graphs


def capture_e2e_graph(torch, ql, work, stream):
    """Graph of one end-to-end step: H2D of all 14 tokens (pinned host ->
    device), 14 public-API forward() calls, D2H of all outputs."""
    K_tot = sum(i["K"] for i in work)
    N_tot = sum(i["N"] for i in work)
    h_x = torch.empty(K_tot, dtype=torch.bfloat16, pin_memory=True)
    h_y = torch.empty(N_tot, dtype=torch.bfloat16, pin_memory=True)
    off = 0
    for i in work:
        h_x[off:off + i["K"]].copy_(i["xs"][0].cpu())
        off += i["K"]
    d_x = torch.empty(K_tot, dtype=torch.bfloat16, device="cuda")
    d_y = torch.empty(N_tot, dtype=torch.bfloat16, device="cuda")
    views = []
    ox = oy = 0
    for i in work:
        views.append((i, d_x[ox:ox + i["K"]].view(1, -1), d_y[oy:oy + i["N"]].view(1, -1)))
        ox += i["K"]
        oy += i["N"]
    with torch.cuda.stream(stream):
        for i, xv, yv in views:
            ql.forward(i["scheme"], xv, i["wq"], i["sw"], y=yv)
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        d_x.copy_(h_x, non_blocking=True)
        for i, xv, yv in views:
            ql.forward(i["scheme"], xv, i["wq"], i["sw"], y=yv)
        h_y.copy_(d_y, non_blocking=True)
    return g, 2 * K_tot, 2 * N_tot


# ------------------------------------------------------------------ CPU oracle
def oracle_decode_sample(budget_s: float, rows_cap=None):
    """Time the CPU oracle on the decode step (or a row sample of it) for about
    budget_s seconds.  Returns (GB/s, seconds, sample description)."""
    import numpy as np
    import oracle
    from fp8_linear_layers_b200 import synthetic
    items = []
    for name, N, K in synthetic.LLAMA31_8B:
        rows = N if rows_cap is None else min(N, rows_cap)
        w = synthetic.make_w(rows, K, seed=0, tag=f"oracle.llama31_8b.{name}")
        x = synthetic.make_x(1, K, seed=0, tag=f"oracle.llama31_8b.{name}.x",
                             outliers=synthetic.outlier_count(K))
        for scheme in (0, 1):
            wq, sw = oracle.quantize_weight(scheme, w)
            items.append((scheme, x, wq, sw, algorithmic_bytes(scheme, rows, K)))
    done_bytes, t_used, reps = 0, 0.0, 0
    while t_used < budget_s or reps == 0:
        t0 = time.perf_counter()
        for scheme, x, wq, sw, nb in items:
            oracle.forward(scheme, x, wq, sw)
            done_bytes += nb
        t_used += time.perf_counter() - t0
        reps += 1
    what = "full step" if rows_cap is None else f"first {rows_cap} output rows of each projection"
    return done_bytes / t_used / 1e9, t_used, f"{what} (14 GEMVs, M=1) x {reps} passes, {t_used:.1f} s"


# ------------------------------------------------------------------ main legs
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    # calibrate the per-step sample so that warmup + steps take about a minute
    from fp8_linear_layers_b200 import synthetic
    import oracle
    _, t64, _ = oracle_decode_sample(0.0, rows_cap=64)  # one pass over 64 rows per projection
    per_step_target = max(0.002, 60.0 / max(1, args.steps + args.warmup))
    rows = max(1, min(14336, int(64 * per_step_target / max(t64, 1e-6))))
    full_bytes = sum(algorithmic_bytes(s, N, K) for _, N, K in synthetic.LLAMA31_8B for s in (0, 1))
    import numpy as np
    items = []
    for name, N, K in synthetic.LLAMA31_8B:
        r = min(N, rows)
        w = synthetic.make_w(r, K, seed=0, tag=f"oracle.llama31_8b.{name}")
        x = synthetic.make_x(1, K, seed=0, tag=f"oracle.llama31_8b.{name}.x",
                             outliers=synthetic.outlier_count(K))
        for scheme in (0, 1):
            wq, sw = oracle.quantize_weight(scheme, w)
            items.append((scheme, x, wq, sw, algorithmic_bytes(scheme, r, K)))
    step_bytes = sum(i[4] for i in items)
    for _ in range(args.warmup):
        for scheme, x, wq, sw, _ in items:
            oracle.forward(scheme, x, wq, sw)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        for scheme, x, wq, sw, _ in items:
            oracle.forward(scheme, x, wq, sw)
    dt = time.perf_counter() - t0
    value = step_bytes * args.steps / dt / 1e9
    sample = (f"first {rows} output rows of each of the 14 projections (M=1), "
              f"{step_bytes / full_bytes * 100:.2f}% of a full step, per step")
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "impl": "reference",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "s8*s8->s32 (int8), e4m3*e4m3 exact (int64 fixed point)",
        "data": "synthetic (seeded N(0,1) tokens with 1% outlier channels x20; N(0,0.02) weights)",
        "config": {"workload": WORKLOAD, "M": 1, "note": "CPU oracle, single thread"},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist
    import fp8_linear_layers_b200 as ql
    from fp8_linear_layers_b200 import synthetic

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    dev = torch.cuda.current_device()

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(v: float) -> float:
        if world == 1:
            return v
        t = torch.tensor([v], dtype=torch.float64, device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    peaks, peak_src = measured_peaks()
    tokens = 2
    stream = torch.cuda.Stream()
    work = build_decode(torch, ql, synthetic, "cuda", tokens)
    graphs = capture_step_graphs(torch, ql, work, tokens, stream)
    launches_per_step = len(work)
    step_bytes = sum(i["bytes"] for i in work)

    sampler = ClockSampler(nvsmi_index(torch, dev) if rank == 0 else None).start()
    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            graphs[i % tokens].replay()
    stream.synchronize()
    barrier()
    torch.cuda.synchronize()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        ev0.record(stream)
        for i in range(args.steps):
            graphs[i % tokens].replay()
        ev1.record(stream)
    ev1.synchronize()
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop()
    ms_local = ev0.elapsed_time(ev1)
    ms = max_over_ranks(ms_local)
    value = world * step_bytes * args.steps / (ms / 1e3) / 1e9
    status, detail = ql.device_status(stream)
    if status != 0:
        raise RuntimeError(f"device status {status} detail {detail:#x} after the timed region")

    # per-projection kernel durations (outside the timed region), for the record
    per_kernel = {}
    for item in work:
        g = torch.cuda.CUDAGraph()
        y = item["ys"][0]
        with torch.cuda.graph(g, stream=stream):
            for _ in range(10):
                ql.gemv(item["scheme"], item["xs"][0:1], item["wq"], item["sw"], y=y)
        with torch.cuda.stream(stream):
            g.replay()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(5):
                g.replay()
            b.record(stream)
        b.synchronize()
        us = a.elapsed_time(b) * 1e3 / 50
        key = f"{ql.SCHEME_NAMES[item['scheme']]}.{item['name']}"
        per_kernel[key] = {"us": round(us, 2), "GB/s": round(item["bytes"] / us / 1e3, 1)}
        del g

    # end-to-end through the public API with host buffers
    e2e_steps = args.e2e_steps or max(10, min(args.steps, 2000))
    g_e2e, h2d, d2h = capture_e2e_graph(torch, ql, work, stream)
    with torch.cuda.stream(stream):
        for _ in range(min(args.warmup, 20)):
            g_e2e.replay()
            stream.synchronize()
    barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(e2e_steps):
            g_e2e.replay()
            stream.synchronize()  # the host reads each step's outputs
        e1.record(stream)
    e1.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1))
    e2e_value = world * step_bytes * e2e_steps / (e2e_ms / 1e3) / 1e9
    del g_e2e

    # roofline of the (only) kernel: average algorithmic bytes per launch over
    # the average launch duration inside the timed region
    per_launch_bytes = step_bytes / launches_per_step
    per_launch_s = (ms_local / 1e3) / (args.steps * launches_per_step)
    achieved = per_launch_bytes / per_launch_s / 1e9
    peak = float(peaks["hbm_gbs"])
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "traffic": None,
                "kernel": "ql::gemv_kernel", "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)"
                if peak_src == "measured" else "fallback 6.65 TB/s",
                "duration_source": "timed-region step time / launches (graph gaps included)"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        gbs, secs, sample = oracle_decode_sample(args.cpu_seconds)
        cpu = {"value": round(gbs, 4), "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample}

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "s8*s8->s32 (W8A8), e4m3*e4m3->f32 (FP8 row)",
            "data": "synthetic (seeded N(0,1) tokens with 1% outlier channels x20; N(0,0.02) "
                    "weights quantized on the GPU)",
            "config": {"workload": WORKLOAD, "M": 1,
                       "shapes": [f"{n} {N}x{K}" for n, N, K in synthetic.LLAMA31_8B],
                       "schemes": ["w8a8_int8_row", "fp8_e4m3_row"], "launches_per_step": launches_per_step,
                       "bytes_per_step": step_bytes, "parallelism": f"replicas x{world}",
                       "l2": "inputs larger than L2: 436 MB of weights streamed per step (L2 126 MB)",
                       "timing": "one CUDA graph replay per step, CUDA events on the launch stream"},
            "roofline": roofline,
            "cpu_baseline": cpu,
            "e2e": {"value": round(e2e_value, 1), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                    "how": "graph of H2D tokens + 14 forward() + D2H outputs, host sync per step"},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks,
            "per_kernel": per_kernel,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
