#!/usr/bin/env python3
"""Benchmark of the quantized decoder projection on B200.

Default workload ("decode", one step): M = 1 decode through one
Llama-3.1-8B layer's seven projections (q 4096x4096, k/v 1024x4096, o
4096x4096, gate/up 14336x4096, down 4096x14336) in W8A8 int8 and in FP8 E4M3
per-row: 14 GEMV launches (activation quantization fused) per step.  Metric:
HBM GB/s of algorithmic bytes (weights + scales + x + y) per second, whole job.

Other workloads (``--workload``), same JSON line:
  decode-fused  the decode layer with q|k|v and gate|up side by side along N: 8 GEMVs
  prefill       W8A8, M in {512, 1024} x gate/up/down/fused-qkv: TOPS
  small         M in {2, 8, 16, 32} x the 7 Llama shapes x {W8A8, FP8 row}: GB/s
  kproj         W8A8, M = 8, N = 1024, K = 4096 (8 outlier channels): GB/s
  qwen-decode   FP8 128x128 block, M = 1 x the 7 Qwen3-8B shapes: GB/s
  qwen-small    FP8 block, M = 32 x the Qwen shapes: GB/s
  qwen-prefill  FP8 block, M = 512 x the Qwen shapes: TOPS
  decode-wo     the decode layer as weight-only products (x not rounded; int8
                and FP8 per-row weights): 14 weight-only GEMVs, GB/s

Legs of the line:
  value     device time of K steps replayed from CUDA graphs (the pages decode
            under CUDA graphs), 16 or more consecutive steps per graph so that
            steps chain like a model's layers; inputs resident in HBM; decode
            and small-M steps stream more than L2 every step.
  e2e       the same metric through the public API (``forward``) with the
            step's activations copied host->device from pinned memory and the
            outputs read back device->host every step (captured in a graph,
            host synchronised per step).
  roofline  the dominant kernel's algorithmic bytes (or ops) per launch over
            its average launch duration, CUDA events, against the measured HBM
            copy bandwidth or the measured bf16 GEMM rate x the nominal
            8-bit/bf16 ratio of 2.
  cpu_baseline  the CPU oracle (test infrastructure) on a bounded row sample
            of the same workload, host cores; reported, not the target.

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
from dataclasses import dataclass, field

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "quantized linear: M=1 GEMV HBM GB/s; M≥512 int8/FP8 TOPS; % of B200 roofline"
HBM_FALLBACK_GBS = 6650.0
BF16_FALLBACK_TFLOPS = 1590.0
INT8, FP8R, FP8B = 0, 1, 2
SCHEME_NAME = {INT8: "w8a8_int8_row", FP8R: "fp8_e4m3_row", FP8B: "fp8_e4m3_block128"}


# ------------------------------------------------------------------ workloads
@dataclass
class Product:
    name: str
    scheme: int
    M: int
    N: int
    K: int
    outliers: int
    wo: bool = False  # weight-only product (activations not rounded)
    group: str = ""   # products of one (scheme, group) read one input; M = 1 ones share a launch
    pre: bool = False  # the input arrives quantized (codes + scales from its producer); with M > 32
                       # the product also quantizes its own output for the next product


@dataclass
class Workload:
    key: str
    description: str
    unit: str                # "GB/s" or "TOPS"
    products: list = field(default_factory=list)

    @property
    def bound(self):
        return "hbm" if self.unit == "GB/s" else "tensor"

    @property
    def kernel(self):
        p = self.products[0]
        if p.wo:
            return "ql::gemv_kernel (weight-only)"
        if p.M > 32 and p.pre:
            return "ql::gemm_kernel (output quantization fused)"
        if p.M == 1 or all(not g[0].pre and not g[0].wo and gemv_route(g[0].M, g[0].K, g)
                           for g in input_groups(self)):
            return "ql::gemv_kernel"
        return "ql::gemm_small_kernel" if p.M <= 32 else "ql::gemm_kernel"

    @staticmethod
    def input_bytes(p: Product) -> float:
        """Bytes of one product's input: bf16 x, or codes + f32 scales when it arrives quantized."""
        if not p.pre:
            return 2 * p.M * p.K
        return p.M * p.K + 4 * p.M * (p.K // 128 if p.scheme == FP8B else 1)

    def bytes_touched(self, p: Product) -> float:
        """Bytes one product reads and writes in HBM (weights, scales, x, y)."""
        sw = 4 * (p.N // 128) * (p.K // 128) if p.scheme == FP8B else 4 * p.N
        return p.N * p.K + sw + self.input_bytes(p) + 2 * p.M * p.N + p.M * p.K

    def amount(self, p: Product) -> float:
        """Algorithmic bytes (HBM-bound regimes) or ops (tensor-bound) of one product."""
        if self.unit == "TOPS":
            return 2.0 * p.M * p.N * p.K
        sw = 4 * (p.N // 128) * (p.K // 128) if p.scheme == FP8B else 4 * p.N
        return p.N * p.K + sw + self.input_bytes(p) + 2 * p.M * p.N


# The projections of a decoder layer that read one input: q, k, v (the
# normalised hidden state) and gate, up (the normalised attention output).
LAYER_INPUT = {"q_proj": "qkv", "k_proj": "qkv", "v_proj": "qkv", "gate_proj": "gate_up",
               "up_proj": "gate_up"}


def gemv_route(M: int, K: int, group=()) -> bool:
    """True when the library runs M-token products on bf16 input (`group`: the
    products of one launch) on the GEMV kernel: M = 1 up to K = 32768, two
    tokens up to 16384, three or four up to 8192, and five to eight up to 8192
    when the launch's weights take at most 8 MiB (two products of up to four
    tokens each)."""
    if (M == 1 and K <= 32768) or (M == 2 and K <= 16384) or (M in (3, 4) and K <= 8192):
        return True
    return 5 <= M <= 8 and K <= 8192 and sum(q.N * q.K for q in group) <= (8 << 20)


def workloads():
    from fp8_linear_layers_b200 import synthetic as S
    oc = S.outlier_count
    w = {}
    w["decode"] = Workload(
        "decode", "decode GEMV M=1: one Llama-3.1-8B layer's 7 projections (q,k,v,o,gate,up,down) "
        "in W8A8 int8 and in FP8 E4M3 per-row, per-token dynamic activation quantization fused; "
        "the projections that read one input (q|k|v, gate|up) run as one grouped launch each, "
        "from their own weight buffers: 4 launches per scheme", "GB/s",
        [Product(n, s, 1, N, K, oc(K), group=LAYER_INPUT.get(n, n))
         for s in (INT8, FP8R) for n, N, K in S.LLAMA31_8B])
    w["decode-separate"] = Workload(
        "decode-separate", "decode GEMV M=1: one Llama-3.1-8B layer's 7 projections in W8A8 int8 and in "
        "FP8 E4M3 per-row, each its own launch (14 launches per step)", "GB/s",
        [Product(n, s, 1, N, K, oc(K)) for n, N, K in S.LLAMA31_8B for s in (INT8, FP8R)])
    w["decode-fused"] = Workload(
        "decode-fused", "decode GEMV M=1: one Llama-3.1-8B layer with q|k|v and gate|up stored side by "
        "side along N (qkv 6144x4096, o 4096x4096, gate_up 28672x4096, down 4096x14336) in W8A8 int8 and "
        "in FP8 E4M3 per-row, per-token dynamic activation quantization fused", "GB/s",
        [Product(n, s, 1, N, K, oc(K)) for n, N, K in S.LLAMA31_8B_FUSED for s in (INT8, FP8R)])
    w["prefill"] = Workload(
        "prefill", "prefill W8A8 int8 GEMM: M in {512, 1024} x Llama-3.1-8B gate/up 14336x4096, "
        "down 4096x14336, fused qkv 6144x4096; per-token quantization + tcgen05 kind::i8; gate|up one "
        "grouped launch on their shared input", "TOPS",
        [Product(n, INT8, M, N, K, oc(K), group=LAYER_INPUT.get(n, n)) for M in (512, 1024)
         for n, N, K in S.LLAMA31_8B_PREFILL])
    w["small"] = Workload(
        "small", "small-batch tensor-core path: M in {2, 8, 16, 32} x the 7 Llama-3.1-8B shapes x "
        "{W8A8 int8, FP8 E4M3 per-row}, quantization fused; q|k|v and gate|up one grouped launch each "
        "on their shared tokens", "GB/s",
        [Product(n, s, M, N, K, oc(K), group=LAYER_INPUT.get(n, n)) for M in (2, 8, 16, 32)
         for s in (INT8, FP8R) for n, N, K in S.LLAMA31_8B])
    w["kproj"] = Workload(
        "kproj", "W8A8 int8 k_proj shape: X [8, 4096] with 8 outlier channels, W [1024, 4096]",
        "GB/s", [Product("k_proj", INT8, 8, 1024, 4096, 8)])
    w["decode-wo"] = Workload(
        "decode-wo", "weight-only decode GEMV M=1 (activations kept bf16, \"equivalent\" numerics): one "
        "Llama-3.1-8B layer's 7 projections with int8 and with FP8 E4M3 per-row weights", "GB/s",
        [Product(n, s, 1, N, K, oc(K), wo=True) for n, N, K in S.LLAMA31_8B for s in (INT8, FP8R)])
    w["qwen-decode"] = Workload(
        "qwen-decode", "Qwen3-8B FP8 128x128-block projections at M=1 (7 shapes; q|k|v and gate|up "
        "one grouped launch each on their shared input)", "GB/s",
        [Product(n, FP8B, 1, N, K, 0, group=LAYER_INPUT.get(n, n)) for n, N, K in S.QWEN3_8B])
    w["qwen-small"] = Workload(
        "qwen-small", "Qwen3-8B FP8 128x128-block projections at M=32 (7 shapes; q|k|v and gate|up one "
        "grouped launch each on their shared tokens)", "GB/s",
        [Product(n, FP8B, 32, N, K, 0, group=LAYER_INPUT.get(n, n)) for n, N, K in S.QWEN3_8B])
    w["decode-f2"] = Workload(
        "decode-f2", "decode GEMV M=1 as the decode workload, each input arriving already quantized "
        "(codes + scales written by its producer): q|k|v and gate|up grouped, 4 launches per scheme",
        "GB/s", [Product(n, s, 1, N, K, oc(K), group=LAYER_INPUT.get(n, n), pre=True)
                 for s in (INT8, FP8R) for n, N, K in S.LLAMA31_8B])
    w["small-f2"] = Workload(
        "small-f2", "small-batch tensor-core path as the small workload (M in {2, 8, 16, 32} x the 7 "
        "Llama-3.1-8B shapes x {W8A8, FP8 row}), each input arriving already quantized: one kernel "
        "per group (q|k|v and gate|up grouped on their shared tokens)", "GB/s",
        [Product(n, s, M, N, K, oc(K), group=LAYER_INPUT.get(n, n), pre=True) for M in (2, 8, 16, 32)
         for s in (INT8, FP8R) for n, N, K in S.LLAMA31_8B])
    w["qwen-prefill-f2"] = Workload(
        "qwen-prefill-f2", "Qwen3-8B FP8 128x128-block projections at M=512 (7 shapes), each input "
        "arriving already quantized and each product also writing its own output's E4M3 codes and "
        "per-128 scales for the product that reads it next: no quantization launch, q|k|v and gate|up "
        "one grouped launch each on their shared input", "TOPS",
        [Product(n, FP8B, 512, N, K, 0, group=LAYER_INPUT.get(n, n), pre=True) for n, N, K in S.QWEN3_8B])
    w["qwen-prefill"] = Workload(
        "qwen-prefill", "Qwen3-8B FP8 128x128-block projections at M=512 (7 shapes), per-K-block "
        "promotion; q|k|v and gate|up one grouped launch each on their shared input", "TOPS",
        [Product(n, FP8B, 512, N, K, 0, group=LAYER_INPUT.get(n, n)) for n, N, K in S.QWEN3_8B])
    return w


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["qlinear", "reference"], default="qlinear")
    ap.add_argument("--workload", default="decode",
                    choices=["decode", "decode-separate", "decode-fused", "prefill", "small", "kproj",
                             "qwen-decode", "qwen-small", "qwen-prefill", "decode-wo", "decode-f2",
                             "small-f2", "qwen-prefill-f2"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="CPU time budget of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="time only --workload (the default run also times the tensor-bound configs)")
    ap.add_argument("--e2e-steps", type=int, default=None)
    return ap.parse_args()


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "measured"
    except (OSError, ValueError):
        return {"hbm_gbs": HBM_FALLBACK_GBS, "bf16_tflops": BF16_FALLBACK_TFLOPS,
                "bf16_tflops_sustained": 1400.0}, "fallback"


def roofline_peak(wl: Workload):
    peaks, src = measured_peaks()
    if wl.unit == "GB/s":
        return float(peaks["hbm_gbs"]), f"{src} HBM copy bandwidth (hbm_gbs)"
    # 8-bit (int8 / E4M3) dense tensor rate = measured bf16 burst x nominal ratio 4.5/2.25
    return 2.0 * float(peaks["bf16_tflops"]), f"{src} bf16 GEMM burst x 2 (nominal 8-bit/bf16 ratio)"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while running."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,utilization.gpu,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.idx, self.proc, self.lines, self.thread = gpu_index, None, [], None

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


# ------------------------------------------------------------------ GPU legs
L2_BYTES = 126e6

# DRAM bytes per launch of the dominant kernel from one ncu capture (dram__bytes_read.sum +
# dram__bytes_write.sum), with the hash of the kernel sources it was taken on (the kernel's
# file and the device headers it includes; ql_internal.h declares host functions only): when
# the sources differ the figure no longer describes the kernel and the line reports null.
_GEMV_SOURCES = ["ql_gemv.cu", "ql_common.cuh", "ql_tc.cuh"]
_GEMM_SOURCES = ["ql_gemm.cu", "ql_common.cuh", "ql_tc.cuh"]
# the small-M workload's products run on the small-M kernel and (two tokens) on the GEMV
_SMALL_SOURCES = ["ql_gemm_small.cu", "ql_gemv.cu", "ql_common.cuh", "ql_tc.cuh"]
KERNEL_SOURCES = {"ql::gemv_kernel": _GEMV_SOURCES, "ql::gemv_kernel (weight-only)": _GEMV_SOURCES,
                  "ql::gemm_kernel": _GEMM_SOURCES, "ql::gemm_kernel (output quantization fused)": _GEMM_SOURCES,
                  "ql::gemm_small_kernel": _SMALL_SOURCES}
TRAFFIC = {
    # workload: (bytes per launch, kernel source hash, summary file)
    "decode": (54660384, "10803db7fb9f04b9", "profiles/gemv_decode_dram.md"),
    "kproj": (4325504, "10803db7fb9f04b9", "profiles/gemv_kproj_dram.md"),
    "prefill": (75848448, "87b077ff18efb3b1", "profiles/gemm_prefill_int8_dram.md"),
    "qwen-prefill": (52170240, "87b077ff18efb3b1", "profiles/gemm_qwen_prefill_block_dram.md"),
    "small": (55263000, "bb1a70d5446e5ea7", "profiles/gemm_small_dram.md"),
}


def kernel_source_hash(kernel: str):
    import hashlib
    files = KERNEL_SOURCES.get(kernel)
    if not files:
        return None
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "fp8_linear_layers_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_traffic(wl):
    t = TRAFFIC.get(wl.key)
    if t is None or kernel_source_hash(wl.kernel) != t[1]:
        return None, None
    return t[0], t[2]


class Runner:
    """Device buffers and launch closures for one workload (public API calls only).

    Products of one (scheme, group) read one input; M = 1 ones run as one
    grouped GEMV launch, M > 32 ones as one quantization of the input and one
    grouped GEMM launch.  Steps cycle through `copies` independent sets of
    quantized weights, activations and outputs, enough that the bytes touched
    by consecutive steps exceed twice the L2: no step finds its inputs in L2
    from an earlier one, so no flush is needed between timed steps.
    """

    def __init__(self, torch, ql, synthetic, wl: Workload):
        self.torch, self.ql, self.wl = torch, ql, wl
        per_step = sum(wl.bytes_touched(p) for p in wl.products)
        self.copies = max(2, -(-int(2 * L2_BYTES) // int(per_step)))
        self.groups = []  # [{"p0", "xs", "items"}] in launch order
        by_key = {}
        weights = {}
        for j, p in enumerate(wl.products):
            key = (p.scheme, p.M, p.K, p.wo, p.group) if p.group else j
            g = by_key.get(key)
            if g is None:
                xs = [synthetic.make_x_device(p.M, p.K, seed=t, tag=f"bench.{p.group or p.name}.x.M{p.M}",
                                              outliers=p.outliers) for t in range(self.copies)]
                g = by_key[key] = {"p0": p, "xs": xs, "items": []}
                # the step's input: bf16 x, or its codes + scales as a producer would write them
                g["x_in"] = [ql.quantize_act(p.scheme, x) for x in xs] if p.pre else xs
                self.groups.append(g)
            wkey = (p.name, p.N, p.K)
            if wkey not in weights:
                weights[wkey] = synthetic.make_w_device(p.N, p.K, seed=0, tag=f"bench.{p.name}")
            n_w = 1 if per_step >= 2 * L2_BYTES else self.copies
            wqs = [ql.quantize_weight(p.scheme, weights[wkey]) for _ in range(n_w)]
            ys = [torch.empty((p.M, p.N), dtype=torch.bfloat16, device="cuda") for _ in range(self.copies)]
            ws_bytes = ql.forward_workspace_bytes(p.scheme, p.M, p.N, p.K)
            ws = ql.new_workspace(ws_bytes) if ws_bytes else None
            item = dict(p=p, wqs=wqs, ys=ys, ws=ws, xs=g["xs"], amount=wl.amount(p))
            if p.pre and p.M > 32:  # the output's own codes and scales
                item["qy"] = [(torch.empty((p.M, p.N), dtype=torch.uint8, device="cuda"),
                               torch.empty((p.M, p.N // 128), dtype=torch.float32, device="cuda"))
                              for _ in range(self.copies)]
            g["items"].append(item)
        del weights
        for g in self.groups:
            p = g["p0"]
            if gemm_grouped_route(p) and not p.pre:
                # the step's quantized input (written by the step), a quantized copy of each
                # input for the dominant-kernel timing, and the group's K-split workspace
                g["qbuf"] = ql.quantize_act(p.scheme, g["xs"][0])
                g["q"] = [ql.quantize_act(p.scheme, x) for x in g["xs"]]
            if gemm_grouped_route(p):
                gws = ql.gemm_grouped_workspace_bytes(p.scheme, [i["p"].N for i in g["items"]], p.M, p.K)
                g["ws_gemm"] = ql.new_workspace(gws) if gws else None
            if small_grouped_route(p):
                g["ws_small"] = ql.new_workspace(
                    ql.gemm_small_grouped_workspace_bytes(p.scheme, [i["p"].N for i in g["items"]], p.M, p.K))
        torch.cuda.synchronize()
        self.items = [i for g in self.groups for i in g["items"]]
        self.step_amount = step_amount(wl)  # a group reads its one input once
        self.launches_per_step = sum(self._launches(g) for g in self.groups)
        self.dominant_launches = dominant_launch_count(wl)

    @staticmethod
    def _grouped(g) -> int:
        """1 when the group runs as one qlinear_gemv_grouped launch (every M = 1
        quantized product: a group of one included), else 0."""
        p = g["p0"]
        return int(p.M == 1 and not p.wo)

    def _launches(self, g) -> int:
        if self._grouped(g):
            return 1
        if gemm_grouped_route(g["p0"]):
            return 1 if g["p0"].pre else 2
        if small_grouped_route(g["p0"]):
            p = g["p0"]
            return 1 if (p.pre or gemv_route(p.M, p.K, [i["p"] for i in g["items"]])) else 2
        return sum(1 if (i["p"].wo or i["p"].pre or gemv_route(i["p"].M, i["p"].K, [i["p"]])) else 2
                   for i in g["items"])

    def _w(self, i, t):
        return i["wqs"][t % len(i["wqs"])]

    def _forward(self, i, x, wq, sw, y):
        p = i["p"]
        if p.wo:
            self.ql.gemv_weight_only(p.scheme, x, wq, sw, y=y)
        else:
            self.ql.forward(p.scheme, x, wq, sw, workspace=i["ws"], y=y)

    def _run_group(self, g, x, t, ys=None):
        """The group's products on input x (bf16, or a (codes, scales) pair when
        it arrives quantized) through the public API (grouped when M = 1)."""
        items = g["items"]
        ys = ys or [i["ys"][t] for i in items]
        if self._grouped(g):
            self.ql.gemv_grouped(g["p0"].scheme, [(x, *self._w(i, t), y) for i, y in zip(items, ys)])
        elif gemm_grouped_route(g["p0"]) and g["p0"].pre:
            qx, sx = x  # arrives quantized; each output also leaves quantized for its reader
            self.ql.gemm_grouped(g["p0"].scheme, qx, sx,
                                 [(*self._w(i, t), y, *i["qy"][t]) for i, y in zip(items, ys)],
                                 workspace=g["ws_gemm"])
        elif gemm_grouped_route(g["p0"]):
            qx, sx = g["qbuf"]
            self.ql.quantize_act(g["p0"].scheme, x, qx, sx)
            self.ql.gemm_grouped(g["p0"].scheme, qx, sx, [(*self._w(i, t), y) for i, y in zip(items, ys)],
                                 workspace=g["ws_gemm"])
        elif small_grouped_route(g["p0"]):
            self.ql.gemm_small_grouped(g["p0"].scheme, x, [(*self._w(i, t), y) for i, y in zip(items, ys)],
                                       g["ws_small"])
        else:
            for i, y in zip(items, ys):
                self._forward(i, x, *self._w(i, t), y)

    def step(self, t):
        for g in self.groups:
            self._run_group(g, g["x_in"][t], t)

    def dominant(self, t):
        """Launches of the dominant kernel alone (the product on quantized inputs)."""
        for g in self.groups:
            self.dominant_group(g, t)

    def dominant_group(self, g, t):
        ql = self.ql
        if self._grouped(g) or g["p0"].pre or small_grouped_route(g["p0"]):  # one launch (+ its quantization)
            self._run_group(g, g["x_in"][t], t)
        elif gemm_grouped_route(g["p0"]) and not g["p0"].pre:
            qx, sx = g["q"][t]
            ql.gemm_grouped(g["p0"].scheme, qx, sx, [(*self._w(i, t), i["ys"][t]) for i in g["items"]],
                            workspace=g["ws_gemm"])
        else:
            for i in g["items"]:
                p = i["p"]
                wq, sw = self._w(i, t)
                if p.wo:
                    ql.gemv_weight_only(p.scheme, i["xs"][t], wq, sw, y=i["ys"][t])
                else:  # M = 1 (2 <= M <= 32 and M > 32 run grouped)
                    ql.gemv(p.scheme, i["xs"][t], wq, sw, y=i["ys"][t])

    def capture(self, fn, stream):
        """Graphs of fn(t) for every input copy t, and one graph of a chain of
        consecutive steps (a whole number of copy cycles, at least 16 steps):
        see Steps."""
        torch = self.torch
        with torch.cuda.stream(stream):
            fn(0)  # warms the launch path (device info, attributes) before capture
        stream.synchronize()
        graphs = []
        for t in range(self.copies):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                fn(t)
            graphs.append(g)
        n = self.copies * max(1, -(-STEP_CHAIN // self.copies))
        chain = torch.cuda.CUDAGraph()
        with torch.cuda.graph(chain, stream=stream):
            for t in range(n):
                fn(t % self.copies)
        return Steps(graphs, chain, n)

    def e2e_graph(self, stream):
        """H2D of every group's input (pinned host -> device: bf16 x, or codes
        and scales), the public API calls, D2H of every output."""
        torch = self.torch
        ys_tot = sum(i["p"].M * i["p"].N for i in self.items)
        h_y = torch.empty(ys_tot, dtype=torch.bfloat16, pin_memory=True)
        d_y = torch.empty(ys_tot, dtype=torch.bfloat16, device="cuda")
        # every group's input in one pinned buffer and one device buffer (256-byte
        # aligned parts), so that a step's inputs cross in one copy
        srcs = []
        for g in self.groups:
            src = g["x_in"][0]
            srcs.append(list(src) if isinstance(src, tuple) else [src])
        sizes = [[a.numel() * a.element_size() for a in parts] for parts in srcs]
        total = sum((n + 255) // 256 * 256 for ns in sizes for n in ns)
        h_x = torch.empty(total, dtype=torch.uint8, pin_memory=True)
        d_x = torch.empty(total, dtype=torch.uint8, device="cuda")
        views, h2d, oy, ox = [], 0, 0, 0
        for g, parts, ns in zip(self.groups, srcs, sizes):
            dev = []
            for a, n in zip(parts, ns):
                h_x[ox:ox + n].copy_(a.contiguous().view(-1).view(torch.uint8).cpu())
                dev.append(d_x[ox:ox + n].view(a.dtype).view(a.shape))
                ox += (n + 255) // 256 * 256
                h2d += n
            yv = []
            for i in g["items"]:
                q = i["p"]
                yv.append(d_y[oy:oy + q.M * q.N].view(q.M, q.N))
                oy += q.M * q.N
            views.append((g, tuple(dev) if len(dev) > 1 else dev[0], yv))
        copies = [(d_x, h_x)]

        def body(c):
            for g, xv, yv in views:
                self._run_group(g, xv, c, ys=yv)

        with torch.cuda.stream(stream):
            body(0)
        stream.synchronize()
        graphs = []
        for c in range(self.copies):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for d, h in copies:
                    d.copy_(h, non_blocking=True)
                body(c)
                h_y.copy_(d_y, non_blocking=True)
            graphs.append(g)
        return graphs, h2d, 2 * ys_tot


def max_over_ranks_of(torch, dist, v: float, device) -> float:
    """The largest of every rank's v (the job's time is its slowest rank's)."""
    if dist is None:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(world: int, amount_per_step: float, steps: int, ms: float, scale: float) -> float:
    """Replicas: every rank runs the same step, so the job moves world x the
    step's amount in the max-over-ranks time."""
    return world * amount_per_step * steps / (ms / 1e3) / scale


def gemm_grouped_route(p: Product) -> bool:
    """True when a group of M > 32 products runs as one qlinear_gemm_grouped
    launch (a group of one included), after one quantization of its input
    unless the input arrives quantized."""
    return p.M > 32 and not p.wo


def small_grouped_route(p: Product) -> bool:
    """True when a group of 2 <= M <= 32 products runs as one
    qlinear_gemm_small_grouped call (a group of one included)."""
    return 2 <= p.M <= 32 and not p.wo


def dominant_launch_count(wl) -> int:
    """Launches of the dominant kernel in one step: one per group that runs
    grouped (M = 1 quantized GEMV, 2 <= M <= 32 small-M, M > 32 GEMM), else one
    per product."""
    n = 0
    for g in input_groups(wl):
        p = g[0]
        n += 1 if ((p.M == 1 and not p.wo) or gemm_grouped_route(p) or small_grouped_route(p)) else len(g)
    return n


def step_bytes(wl) -> float:
    """Algorithmic HBM bytes of one step's dominant launches: weights, scales,
    the kernel's input (q_x and s_x when M > 32; a group's input once) and y."""
    total = 0.0
    for g in input_groups(wl):
        for j, p in enumerate(g):
            sw = 4 * (p.N // 128) * (p.K // 128) if p.scheme == FP8B else 4 * p.N
            if p.M > 32:
                inp = p.M * p.K + 4 * p.M * (p.K // 128 if p.scheme == FP8B else 1)
            else:
                inp = Workload.input_bytes(p)
            total += p.N * p.K + sw + 2 * p.M * p.N + (inp if j == 0 else 0)
    return total


def input_groups(wl):
    """Products grouped by the input they read, in launch order."""
    groups = {}
    for j, p in enumerate(wl.products):
        key = (p.scheme, p.M, p.K, p.wo, p.group) if p.group else j
        groups.setdefault(key, []).append(p)
    return list(groups.values())


def step_amount(wl) -> float:
    """Algorithmic amount of one step: a group's shared input counts once."""
    total = sum(wl.amount(p) for p in wl.products)
    if wl.unit == "GB/s":
        total -= sum((len(g) - 1) * Workload.input_bytes(g[0]) for g in input_groups(wl))
    return total


def workload_config(wl):
    return {"workload": wl.description, "key": wl.key,
            "products": [f"{SCHEME_NAME[p.scheme]} M={p.M} {p.name} {p.N}x{p.K}" for p in wl.products],
            "input_groups": ["|".join(p.name for p in g) + f" ({SCHEME_NAME[g[0].scheme]})"
                             for g in input_groups(wl) if len(g) > 1],
            "amount_per_step": step_amount(wl)}


# Steps replayed as one graph: a decode forward runs its layers inside one graph,
# where each kernel's start overlaps the previous one's end (programmatic
# dependent launch); a graph boundary per step would add a full drain and a
# graph launch that the model does not pay.
STEP_CHAIN = 16


class Steps:
    """Step i runs input copy i % copies: `chain` consecutive steps from a
    multiple of `chain` (a multiple of the copies) replay as one captured graph
    of those steps, any other step as the graph of its copy alone.  Every
    kernel reads and writes global memory only after its grid-dependency wait
    (before it: weight loads and shared-memory set-up), so a step's first
    kernels may overlap the previous step's last ones exactly as the kernels
    inside a step overlap."""

    def __init__(self, singles, chain_graph, chain):
        self.singles, self.chain_graph, self.chain = singles, chain_graph, chain

    def run(self, i0, n):
        i, end = i0, i0 + n
        while i < end:
            if i % self.chain == 0 and i + self.chain <= end:
                self.chain_graph.replay()
                i += self.chain
            else:
                self.singles[i % len(self.singles)].replay()
                i += 1


def timed(torch, stream, steps_graphs, steps):
    """Device time (ms) of `steps` steps from step 0, CUDA events on the stream."""
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        steps_graphs.run(0, steps)
        e1.record(stream)
    e1.synchronize()
    return e0.elapsed_time(e1)


# ------------------------------------------------------------------ CPU oracle
def _host_bits(torch, t):
    """bf16 tensor -> uint16 bit patterns on the host."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view("uint16")


def parity_sample(run, torch, rows: int = 8):
    """The step's outputs (input copy 0) against the CPU oracle on the first
    `rows` output rows of every product: the largest absolute and relative
    error and whether every sampled output is within 2^-7 |y| + 1e-3.  A
    report beside the throughput; the parity tests are the gate."""
    import numpy as np
    import oracle
    max_abs, max_rel, ok, count = 0.0, 0.0, True, 0
    for i in run.items:
        p = i["p"]
        wq, sw = run._w(i, 0)
        r = min(rows, p.N)
        sub = 128 if p.scheme == FP8B else r  # block scales cover 128-row blocks
        x = _host_bits(torch, i["xs"][0])
        wq_h = np.ascontiguousarray(wq[:sub].cpu().numpy())
        sw_h = np.ascontiguousarray((sw[:1] if p.scheme == FP8B else sw[:sub]).cpu().numpy())
        if p.wo:
            ref = oracle.linear_weight_only(p.scheme, x, wq_h, sw_h, 0, r)
        else:
            qx, sx = oracle.quantize_act(p.scheme, x)
            ref = oracle.linear_rows(p.scheme, qx, sx, wq_h, sw_h, 0, r)
        got = _host_bits(torch, i["ys"][0])[:, :r]
        g, e = oracle.bf16_bits_to_f64(got), oracle.bf16_bits_to_f64(ref)
        err = np.abs(g - e)
        max_abs = max(max_abs, float(err.max()))
        nz = np.abs(e) > 0
        if nz.any():
            max_rel = max(max_rel, float((err[nz] / np.abs(e[nz])).max()))
        ok = ok and bool(np.all(err <= 2.0 ** -7 * np.abs(e) + 1e-3))
        count += got.size
    return {"outputs": count, "rows_per_product": rows, "max_abs_err": max_abs,
            "max_rel_err": max_rel, "within_tolerance": ok, "tolerance": "2^-7 |y_oracle| + 1e-3"}


def _oracle_items(wl: Workload, rows_cap: int):
    import oracle
    from fp8_linear_layers_b200 import synthetic
    items = []
    for p in wl.products:
        rows = min(p.N, rows_cap)
        if p.scheme == FP8B:
            rows = max(128, rows // 128 * 128)
        w = synthetic.make_w(rows, p.K, seed=0, tag=f"oracle.{p.name}")
        x = synthetic.make_x(p.M, p.K, seed=0, tag=f"oracle.{p.name}.x", outliers=p.outliers)
        wq, sw = oracle.quantize_weight(p.scheme, w)
        # kind: "wo" weight-only; "pre" input already quantized (the codes are
        # the oracle's, made here, outside the timed work); "preq" also
        # quantizes the product's output; None the whole method from bf16 x
        kind = "wo" if p.wo else (("preq" if p.M > 32 else "pre") if p.pre else None)
        xin = oracle.quantize_act(p.scheme, x) if p.pre else x
        items.append((p.scheme, xin, wq, sw,
                      wl.amount(Product(p.name, p.scheme, p.M, rows, p.K, 0, pre=p.pre)), kind))
    return items


_POOL = {}


def host_threads() -> int:
    """The host's cores (nproc: the CPU set this process may run on)."""
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except (AttributeError, OSError):
        return max(1, os.cpu_count() or 1)


def _oracle_run(scheme, x, wq, sw, kind, threads=1):
    """One product through the oracle (kind as in _oracle_items); with threads
    > 1 its output rows are split over host threads (the oracle's C calls
    release the GIL; the block scheme keeps whole 128-row blocks).  The
    arithmetic is the oracle's."""
    import oracle
    wo = kind == "wo"
    if kind in ("pre", "preq"):
        qx, sx = x
        if threads <= 1:
            y = oracle.linear(scheme, qx, sx, wq, sw)
        else:
            y = _oracle_rows(lambda b: oracle.linear_rows(scheme, qx, sx, wq, sw, b[0], b[1]),
                             scheme, wq.shape[0], threads)
            y = __import__("numpy").concatenate(y, axis=1)
        if kind == "preq":
            oracle.quantize_act(scheme, y)
        return y
    if threads <= 1:
        return oracle.linear_weight_only(scheme, x, wq, sw) if wo else oracle.forward(scheme, x, wq, sw)
    if wo:
        fn = lambda b: oracle.linear_weight_only(scheme, x, wq, sw, b[0], b[1])  # noqa: E731
    else:
        qx, sx = oracle.quantize_act(scheme, x)
        fn = lambda b: oracle.linear_rows(scheme, qx, sx, wq, sw, b[0], b[1])  # noqa: E731
    return _oracle_rows(fn, scheme, wq.shape[0], threads)


def _oracle_rows(fn, scheme, N, threads):
    """fn over output-row ranges on a pool of host threads."""
    import concurrent.futures
    if threads not in _POOL:
        _POOL[threads] = concurrent.futures.ThreadPoolExecutor(max_workers=threads)
    step = -(-N // threads)
    if scheme == FP8B:
        step = -(-step // 128) * 128
    bounds = [(n0, min(N, n0 + step)) for n0 in range(0, N, step)]
    return list(_POOL[threads].map(fn, bounds))


def sample_rows_text(wl: Workload, rows_cap: int) -> str:
    """The output rows the oracle sample covers: the first rows_cap of each
    product, capped at the product's N (whole 128-row blocks for the block scheme)."""
    counts = []
    for p in wl.products:
        rows = min(p.N, rows_cap)
        if p.scheme == FP8B:
            rows = max(128, rows // 128 * 128)
        counts.append(rows)
    if len(counts) == 1:
        return f"first {counts[0]} output rows of the workload's one product"
    if len(set(counts)) == 1:
        return f"first {counts[0]} output rows of each of the {len(counts)} products"
    return (f"first min(N, {rows_cap}) output rows of each of the {len(counts)} products "
            f"({sum(counts)} rows in all)")


def oracle_sample(wl: Workload, budget_s: float, rows_cap: int, threads: int = 1):
    """The CPU oracle (whole method from bf16 X) on the first rows_cap output
    rows of every product of the workload, repeated for about budget_s, on
    `threads` host threads.
    Returns (throughput in the workload's unit, seconds, passes, amount per pass)."""
    items = _oracle_items(wl, rows_cap)
    per_pass = sum(i[4] for i in items)
    done, t_used, passes = 0.0, 0.0, 0
    while t_used < budget_s or passes == 0:
        t0 = time.perf_counter()
        for scheme, x, wq, sw, amt, kind in items:
            _oracle_run(scheme, x, wq, sw, kind, threads)
            done += amt
        t_used += time.perf_counter() - t0
        passes += 1
    scale = 1e9 if wl.unit == "GB/s" else 1e12
    return done / t_used / scale, t_used, passes, per_pass


def pick_rows(wl: Workload, seconds: float, threads: int = 1) -> int:
    """Rows per product so that one oracle pass on `threads` threads takes about `seconds`."""
    probe = 8 * threads
    _, t, _, _ = oracle_sample(wl, 0.0, probe, threads)
    return max(1, int(probe * seconds / max(t, 1e-6)))


def cpu_baseline(wl, seconds: float, step_amount: float) -> dict:
    """The oracle on all host cores (threads over output rows) and on one
    thread, each on a bounded row sample of the workload for about `seconds`."""
    out = {}
    for threads in (host_threads(), 1):
        rows = pick_rows(wl, min(seconds, 4.0), threads)
        v, secs, passes, per_pass = oracle_sample(wl, seconds, rows, threads)
        out[threads] = {"value": round(v, 6), "unit": wl.unit, "cores": threads, "kind": "oracle",
                        "sample": f"{sample_rows_text(wl, rows)} "
                                  f"({100 * per_pass / step_amount:.3g}% of a step) x {passes} passes, "
                                  f"{secs:.1f} s, {threads} host thread{'s' if threads > 1 else ''}"}
    top = out[host_threads()]
    if host_threads() > 1:
        top["single_thread"] = {k: out[1][k] for k in ("value", "sample")}
    return top


def base_line(wl, args, world):
    return {"metric": METRIC, "unit": wl.unit, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": ("bf16 x (int8|e4m3 weights as f16) -> f32 (weight-only)" if wl.products[0].wo
                      else "s8*s8->s32 (W8A8), e4m3*e4m3->f32 (FP8)"),
            "data": "synthetic (seeded N(0,1) activations with outlier channels x20; N(0,0.02) weights)"}


def run_reference(args):
    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    import oracle
    wl = workloads()[args.workload]
    threads = host_threads()
    per_step = max(0.002, 60.0 / max(1, args.steps + args.warmup))
    rows = pick_rows(wl, per_step, threads)
    items = _oracle_items(wl, rows)
    step_amount = sum(i[4] for i in items)
    for _ in range(args.warmup):
        for scheme, x, wq, sw, _, kind in items:
            _oracle_run(scheme, x, wq, sw, kind, threads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        for scheme, x, wq, sw, _, kind in items:
            _oracle_run(scheme, x, wq, sw, kind, threads)
    dt = time.perf_counter() - t0
    scale = 1e9 if wl.unit == "GB/s" else 1e12
    value = step_amount * args.steps / dt / scale
    full = sum(wl.amount(p) for p in wl.products)
    sample = (f"{sample_rows_text(wl, rows)}, "
              f"{100 * step_amount / full:.3g}% of a full step, per step; {threads} host threads "
              f"over output rows")
    line = base_line(wl, args, args.gpus)
    line.update({"value": value, "impl": "reference", "ms_per_step": dt / args.steps * 1e3,
                 "dtype": ("f64 sums of exact bf16 x dequantized-weight products" if wl.products[0].wo
                           else "s8*s8->s32 (int8), e4m3*e4m3 exact (int64 fixed point)"),
                 "config": {**workload_config(wl), "parallelism": f"replicas x{args.gpus}",
                            "note": "CPU oracle, the plain definition, on a row sample per step"},
                 "cpu_baseline": {"value": value, "unit": wl.unit, "cores": threads, "kind": "oracle",
                                  "sample": sample},
                 "e2e": {"value": value, "unit": wl.unit, "h2d_bytes_per_step": 0,
                         "d2h_bytes_per_step": 0}})
    print(json.dumps(line), flush=True)
    return 0


# Configurations timed after the headline in the default run, each reported
# under "extra" in the same line: the W8A8 k_proj case (M = 8), W8A8 prefill
# (M = 512, 1024) and the Qwen3-8B block scheme at M = 512.
EXTRA_WORKLOADS = ("kproj", "prefill", "qwen-prefill")


def per_product_times(torch, run, stream, wl, peak, scale, reps=50):
    """Each product's dominant-kernel launches (its group's, when grouped)
    timed alone: graph replays cycling through the input copies, CUDA events;
    the product's algorithmic amount over its time, and that against the
    roofline peak."""
    out = []
    for g in run.groups:
        def fn(t, g=g):
            run.dominant_group(g, t)
        graphs = run.capture(fn, stream)
        with torch.cuda.stream(stream):
            graphs.run(0, graphs.chain + 5)  # every graph warm
        ms = timed(torch, stream, graphs, reps) / reps
        amount = sum(i["amount"] for i in g["items"])
        if wl.unit == "GB/s":  # a grouped launch reads its shared input once
            amount -= (len(g["items"]) - 1) * Workload.input_bytes(g["p0"])
        v = amount / (ms / 1e3) / scale
        p = g["p0"]
        out.append({"products": "|".join(i["p"].name for i in g["items"]), "scheme": SCHEME_NAME[p.scheme],
                    "M": p.M, "us": round(ms * 1e3, 2), "value": round(v, 1), "frac": round(v / peak, 4)})
        del graphs
    return out


def measure(torch, ql, synthetic, wl, args, steps, warmup, world, rank, barrier, max_over_ranks,
            cpu_seconds):
    """Every leg of one workload's line: the timed graph replays, the dominant
    kernel's own launches (roofline), end to end from host buffers, the parity
    report and the oracle baseline.  Returns the line's fields."""
    scale = 1e9 if wl.unit == "GB/s" else 1e12
    stream = torch.cuda.Stream()
    run = Runner(torch, ql, synthetic, wl)
    graphs = run.capture(run.step, stream)

    # ---- timed region: K steps (chains of steps captured as one graph)
    with torch.cuda.stream(stream):
        graphs.run(0, warmup)
        if warmup < graphs.chain:
            graphs.chain_graph.replay()  # the chain graph warm too (untimed)
    stream.synchronize()
    barrier()
    torch.cuda.synchronize()
    ms_local = timed(torch, stream, graphs, steps)
    torch.cuda.synchronize()
    barrier()
    ms = max_over_ranks(ms_local)
    value = whole_job_value(world, run.step_amount, steps, ms, scale)
    status, detail = ql.device_status(stream)
    if status != 0:
        raise RuntimeError(f"device status {status} detail {detail:#x} after the timed region")
    del graphs

    # ---- the dominant kernel's own launches (for the roofline), same kind of timing
    dgraphs = run.capture(run.dominant, stream)
    dsteps = max(3, min(steps, 500))
    with torch.cuda.stream(stream):
        dgraphs.run(0, dgraphs.chain + min(warmup, 10))
    d_ms = timed(torch, stream, dgraphs, dsteps)
    n_dom = run.dominant_launches
    per_launch_amount = run.step_amount / n_dom
    per_launch_s = (d_ms / 1e3) / (dsteps * n_dom)
    achieved = per_launch_amount / per_launch_s / scale
    peak, peak_src = roofline_peak(wl)
    traffic, traffic_src = measured_traffic(wl)
    roofline = {"bound": wl.bound, "achieved": round(achieved, 1), "peak": round(peak, 1),
                "unit": wl.unit, "frac": round(achieved / peak, 4), "traffic": traffic,
                "traffic_source": traffic_src,
                "kernel": wl.kernel, "peak_source": peak_src,
                "duration_source": "CUDA events over graph replays of this kernel's launches "
                                   "(inputs already quantized where the step quantizes separately)"}
    del dgraphs
    per_product = per_product_times(torch, run, stream, wl, peak, scale) if len(run.groups) > 1 else None

    # ---- end to end through the public API with host buffers
    e2e_steps = args.e2e_steps or max(10, min(steps, 1000))
    g_e2e, h2d, d2h = run.e2e_graph(stream)
    with torch.cuda.stream(stream):
        for i in range(min(warmup, 10)):
            g_e2e[i % len(g_e2e)].replay()
            stream.synchronize()
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for i in range(e2e_steps):
            g_e2e[i % len(g_e2e)].replay()
            stream.synchronize()  # the host reads every step's outputs
        e1.record(stream)
    e1.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1))
    e2e_value = whole_job_value(world, run.step_amount, e2e_steps, e2e_ms, scale)
    del g_e2e

    # ---- the outputs against the oracle on a row sample (rank 0; never fatal)
    parity = None
    if rank == 0:
        try:
            with torch.cuda.stream(stream):
                run.step(0)
            stream.synchronize()
            parity = parity_sample(run, torch)
        except Exception as exc:  # the report must not cost the bench line
            parity = {"error": f"{type(exc).__name__}: {exc}"}

    cpu = None
    if rank == 0 and world == 1 and cpu_seconds > 0:
        cpu = cpu_baseline(wl, cpu_seconds, run.step_amount)
    weight_bytes = sum(p.N * p.K for p in wl.products)
    out = {
        "metric": METRIC, "unit": wl.unit, "value": round(value, 1), "ms_per_step": ms / steps,
        "steps": steps, "warmup": warmup,
        "config": {**workload_config(wl),
                   "launches_per_step": run.launches_per_step,
                   "parallelism": f"replicas x{world}",
                   "l2": (f"inputs larger than L2 (126 MB): consecutive steps cycle through "
                          f"{run.copies} sets of weights/activations/outputs, "
                          f"{run.copies * sum(wl.bytes_touched(p) for p in wl.products) / 1e6:.0f} MB "
                          f"touched per cycle ({weight_bytes / 1e6:.0f} MB of weights per step); no flush"),
                   "timing": (f"steps replayed {STEP_CHAIN}+ at a time as one captured CUDA graph "
                              "(each step's kernels overlap the previous step's by programmatic dependent "
                              "launch, as layers inside one model graph), CUDA events on the launch stream")},
        "roofline": roofline,
        **({"per_product": per_product} if per_product else {}),
        "parity": parity,
        "cpu_baseline": cpu,
        "e2e": {"value": round(e2e_value, 1), "unit": wl.unit, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "how": "graph of H2D activations + the public API per product (grouped where a "
                       "layer's products read one input) + D2H outputs, host sync per step"},
        "gpu_launches": run.launches_per_step * steps,
    }
    del run
    torch.cuda.empty_cache()
    return out


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
        return max_over_ranks_of(torch, dist if world > 1 else None, v, "cuda")

    cpu_s = 0.0 if args.no_cpu_baseline else args.cpu_seconds
    # one clock record spans every leg of every workload of the line
    sampler = ClockSampler(nvsmi_index(torch, dev) if rank == 0 else None).start()
    wl = workloads()[args.workload]
    head = measure(torch, ql, synthetic, wl, args, args.steps, args.warmup, world, rank, barrier,
                   max_over_ranks, cpu_s)
    extra = {}
    if args.workload == "decode" and not args.no_extra:
        # the tensor-bound configurations, each timed the same way; fewer steps
        # (each of their steps is 10-400 us) so the whole run stays within minutes
        for key in EXTRA_WORKLOADS:
            xs = max(3, min(args.steps, 200))
            extra[key] = measure(torch, ql, synthetic, workloads()[key], args, xs, max(3, min(args.warmup, 20)),
                                 world, rank, barrier, max_over_ranks, min(cpu_s, 6.0))
    clocks = sampler.stop()

    if rank == 0:
        line = base_line(wl, args, world)
        line.update(head)
        line["clocks"] = clocks
        if extra:
            line["extra"] = extra
            line["gpu_launches"] = head["gpu_launches"] + sum(e["gpu_launches"] for e in extra.values())
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
