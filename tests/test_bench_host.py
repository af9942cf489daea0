"""Host-side logic of bench.py (CPU only): the workloads' algorithmic amounts
against the shape totals, the oracle sample's description, the rule that a
DRAM-traffic figure is reported only for the kernel sources it was taken on,
the routing that decides each step's launch count, and the replay of exactly
K steps from chained step graphs."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

LLAMA_WEIGHT_BYTES = 218_103_808  # q/o 4096x4096, k/v 1024x4096, gate/up/down 14336x4096
QWEN_WEIGHT_BYTES = 192_937_984   # gate/up/down 12288x4096


def _weights(wl):
    return sum(p.N * p.K for p in wl.products)


def test_decode_layer_bytes():
    w = bench.workloads()
    dec = w["decode"]
    assert _weights(dec) == 2 * LLAMA_WEIGHT_BYTES  # int8 and FP8 per-row copies
    # weights + 4N scales + 2K x + 2N y per product
    extra = sum(4 * p.N + 2 * p.K + 2 * p.N for p in dec.products)
    assert sum(dec.amount(p) for p in dec.products) == 2 * LLAMA_WEIGHT_BYTES + extra == 436_879_360
    # the weight-only layer moves the same bytes through the same 14 products
    wo = w["decode-wo"]
    assert all(p.wo for p in wo.products) and not any(p.wo for p in dec.products)
    assert sorted((p.name, p.scheme, p.N, p.K) for p in wo.products) == \
        sorted((p.name, p.scheme, p.N, p.K) for p in dec.products)
    assert sum(wo.amount(p) for p in wo.products) == 436_879_360
    # the same 14 products, each its own launch
    sep = w["decode-separate"]
    assert sorted((p.name, p.scheme) for p in sep.products) == sorted((p.name, p.scheme) for p in dec.products)
    assert bench.step_amount(sep) == 436_879_360
    # grouped decode: per scheme q|k|v and gate|up read one input each, counted once:
    # 2 schemes x (2 + 1) duplicate 4096-wide bf16 inputs fewer
    groups = bench.input_groups(dec)
    assert [[p.name for p in g] for g in groups][:4] == [["q_proj", "k_proj", "v_proj"], ["o_proj"],
                                                         ["gate_proj", "up_proj"], ["down_proj"]]
    assert len(groups) == 8
    assert bench.step_amount(dec) == 436_879_360 - 2 * 3 * 2 * 4096
    # side by side along N: the same weight bytes in 8 products
    assert _weights(w["decode-fused"]) == 2 * LLAMA_WEIGHT_BYTES
    assert len(w["decode-fused"].products) == 8


def test_qwen_block_layer_bytes_and_scales():
    w = bench.workloads()
    q = w["qwen-decode"]
    assert _weights(q) == QWEN_WEIGHT_BYTES
    for p in q.products:  # one f32 scale per 128x128 block
        assert q.amount(p) == p.N * p.K + 4 * (p.N // 128) * (p.K // 128) + 2 * p.K + 2 * p.N


def test_prefill_ops():
    pre = bench.workloads()["prefill"]
    assert pre.unit == "TOPS" and pre.bound == "tensor"
    ops = {(p.M, p.name): pre.amount(p) for p in pre.products}
    assert ops[(512, "gate_proj")] == 2 * 512 * 14336 * 4096  # 60.13 G
    assert ops[(1024, "down_proj")] == 2 * 1024 * 4096 * 14336


def test_workload_kernels_and_bounds():
    w = bench.workloads()
    assert w["decode"].kernel == "ql::gemv_kernel" and w["decode"].bound == "hbm"
    assert w["decode-wo"].kernel == "ql::gemv_kernel (weight-only)"
    assert w["small"].kernel == "ql::gemm_small_kernel"
    assert w["qwen-prefill"].kernel == "ql::gemm_kernel"


def test_sample_description_caps_rows_at_n():
    w = bench.workloads()
    assert bench.sample_rows_text(w["kproj"], 10 ** 6) == \
        "first 1024 output rows of the workload's one product"
    assert bench.sample_rows_text(w["decode"], 300) == \
        "first 300 output rows of each of the 14 products"
    t = bench.sample_rows_text(w["decode"], 5000)
    assert t.startswith("first min(N, 5000)") and f"({2 * (4096 + 1024 + 1024 + 4096 + 4096) + 4 * 5000} rows" in t
    # block scheme: whole 128-row blocks
    assert bench.sample_rows_text(w["qwen-decode"], 300) == \
        "first 256 output rows of each of the 7 products"


def test_traffic_is_tied_to_kernel_sources(monkeypatch):
    wl = bench.workloads()["decode"]
    h = bench.kernel_source_hash(wl.kernel)
    assert h is not None and len(h) == 16
    monkeypatch.setitem(bench.TRAFFIC, "decode", (123, h, "profiles/x.md"))
    assert bench.measured_traffic(wl) == (123, "profiles/x.md")
    monkeypatch.setitem(bench.TRAFFIC, "decode", (123, "0" * 16, "profiles/x.md"))
    assert bench.measured_traffic(wl) == (None, None)
    # a workload without a capture reports null
    assert bench.measured_traffic(bench.workloads()["qwen-small"]) == (None, None)


def test_committed_traffic_summaries_exist():
    for key, (bytes_per_launch, _, path) in bench.TRAFFIC.items():
        assert os.path.exists(os.path.join(ROOT, path)), path
        wl = bench.workloads()[key]
        per_launch = bench.step_bytes(wl) / bench.dominant_launch_count(wl)
        if wl.bound == "hbm":
            # the recorded DRAM traffic is within 1% of the algorithmic bytes (no re-reads),
            # or within the ~50 KB every cold-cache launch adds (a 4 MB launch's 1%)
            assert abs(bytes_per_launch - per_launch) <= max(0.01 * per_launch, 64 * 1024)
        else:
            # GEMMs: no operand re-read from HBM; y may still sit in L2 when the kernel ends
            assert 0.6 * per_launch <= bytes_per_launch <= 1.02 * per_launch


def test_grouped_launch_counts():
    w = bench.workloads()
    assert bench.dominant_launch_count(w["decode"]) == 8
    assert bench.dominant_launch_count(w["decode-separate"]) == 14
    # prefill: per M, gate|up on one input, down, fused qkv
    assert bench.dominant_launch_count(w["prefill"]) == 6
    # Qwen3 block prefill: q|k|v, o, gate|up, down
    assert bench.dominant_launch_count(w["qwen-prefill"]) == 4
    # inputs arriving quantized, outputs leaving quantized: the same 4 launches, no quantization launch
    assert bench.dominant_launch_count(w["qwen-prefill-f2"]) == 4
    # small-M: per M and scheme, q|k|v and gate|up grouped, o and down alone
    assert bench.dominant_launch_count(w["small"]) == 4 * 2 * 4
    assert bench.dominant_launch_count(w["kproj"]) == 1
    # the step's bytes: decode reads each group's input once
    dec = w["decode"]
    assert bench.step_bytes(dec) == bench.step_amount(dec)


class _FakeRun:
    """CPU stand-in for bench.Runner: items whose outputs come from the oracle."""

    def __init__(self, items):
        self.items = items

    def _w(self, i, t):
        return i["wqs"][t % len(i["wqs"])]


def _fake_item(scheme, M, N, K, wo):
    import numpy as np
    import torch
    import oracle
    from fp8_linear_layers_b200 import synthetic
    x = synthetic.make_x(M, K, seed=2, tag=f"fake.{scheme}.{wo}", outliers=2)
    w = synthetic.make_w(N, K, seed=2, tag=f"fake.w.{scheme}")
    wq, sw = oracle.quantize_weight(scheme, w)
    y = oracle.linear_weight_only(scheme, x, wq, sw) if wo else oracle.forward(scheme, x, wq, sw)
    t16 = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
    p = bench.Product("fake", scheme, M, N, K, 2, wo=wo)
    return dict(p=p, xs=[t16(x)], ys=[t16(y)],
                wqs=[(torch.from_numpy(wq), torch.from_numpy(np.ascontiguousarray(sw)))])


def test_parity_sample_against_oracle_outputs():
    import torch
    items = [_fake_item(s, M, 256, 256, wo) for s in (0, 1, 2) for M, wo in ((1, False), (3, False), (1, True))]
    rep = bench.parity_sample(_FakeRun(items), torch, rows=8)
    assert rep["within_tolerance"] and rep["max_abs_err"] == 0.0
    assert rep["outputs"] == sum(i["p"].M * 8 for i in items)
    # a wrong output is reported
    items[4]["ys"][0][0, 3] = items[4]["ys"][0][0, 3] * 1.5 + 1.0
    rep = bench.parity_sample(_FakeRun(items), torch, rows=8)
    assert not rep["within_tolerance"] and rep["max_abs_err"] > 0.5


class _FakeGraph:
    """Stands in for a captured CUDA graph: records which steps a replay runs."""

    def __init__(self, log, steps):
        self.log, self.steps = log, steps

    def replay(self):
        self.log.extend(self.steps)


@pytest.mark.parametrize("copies,n", [(2, 300), (2, 7), (59, 200), (3, 16), (2, 0), (5, 1)])
def test_chained_steps_replay_exactly_k_steps_in_copy_order(copies, n):
    """Steps.run(0, n) replays n steps, step i on input copy i % copies, whether
    a step comes from the chain graph or from its copy's own graph."""
    chain = copies * max(1, -(-bench.STEP_CHAIN // copies))
    log = []
    singles = [_FakeGraph(log, [t]) for t in range(copies)]
    chained = _FakeGraph(log, [t % copies for t in range(chain)])
    bench.Steps(singles, chained, chain).run(0, n)
    assert log == [i % copies for i in range(n)]


def test_five_to_eight_tokens_route_follows_the_weight_bytes():
    """The GEMV takes 5-8 tokens only when the launch's weights are at most
    8 MiB (the library's rule); the launch count follows (one launch instead of
    a quantization launch and the split-K kernel)."""
    P = bench.Product
    kproj = bench.workloads()["kproj"]
    p = kproj.products[0]
    assert bench.gemv_route(p.M, p.K, [p])
    assert kproj.kernel == "ql::gemv_kernel"
    assert bench.gemv_route(8, 4096, [P("x", bench.INT8, 8, 2048, 4096, 0)])
    assert not bench.gemv_route(8, 4096, [P("x", bench.INT8, 8, 2056, 4096, 0)])
    assert not bench.gemv_route(8, 8208, [P("x", bench.INT8, 8, 8, 8208, 0)])
    assert not bench.gemv_route(9, 4096, [P("x", bench.INT8, 9, 8, 4096, 0)])
    assert bench.gemv_route(4, 8192) and not bench.gemv_route(4, 8208)
    # the small-M workload: at M = 8 every launch carries more than 8 MiB of weights
    small = bench.workloads()["small"]
    assert small.kernel == "ql::gemm_small_kernel"
