"""GPU parity: several M = 1 products in one grouped launch (qlinear_gemv_grouped).

Each product of a group must come out exactly as qlinear_gemv computes it
alone (the same per-row arithmetic: only the CTAs that stream it differ), and
so within the output tolerance of the oracle (bit for bit for int8).  Groups:
a layer's q|k|v and gate|up on one shared input, all K = 4096 products of a
Llama-3.1-8B layer on separate inputs, Qwen3-8B block-scheme groups, ragged
and tiny row counts, the largest group, and the argument checks.
"""
import numpy as np
import pytest
import torch

import fp8_linear_layers_b200 as ql
import oracle
from fp8_linear_layers_b200 import synthetic
from tests._util import assert_y_close, bf16_dev, bits, f32_dev, u8_dev

pytestmark = pytest.mark.gpu

LLAMA = dict((n, (N, K)) for n, N, K in synthetic.LLAMA31_8B)
QWEN = dict((n, (N, K)) for n, N, K in synthetic.QWEN3_8B)


def _group(scheme, shapes, shared_x, seed=0, outliers=None):
    """shapes: list of (name, N, K) with one K.  Returns host and device operands."""
    K = shapes[0][2]
    oc = synthetic.outlier_count(K) if outliers is None else outliers
    xs, ws = [], []
    x0 = synthetic.make_x(1, K, seed=seed, tag="grp-x", outliers=oc)
    for j, (name, N, _) in enumerate(shapes):
        x = x0 if shared_x else synthetic.make_x(1, K, seed=seed, tag=f"grp-x{j}", outliers=oc)
        w = synthetic.make_w(N, K, seed=seed, tag=f"grp-w.{name}.{j}")
        wq, sw = oracle.quantize_weight(scheme, w)
        xs.append(x)
        ws.append((wq, sw))
    return K, xs, ws


def _check_group(scheme, shapes, shared_x, seed=0, outliers=None):
    K, xs, ws = _group(scheme, shapes, shared_x, seed, outliers)
    dx = [bf16_dev(x) for x in xs]
    dw = [(u8_dev(wq), f32_dev(sw)) for wq, sw in ws]
    # outputs side by side in one buffer with a canary after each (16-byte aligned starts)
    sizes = [N for _, N, _ in shapes]
    span = [(N + 64 + 7) // 8 * 8 for N in sizes]
    buf = torch.full((sum(span),), -7.0, dtype=torch.bfloat16, device="cuda")
    ys, off = [], 0
    for N, sp in zip(sizes, span):
        ys.append(buf[off:off + N].view(1, N))
        off += sp
    ql.gemv_grouped(scheme, [(dx[j], dw[j][0], dw[j][1], ys[j]) for j in range(len(shapes))])
    torch.cuda.synchronize()
    assert ql.device_status()[0] == 0
    canary = bits(torch.tensor([-7.0], dtype=torch.bfloat16))[0]
    off = 0
    for j, (N, sp) in enumerate(zip(sizes, span)):
        assert np.all(bits(buf[off + N:off + sp]) == canary), f"product {j} wrote past its output"
        off += sp
    for j, (name, N, _) in enumerate(shapes):
        alone = ql.gemv(scheme, dx[j], dw[j][0], dw[j][1])
        torch.cuda.synchronize()
        got = bits(ys[j])
        assert np.array_equal(got, bits(alone)), f"{name}: grouped output differs from qlinear_gemv"
        ref = oracle.forward(scheme, xs[j], *ws[j])
        assert_y_close(got, ref, f"grouped {name} scheme {scheme}")
        if scheme == ql.W8A8_INT8_ROW:
            assert np.array_equal(got, ref), f"{name}: int8 outputs must match the oracle exactly"


@pytest.mark.parametrize("scheme", [ql.W8A8_INT8_ROW, ql.FP8_E4M3_ROW])
@pytest.mark.parametrize("names", [("q_proj", "k_proj", "v_proj"), ("gate_proj", "up_proj")])
def test_grouped_llama_shared_input(cuda, scheme, names):
    _check_group(scheme, [(n, *LLAMA[n]) for n in names], shared_x=True)


@pytest.mark.parametrize("scheme", [ql.W8A8_INT8_ROW, ql.FP8_E4M3_ROW])
def test_grouped_llama_all_k4096_separate_inputs(cuda, scheme):
    names = [n for n, (N, K) in LLAMA.items() if K == 4096]
    _check_group(scheme, [(n, *LLAMA[n]) for n in names], shared_x=False, seed=1)


@pytest.mark.parametrize("names", [("q_proj", "k_proj", "v_proj"), ("gate_proj", "up_proj"),
                                   ("q_proj", "k_proj", "v_proj", "o_proj", "gate_proj", "up_proj")])
def test_grouped_qwen_block(cuda, names):
    _check_group(ql.FP8_E4M3_BLOCK128, [(n, *QWEN[n]) for n in names], shared_x=len(names) < 6,
                 outliers=0)


@pytest.mark.parametrize("scheme", [ql.W8A8_INT8_ROW, ql.FP8_E4M3_ROW])
def test_grouped_ragged_and_tiny(cuda, scheme):
    shapes = [("a", 37, 1024), ("b", 1, 1024), ("c", 1000, 1024), ("d", 129, 1024), ("e", 8, 1024)]
    _check_group(scheme, shapes, shared_x=False, seed=2, outliers=3)


@pytest.mark.parametrize("scheme", [ql.W8A8_INT8_ROW, ql.FP8_E4M3_ROW, ql.FP8_E4M3_BLOCK128])
def test_grouped_largest_group_long_rows(cuda, scheme):
    # eight products of K = 14336 (two-row stages), more stages than SMs in total
    shapes = [(f"p{j}", 128 * (j + 1), 14336) for j in range(ql.GEMV_MAX_GROUP)]
    _check_group(scheme, shapes, shared_x=False, seed=3, outliers=0 if scheme == ql.FP8_E4M3_BLOCK128 else 20)


def test_grouped_single_product_equals_gemv(cuda):
    _check_group(ql.FP8_E4M3_ROW, [("down_proj", *LLAMA["down_proj"])], shared_x=True)


def test_grouped_argument_checks(cuda):
    K = 256
    x = torch.zeros((1, K), dtype=torch.bfloat16, device="cuda")
    wq = torch.zeros((100, K), dtype=torch.uint8, device="cuda")
    sw = torch.ones(100, dtype=torch.float32, device="cuda")
    L = ql.lib()
    table = (ql._GemvProblem * 9)(*[ql._GemvProblem(x.data_ptr(), 0, 0, wq.data_ptr(), sw.data_ptr(), 0, 100)] * 9)
    stream = torch.cuda.current_stream().cuda_stream
    import ctypes
    tp = ctypes.cast(table, ctypes.c_void_p)
    assert L.qlinear_gemv_grouped(ql.FP8_E4M3_ROW, tp, 0, K, stream) == 1   # empty group
    assert L.qlinear_gemv_grouped(ql.FP8_E4M3_ROW, tp, 9, K, stream) == 1   # above the limit
    assert L.qlinear_gemv_grouped(ql.FP8_E4M3_ROW, tp, 1, K, stream) == 1   # null y
    y = torch.zeros((1, 100), dtype=torch.bfloat16, device="cuda")
    table[0].y = y.data_ptr()
    assert L.qlinear_gemv_grouped(ql.FP8_E4M3_BLOCK128, tp, 1, K, stream) == 2  # N % 128 != 0
    table[0].y = y.data_ptr() + 2
    assert L.qlinear_gemv_grouped(ql.FP8_E4M3_ROW, tp, 1, K, stream) == 3   # misaligned
    assert L.qlinear_gemv_grouped(ql.FP8_E4M3_ROW, tp, 1, 100, stream) == 2  # K % 16 != 0
    torch.cuda.synchronize()
    assert torch.count_nonzero(y).item() == 0

