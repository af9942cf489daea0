"""GPU parity: the large-M tcgen05 GEMM (pre-quantized activations) vs the oracle.

Inputs are quantized by the oracle, so this file checks the product and the
epilogue alone.  Small and ragged shapes (several tiles, partial M / N tiles,
K not a multiple of the 128-byte stage) are compared output by output; the
prefill configurations (M in {512, 1024} x gate/up, down, fused qkv, W8A8;
Qwen3-8B FP8-block at M = 512) at full size on sampled outputs plus whole rows
and columns.  int8: int32 accumulators and bf16 outputs bit-exact; E4M3:
2^-7 |y| + 1e-3.
"""
import numpy as np
import pytest
import torch

import fp8_linear_layers_b200 as ql
import oracle
from fp8_linear_layers_b200 import synthetic
from tests._util import assert_y_close, bits, f32_dev, u8_dev

pytestmark = pytest.mark.gpu


def _inputs(scheme, M, N, K, seed=0, outliers=None):
    if outliers is None:
        outliers = synthetic.outlier_count(K) if scheme != ql.FP8_E4M3_BLOCK128 else 0
    x = synthetic.make_x(M, K, seed=seed, tag="gemm-x", outliers=outliers)
    w = synthetic.make_w(N, K, seed=seed, tag="gemm-w")
    qx, sx = oracle.quantize_act(scheme, x)
    wq, sw = oracle.quantize_weight(scheme, w)
    return qx, sx, wq, sw


def _gpu(scheme, qx, sx, wq, sw, want_acc=True):
    M, K = qx.shape
    N = wq.shape[0]
    dbg = None
    if want_acc:
        dbg = ql.Debug(acc_i32=torch.empty((M, N), dtype=torch.int32, device="cuda")
                       if scheme == ql.W8A8_INT8_ROW else None,
                       acc_f32=torch.empty((M, N), dtype=torch.float32, device="cuda")
                       if scheme == ql.FP8_E4M3_ROW else None)
    ws_n = ql.workspace_bytes(scheme, M, N, K)
    ws = ql.new_workspace(ws_n) if ws_n else None
    ypad = torch.full((M * N + 64,), -7.0, dtype=torch.bfloat16, device="cuda")
    y = ypad[:M * N].view(M, N)
    ql.gemm(scheme, u8_dev(qx), f32_dev(sx), u8_dev(wq), f32_dev(sw), workspace=ws, y=y, debug=dbg)
    st, detail = ql.device_status()
    assert st == 0, f"device status {st} detail {detail:#x}"
    assert np.all(bits(ypad[M * N:]) == bits(torch.tensor([-7.0], dtype=torch.bfloat16))[0]), \
        "gemm wrote past the end of y"
    return bits(y), dbg


@pytest.mark.parametrize("scheme", [ql.W8A8_INT8_ROW, ql.FP8_E4M3_ROW])
@pytest.mark.parametrize("M,N,K", [(128, 256, 128), (128, 256, 4096), (130, 300, 272), (33, 64, 48),
                                   (1, 1000, 1024), (257, 520, 1040), (384, 768, 2048),
                                   # 160- and 224-wide tiles (ragged last tile, N % 8 != 0)
                                   (384, 6288, 512), (200, 14224, 256), (200, 14220, 256)])
def test_gemm_small_shapes_full_compare(cuda, scheme, M, N, K):
    qx, sx, wq, sw = _inputs(scheme, M, N, K)
    gy, dbg = _gpu(scheme, qx, sx, wq, sw)
    ry, racc_i, racc_d = oracle.linear(scheme, qx, sx, wq, sw, want_acc=True)
    if scheme == ql.W8A8_INT8_ROW:
        assert np.array_equal(dbg.acc_i32.cpu().numpy(), racc_i), "int32 accumulators differ"
        assert np.array_equal(gy, ry), "int8 outputs must be bit-exact"
    else:
        acc = dbg.acc_f32.cpu().numpy().astype(np.float64)
        assert np.all(np.abs(acc - racc_d) <= 1e-5 * np.abs(racc_d).max() + 1e-6)
        assert_y_close(gy, ry, f"gemm {M}x{N}x{K}")


@pytest.mark.parametrize("M,N,K", [(128, 128, 128), (128, 256, 512), (200, 384, 640), (129, 1280, 1024),
                                   (40, 256, 4096)])
def test_gemm_block_small_shapes(cuda, M, N, K):
    scheme = ql.FP8_E4M3_BLOCK128
    qx, sx, wq, sw = _inputs(scheme, M, N, K, outliers=3)
    gy, _ = _gpu(scheme, qx, sx, wq, sw, want_acc=False)
    ry = oracle.linear(scheme, qx, sx, wq, sw)
    assert_y_close(gy, ry, f"gemm block {M}x{N}x{K}")


def _sampled_compare(scheme, M, N, K, nsamp=3000, seed=0):
    qx, sx, wq, sw = _inputs(scheme, M, N, K, seed=seed)
    gy, dbg = _gpu(scheme, qx, sx, wq, sw, want_acc=scheme == ql.W8A8_INT8_ROW)
    rng = np.random.default_rng(seed + 99)
    pm = np.concatenate([rng.integers(0, M, nsamp), np.full(N, M - 1), np.arange(M),
                         [0, M - 1, 0, M - 1]])
    pn = np.concatenate([rng.integers(0, N, nsamp), np.arange(N), np.full(M, N // 2 + 1),
                         [0, 0, N - 1, N - 1]])
    ry, racc_i, _ = oracle.linear_sampled(scheme, qx, sx, wq, sw, pm, pn, want_acc=True)
    if scheme == ql.W8A8_INT8_ROW:
        assert np.array_equal(dbg.acc_i32.cpu().numpy()[pm, pn], racc_i)
        assert np.array_equal(gy[pm, pn], ry)
    else:
        assert_y_close(gy[pm, pn], ry, f"gemm {M}x{N}x{K} sampled")


@pytest.mark.parametrize("M", [512, 1024])
@pytest.mark.parametrize("name,N,K", synthetic.LLAMA31_8B_PREFILL)
def test_gemm_prefill_w8a8_full_size(cuda, M, name, N, K):
    _sampled_compare(ql.W8A8_INT8_ROW, M, N, K)


@pytest.mark.parametrize("M", [512, 1024])
@pytest.mark.parametrize("name,N,K", synthetic.LLAMA31_8B_PREFILL)
def test_gemm_prefill_fp8_row_full_size(cuda, M, name, N, K):
    _sampled_compare(ql.FP8_E4M3_ROW, M, N, K, nsamp=1500)


@pytest.mark.parametrize("M", [512, 1024])
@pytest.mark.parametrize("name,N,K", synthetic.QWEN3_8B)
def test_gemm_qwen_block_full_size(cuda, M, name, N, K):
    _sampled_compare(ql.FP8_E4M3_BLOCK128, M, N, K, nsamp=1500)


@pytest.mark.parametrize("M,N,K", [(200, 384, 8192), (512, 1024, 8192), (512, 4096, 12288),
                                   (512, 1024, 4096), (128, 1024, 4096), (256, 128, 2048)])
def test_gemm_block_split_k(cuda, M, N, K):
    """Block scheme with few output tiles: with a workspace each tile's K
    blocks are split over 2 CTAs (256-wide tiles, K >= 8192) or 2 to 4 CTAs
    (128-wide tiles that fill at most a quarter of the SMs) that meet in f32
    partial sums; the outputs stay within the tolerance of the oracle, two
    calls in a row agree bit for bit (the parts are added in a fixed order
    whichever arrives last), the arrival counters are zero again afterwards,
    and without a workspace the call runs whole tiles."""
    scheme = ql.FP8_E4M3_BLOCK128
    ws_n = ql.workspace_bytes(scheme, M, N, K)
    # f32 partial tiles, then one arrival counter per tile (at most 64 tiles here: the last 256 bytes)
    assert ws_n > 256 * 1024
    slabs = ws_n - 256
    qx, sx, wq, sw = _inputs(scheme, M, N, K, outliers=3)
    args = (u8_dev(qx), f32_dev(sx), u8_dev(wq), f32_dev(sw))
    ws = ql.new_workspace(ws_n)
    y1 = ql.gemm(scheme, *args, workspace=ws)
    y2 = ql.gemm(scheme, *args, workspace=ws)
    y0 = ql.gemm(scheme, *args)
    st, detail = ql.device_status()
    assert st == 0, detail
    assert torch.count_nonzero(ws[slabs:]) == 0, "the arrival counters must be left zero"
    rng = np.random.default_rng(7)
    pm = np.concatenate([rng.integers(0, M, 2000), np.arange(M), np.full(N, M - 1)])
    pn = np.concatenate([rng.integers(0, N, 2000), np.full(M, N - 1), np.arange(N)])
    ry, _, _ = oracle.linear_sampled(scheme, qx, sx, wq, sw, pm, pn, want_acc=True)
    for tag, y in (("whole tiles", y0), ("split, first call", y1), ("split, second call", y2)):
        assert_y_close(bits(y)[pm, pn], ry, f"gemm block {M}x{N}x{K} {tag}")
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    # the same through qlinear_forward, whose workspace holds q_x, s_x and then the sums
    x = synthetic.make_x(M, K, seed=0, tag="gemm-x", outliers=3)
    wsf = ql.new_workspace(ql.forward_workspace_bytes(scheme, M, N, K))
    yf = ql.forward(scheme, torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16), args[2], args[3],
                    workspace=wsf)
    assert ql.device_status()[0] == 0
    assert_y_close(bits(yf)[pm, pn], ry, f"forward block {M}x{N}x{K}")


@pytest.mark.parametrize("scheme", [ql.W8A8_INT8_ROW, ql.FP8_E4M3_ROW])
@pytest.mark.parametrize("M,N,K", [(128, 256, 8192), (200, 384, 8192), (300, 1000, 8320)])
def test_gemm_row_split_k(cuda, scheme, M, N, K):
    """Row schemes with few 256-wide tiles and K >= 8192: with a workspace each
    tile's K blocks are split in two halves that park their raw accumulators
    (s32 / f32) and the second to arrive adds them before the scales.  Every
    output against the oracle (int8: accumulators and outputs bit-exact, and
    equal to whole tiles without a workspace); two calls agree bit for bit and
    leave the arrival counters zero."""
    ws_n = ql.workspace_bytes(scheme, M, N, K)
    assert ws_n > 256 * 1024
    qx, sx, wq, sw = _inputs(scheme, M, N, K, outliers=3)
    args = (u8_dev(qx), f32_dev(sx), u8_dev(wq), f32_dev(sw))
    ws = ql.new_workspace(ws_n)
    dbg = ql.Debug(acc_i32=torch.empty((M, N), dtype=torch.int32, device="cuda")
                   if scheme == ql.W8A8_INT8_ROW else None,
                   acc_f32=torch.empty((M, N), dtype=torch.float32, device="cuda")
                   if scheme == ql.FP8_E4M3_ROW else None)
    y1 = ql.gemm(scheme, *args, workspace=ws, debug=dbg)
    y2 = torch.full((M, N), -7.0, dtype=torch.bfloat16, device="cuda")
    ql.gemm(scheme, *args, workspace=ws, y=y2)
    y0 = ql.gemm(scheme, *args)
    st, detail = ql.device_status()
    assert st == 0, f"device status {st} detail {detail:#x}"
    assert torch.count_nonzero(ws[ws_n - 256:]) == 0, "the arrival counters must be left zero"
    ry, racc_i, racc_d = oracle.linear(scheme, qx, sx, wq, sw, want_acc=True)
    g1 = bits(y1)
    assert np.array_equal(g1, bits(y2)), "two calls on one workspace differ"
    if scheme == ql.W8A8_INT8_ROW:
        assert np.array_equal(dbg.acc_i32.cpu().numpy(), racc_i), "int32 accumulators differ"
        assert np.array_equal(g1, ry) and np.array_equal(bits(y0), ry)
    else:
        acc = dbg.acc_f32.cpu().numpy().astype(np.float64)
        assert np.all(np.abs(acc - racc_d) <= 1e-5 * np.abs(racc_d).max() + 1e-6)
        assert_y_close(g1, ry, f"gemm row split {M}x{N}x{K}")
        assert_y_close(bits(y0), ry, f"gemm row whole tiles {M}x{N}x{K}")


def test_forward_dispatches_large_m_through_quant_and_gemm(cuda):
    """qlinear_forward with M > 32: fused per-token quantization into the
    workspace, then the GEMM; compared with the oracle's whole method."""
    for scheme in ql.SCHEMES:
        M, N, K = 96, 256, 512
        x = synthetic.make_x(M, K, seed=3, tag="fwd-x", outliers=4)
        w = synthetic.make_w(N, K, seed=3, tag="fwd-w")
        wq, sw = oracle.quantize_weight(scheme, w)
        ws = ql.new_workspace(ql.forward_workspace_bytes(scheme, M, N, K))
        xd = torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)
        y = ql.forward(scheme, xd, u8_dev(wq), f32_dev(sw), workspace=ws)
        torch.cuda.synchronize()
        ry = oracle.forward(scheme, x, wq, sw)
        if scheme == ql.W8A8_INT8_ROW:
            assert np.array_equal(bits(y), ry)
        else:
            assert_y_close(bits(y), ry, "forward large M")
