"""GPU parity: several large-M products on one quantized input in one launch
(qlinear_gemm_grouped).

Each product keeps its own weights, scales and output; the launch deals the
output tiles of all of them to the same CTAs.  Checks: every output against
the oracle (int8 bit-exact; E4M3 within 2^-7 |y| + 1e-3), int8 and E4M3-row
outputs bit-equal to qlinear_gemm on each product alone (the same tiles, the
same accumulation order), outputs written only inside their own range
(canaries between them), ragged M and N, the block scheme's K split planned
on the group (two calls on one workspace bit-identical, counters left zero),
and the argument checks.  Shapes: a Llama-3.1-8B layer's gate|up at prefill
(M = 512, 1024), a Qwen3-8B layer's q|k|v and gate|up (M = 512) on sampled
outputs with whole rows and columns, and small ragged groups compared output
by output.
"""
import ctypes

import numpy as np
import pytest
import torch

import fp8_linear_layers_b200 as ql
import oracle
from fp8_linear_layers_b200 import synthetic
from tests._util import assert_y_close, bits, f32_dev, u8_dev

pytestmark = pytest.mark.gpu

LLAMA = dict((n, (N, K)) for n, N, K in synthetic.LLAMA31_8B)
QWEN = dict((n, (N, K)) for n, N, K in synthetic.QWEN3_8B)
CANARY = -7.0


def _operands(scheme, M, Ns, K, seed, outliers=None):
    if outliers is None:
        outliers = 0 if scheme == ql.FP8_E4M3_BLOCK128 else synthetic.outlier_count(K)
    x = synthetic.make_x(M, K, seed=seed, tag="ggemm-x", outliers=outliers)
    qx, sx = oracle.quantize_act(scheme, x)
    ws = [oracle.quantize_weight(scheme, synthetic.make_w(N, K, seed=seed, tag=f"ggemm-w{j}"))
          for j, N in enumerate(Ns)]
    return qx, sx, ws


def _run_group(scheme, qx, sx, ws, M, workspace=None):
    """Outputs side by side in one buffer, a canary span after each."""
    Ns = [wq.shape[0] for wq, _ in ws]
    span = [(M * N + 64 + 7) // 8 * 8 for N in Ns]
    buf = torch.full((sum(span),), CANARY, dtype=torch.bfloat16, device="cuda")
    ys, off = [], 0
    for N, sp in zip(Ns, span):
        ys.append(buf[off:off + M * N].view(M, N))
        off += sp
    dws = [(u8_dev(wq), f32_dev(sw)) for wq, sw in ws]
    ql.gemm_grouped(scheme, u8_dev(qx), f32_dev(sx), [(wq, sw, y) for (wq, sw), y in zip(dws, ys)],
                    workspace=workspace)
    torch.cuda.synchronize()
    st, detail = ql.device_status()
    assert st == 0, f"device status {st} detail {detail:#x}"
    canary = bits(torch.tensor([CANARY], dtype=torch.bfloat16))[0]
    off = 0
    for j, (N, sp) in enumerate(zip(Ns, span)):
        assert np.all(bits(buf[off + M * N:off + sp]) == canary), f"product {j} wrote past its output"
        off += sp
    return [bits(y) for y in ys], dws


def _alone(scheme, qx, sx, dws, workspace_for=None):
    out = []
    for wq, sw in dws:
        M, K, N = qx.shape[0], qx.shape[1], wq.shape[0]
        n = ql.workspace_bytes(scheme, M, N, K)
        w = ql.new_workspace(n) if (n and workspace_for) else None
        out.append(bits(ql.gemm(scheme, u8_dev(qx), f32_dev(sx), wq, sw, workspace=w)))
    torch.cuda.synchronize()
    return out


def _sampled(scheme, qx, sx, wq, sw, got, what, seed=0, nsamp=1500):
    M, N = got.shape
    rng = np.random.default_rng(seed)
    pm = np.concatenate([rng.integers(0, M, nsamp), np.full(N, M - 1), np.arange(M), [0, M - 1]])
    pn = np.concatenate([rng.integers(0, N, nsamp), np.arange(N), np.full(M, N // 2 + 1), [N - 1, 0]])
    ry, _, _ = oracle.linear_sampled(scheme, qx, sx, wq, sw, pm, pn, want_acc=True)
    if scheme == ql.W8A8_INT8_ROW:
        assert np.array_equal(got[pm, pn], ry), f"{what}: int8 outputs must be bit-exact"
    else:
        assert_y_close(got[pm, pn], ry, what)


# the E4M3 row scheme at M = 512 only (its M = 1024 tiles are those of W8A8)
@pytest.mark.parametrize("scheme,M", [(ql.W8A8_INT8_ROW, 512), (ql.W8A8_INT8_ROW, 1024),
                                      (ql.FP8_E4M3_ROW, 512)])
def test_grouped_llama_gate_up(cuda, scheme, M):
    names = ("gate_proj", "up_proj")
    K = LLAMA["gate_proj"][1]
    qx, sx, ws = _operands(scheme, M, [LLAMA[n][0] for n in names], K, seed=11)
    got, dws = _run_group(scheme, qx, sx, ws, M)
    alone = _alone(scheme, qx, sx, dws)
    for j, n in enumerate(names):
        assert np.array_equal(got[j], alone[j]), f"{n}: grouped output differs from qlinear_gemm"
        _sampled(scheme, qx, sx, *ws[j], got[j], f"grouped {n} M={M}", seed=j)


@pytest.mark.parametrize("names", [("q_proj", "k_proj", "v_proj"), ("gate_proj", "up_proj")])
def test_grouped_qwen_block(cuda, names):
    scheme, M = ql.FP8_E4M3_BLOCK128, 512
    K = QWEN[names[0]][1]
    qx, sx, ws = _operands(scheme, M, [QWEN[n][0] for n in names], K, seed=12)
    Ns = [QWEN[n][0] for n in names]
    n_ws = ql.gemm_grouped_workspace_bytes(scheme, Ns, M, K)
    got, _ = _run_group(scheme, qx, sx, ws, M, workspace=ql.new_workspace(n_ws) if n_ws else None)
    for j, n in enumerate(names):
        _sampled(scheme, qx, sx, *ws[j], got[j], f"grouped block {n}", seed=j)


@pytest.mark.parametrize("scheme", ql.SCHEMES)
def test_grouped_ragged_full_compare(cuda, scheme):
    """Four products of different N (ragged last tiles for the row schemes),
    ragged M; every output compared with the oracle."""
    M, K = 300, 1024
    Ns = [128, 640, 384, 1024] if scheme == ql.FP8_E4M3_BLOCK128 else [1000, 8, 520, 129]
    qx, sx, ws = _operands(scheme, M, Ns, K, seed=13, outliers=3)
    got, dws = _run_group(scheme, qx, sx, ws, M)
    alone = _alone(scheme, qx, sx, dws)
    for j, (wq, sw) in enumerate(ws):
        ry = oracle.linear(scheme, qx, sx, wq, sw)
        if scheme == ql.W8A8_INT8_ROW:
            assert np.array_equal(got[j], ry), f"product {j}: int8 outputs must be bit-exact"
        else:
            assert_y_close(got[j], ry, f"grouped ragged product {j}")
        if scheme != ql.FP8_E4M3_BLOCK128:
            assert np.array_equal(got[j], alone[j]), f"product {j}: grouped output differs from qlinear_gemm"


def test_grouped_block_k_split(cuda):
    """Block scheme, a group whose 256-wide tiles fill at most half the SMs
    with K >= 8192: each tile's K blocks split over two CTAs that meet in the
    workspace; two calls agree bit for bit and leave the counters zero."""
    scheme, M, K = ql.FP8_E4M3_BLOCK128, 256, 8192
    Ns = [1024, 2048]
    n_ws = ql.gemm_grouped_workspace_bytes(scheme, Ns, M, K)
    assert n_ws > 256 * 1024
    qx, sx, ws = _operands(scheme, M, Ns, K, seed=14, outliers=3)
    wsp = ql.new_workspace(n_ws)
    got1, _ = _run_group(scheme, qx, sx, ws, M, workspace=wsp)
    got2, _ = _run_group(scheme, qx, sx, ws, M, workspace=wsp)
    got0, _ = _run_group(scheme, qx, sx, ws, M)  # whole tiles without a workspace
    assert torch.count_nonzero(wsp[n_ws - 256:]) == 0, "the arrival counters must be left zero"
    for j, (wq, sw) in enumerate(ws):
        assert np.array_equal(got1[j], got2[j])
        ry = oracle.linear(scheme, qx, sx, wq, sw)
        assert_y_close(got1[j], ry, f"grouped split product {j}")
        assert_y_close(got0[j], ry, f"grouped whole-tile product {j}")


@pytest.mark.parametrize("M", [512, 300])
def test_grouped_quant_out(cuda, M):
    """Block scheme, q|k|v in one launch that also writes each output's E4M3
    codes and per-128 scales for the product that reads it next: y equals the
    grouped launch's y without them, bit for bit, and the codes and scales
    equal the oracle's quantization of that bf16 y, bit for bit; a codes-only
    call (no y) writes the same codes."""
    scheme = ql.FP8_E4M3_BLOCK128
    names = ("q_proj", "k_proj", "v_proj")
    K = QWEN["q_proj"][1]
    Ns = [QWEN[n][0] for n in names]
    qx, sx, ws = _operands(scheme, M, Ns, K, seed=15)
    dqx, dsx = u8_dev(qx), f32_dev(sx)
    dws = [(u8_dev(wq), f32_dev(sw)) for wq, sw in ws]
    n_ws = ql.gemm_grouped_workspace_bytes(scheme, Ns, M, K)
    wsp = ql.new_workspace(n_ws) if n_ws else None
    y_ref = ql.gemm_grouped(scheme, dqx, dsx, [(wq, sw, None) for wq, sw in dws], workspace=wsp)
    q = [(torch.empty((M, N), dtype=torch.uint8, device="cuda"),
          torch.empty((M, N // 128), dtype=torch.float32, device="cuda")) for N in Ns]
    ys = ql.gemm_grouped(scheme, dqx, dsx, [(wq, sw, None, *q[j]) for j, (wq, sw) in enumerate(dws)],
                         workspace=wsp)
    q2 = [(torch.empty_like(a), torch.empty_like(b)) for a, b in q]
    ql.gemm_grouped(scheme, dqx, dsx, [(wq, sw, False, *q2[j]) for j, (wq, sw) in enumerate(dws)], workspace=wsp)
    torch.cuda.synchronize()
    assert ql.device_status()[0] == 0
    for j, n in enumerate(names):
        yb = bits(ys[j])
        assert np.array_equal(yb, bits(y_ref[j])), f"{n}: y differs from the grouped launch without codes"
        rq, rs = oracle.quantize_act(scheme, yb)
        assert np.array_equal(q[j][1].cpu().numpy().view(np.uint32), rs.view(np.uint32)), f"{n}: output scales"
        assert np.array_equal(q[j][0].cpu().numpy(), rq), f"{n}: output codes"
        assert np.array_equal(q2[j][0].cpu().numpy(), rq) and torch.equal(q2[j][1], q[j][1])
        _sampled(scheme, qx, sx, *ws[j], yb, f"grouped quant-out {n}", seed=j, nsamp=500)


def test_grouped_argument_checks(cuda):
    M, K, N = 64, 256, 256
    qx = torch.zeros((M, K), dtype=torch.uint8, device="cuda")
    sx = torch.ones(M, dtype=torch.float32, device="cuda")
    wq = torch.zeros((N, K), dtype=torch.uint8, device="cuda")
    sw = torch.ones(N, dtype=torch.float32, device="cuda")
    y = torch.zeros((M, N), dtype=torch.bfloat16, device="cuda")
    L = ql.lib()
    table = (ql._GemmProblem * 5)(*[ql._GemmProblem(wq.data_ptr(), sw.data_ptr(), y.data_ptr(), 0, 0, N)] * 5)
    tp = ctypes.cast(table, ctypes.c_void_p)
    stream = torch.cuda.current_stream().cuda_stream
    args = (qx.data_ptr(), sx.data_ptr())
    assert L.qlinear_gemm_grouped(ql.W8A8_INT8_ROW, *args, tp, 0, M, K, None, 0, stream) == 1  # empty
    assert L.qlinear_gemm_grouped(ql.W8A8_INT8_ROW, *args, tp, 5, M, K, None, 0, stream) == 1  # > 4
    assert L.qlinear_gemm_grouped(ql.W8A8_INT8_ROW, *args, None, 1, M, K, None, 0, stream) == 1
    table[1].y = 0
    assert L.qlinear_gemm_grouped(ql.W8A8_INT8_ROW, *args, tp, 2, M, K, None, 0, stream) == 1  # null y
    table[1].y = y.data_ptr()
    table[1].N = 200
    assert L.qlinear_gemm_grouped(ql.FP8_E4M3_BLOCK128, *args, tp, 2, M, K, None, 0, stream) == 2  # N % 128
    assert L.qlinear_gemm_grouped(ql.W8A8_INT8_ROW, *args, tp, 2, M, 100, None, 0, stream) == 2  # K % 16
    # output codes: all products or none, block scheme only
    qy = torch.zeros((M, N), dtype=torch.uint8, device="cuda")
    sy = torch.zeros((M, N // 128), dtype=torch.float32, device="cuda")
    table[1].N = N
    table[0].qy, table[0].sy = qy.data_ptr(), sy.data_ptr()
    assert L.qlinear_gemm_grouped(ql.FP8_E4M3_BLOCK128, *args, tp, 2, M, K, None, 0, stream) == 1
    table[1].qy = qy.data_ptr()
    assert L.qlinear_gemm_grouped(ql.FP8_E4M3_BLOCK128, *args, tp, 2, M, K, None, 0, stream) == 1  # no sy
    table[1].sy = sy.data_ptr()
    assert L.qlinear_gemm_grouped(ql.W8A8_INT8_ROW, *args, tp, 2, M, K, None, 0, stream) == 2
    torch.cuda.synchronize()
    assert torch.count_nonzero(y).item() == 0 and torch.count_nonzero(qy).item() == 0
    assert ql.gemm_grouped_workspace_bytes(ql.W8A8_INT8_ROW, [N, N], M, K) == 0
    assert ql.gemm_grouped_workspace_bytes(ql.FP8_E4M3_BLOCK128, [], M, K) == 0
