"""GPU parity: several 1 <= M <= 32 products on the same tokens in one launch
(qlinear_gemm_small_grouped).

The tokens are quantized once and the weight tiles of every product share
one SM-balanced K split (or, up to four tokens within the GEMV's K limits,
one grouped GEMV launch).  Checks: every output against the oracle (int8
bit-exact; E4M3 within 2^-7 |y| + 1e-3), int8 outputs bit-equal to
qlinear_gemm_small on each product alone, outputs written only inside their
own range (canaries), ragged N, pre-quantized tokens, a second call on the
same workspace, and the argument checks.  Shapes: a Llama-3.1-8B layer's
q|k|v and gate|up at M in {2, 3, 8, 16, 32}, a Qwen3-8B layer's in the block
scheme, and small ragged groups.
"""
import numpy as np
import pytest
import torch

import fp8_linear_layers_b200 as ql
import oracle
from fp8_linear_layers_b200 import synthetic
from tests._util import assert_y_close, bf16_dev, bits, f32_dev, oracle_forward_par, u8_dev

pytestmark = pytest.mark.gpu

LLAMA = dict((n, (N, K)) for n, N, K in synthetic.LLAMA31_8B)
QWEN = dict((n, (N, K)) for n, N, K in synthetic.QWEN3_8B)
CANARY = -7.0


def _group(scheme, M, Ns, K, seed, outliers):
    x = synthetic.make_x(M, K, seed=seed, tag="gsmall-x", outliers=outliers)
    ws = [oracle.quantize_weight(scheme, synthetic.make_w(N, K, seed=seed, tag=f"gsmall-w{j}"))
          for j, N in enumerate(Ns)]
    return x, ws


def _run(scheme, xin, dws, M, Ns, K, workspace):
    span = [(M * N + 64 + 7) // 8 * 8 for N in Ns]
    buf = torch.full((sum(span),), CANARY, dtype=torch.bfloat16, device="cuda")
    ys, off = [], 0
    for N, sp in zip(Ns, span):
        ys.append(buf[off:off + M * N].view(M, N))
        off += sp
    ql.gemm_small_grouped(scheme, xin, [(wq, sw, y) for (wq, sw), y in zip(dws, ys)], workspace)
    torch.cuda.synchronize()
    st, detail = ql.device_status()
    assert st == 0, f"device status {st} detail {detail:#x}"
    canary = bits(torch.tensor([CANARY], dtype=torch.bfloat16))[0]
    off = 0
    for j, (N, sp) in enumerate(zip(Ns, span)):
        assert np.all(bits(buf[off + M * N:off + sp]) == canary), f"product {j} wrote past its output"
        off += sp
    return [bits(y) for y in ys]


def _check(scheme, M, names_or_ns, K, seed=0, outliers=None, model=LLAMA, pre=False):
    Ns = [model[n][0] if isinstance(n, str) else n for n in names_or_ns]
    if outliers is None:
        outliers = 0 if scheme == ql.FP8_E4M3_BLOCK128 else synthetic.outlier_count(K)
    x, ws = _group(scheme, M, Ns, K, seed, outliers)
    dws = [(u8_dev(wq), f32_dev(sw)) for wq, sw in ws]
    dx = bf16_dev(x)
    xin = ql.quantize_act(scheme, dx) if pre else dx
    n_ws = ql.gemm_small_grouped_workspace_bytes(scheme, Ns, M, K)
    wsp = ql.new_workspace(n_ws)
    got = _run(scheme, xin, dws, M, Ns, K, wsp)
    again = _run(scheme, xin, dws, M, Ns, K, wsp)  # the workspace is left ready for the next call
    for j, (wq, sw) in enumerate(ws):
        ref = oracle_forward_par(scheme, x, wq, sw)
        what = f"grouped small product {j} (N={Ns[j]}) M={M} scheme {scheme}"
        assert_y_close(got[j], ref, what)
        assert_y_close(again[j], ref, what + ", second call")
        if scheme == ql.W8A8_INT8_ROW:
            assert np.array_equal(got[j], ref) and np.array_equal(again[j], ref), what
            one = ql.new_workspace(ql.workspace_bytes(scheme, M, Ns[j], K))
            alone = ql.gemm_small(scheme, dx, *dws[j], one)
            torch.cuda.synchronize()
            assert np.array_equal(bits(alone), got[j]), what + ": differs from qlinear_gemm_small"


# the E4M3 row scheme at M = 2, 8 and 32 (W8A8 also at 3 and 16)
@pytest.mark.parametrize("scheme,M", [(ql.W8A8_INT8_ROW, m) for m in (2, 3, 8, 16, 32)] +
                         [(ql.FP8_E4M3_ROW, m) for m in (2, 8, 32)])
@pytest.mark.parametrize("names", [("q_proj", "k_proj", "v_proj"), ("gate_proj", "up_proj")])
def test_grouped_small_llama(cuda, M, scheme, names):
    _check(scheme, M, names, LLAMA[names[0]][1], seed=M)


@pytest.mark.parametrize("M", [2, 8, 32])
@pytest.mark.parametrize("names", [("q_proj", "k_proj", "v_proj"), ("gate_proj", "up_proj")])
def test_grouped_small_qwen_block(cuda, M, names):
    _check(ql.FP8_E4M3_BLOCK128, M, names, QWEN[names[0]][1], seed=M, model=QWEN)


@pytest.mark.parametrize("scheme", ql.SCHEMES)
@pytest.mark.parametrize("M", [4, 7, 32])
def test_grouped_small_ragged(cuda, scheme, M):
    """Four products of different N (ragged last tiles for the row schemes;
    a one-tile product beside long ones), K past the GEMV's limits at M = 4."""
    K = 8320 if M == 4 and scheme != ql.FP8_E4M3_BLOCK128 else 1024
    if scheme == ql.FP8_E4M3_BLOCK128:
        Ns = [128, 640, 384, 1024]
        K = 8448 if M == 4 else 1024
    else:
        Ns = [1000, 8, 520, 129]
    _check(scheme, M, Ns, K, seed=20 + M, outliers=3)


@pytest.mark.parametrize("scheme", [ql.W8A8_INT8_ROW, ql.FP8_E4M3_BLOCK128])
@pytest.mark.parametrize("M", [2, 16])
def test_grouped_small_prequantized_tokens(cuda, scheme, M):
    """Tokens arriving quantized (codes and scales from their producer): the
    tensor-core kernel for every M, no quantization launch; the same outputs
    as the bf16-input call (int8 bit for bit)."""
    model = QWEN if scheme == ql.FP8_E4M3_BLOCK128 else LLAMA
    _check(scheme, M, ("q_proj", "k_proj", "v_proj"), 4096, seed=30 + M, model=model, pre=True)
