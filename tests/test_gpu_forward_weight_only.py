"""GPU parity: the weight-only product for 1 <= M <= 32 tokens vs the oracle.

Up to four tokens ride on the GEMV kernel's spare MMA columns (each token
staged with its own power of two) within its K limits (16384 for one or two
tokens, 8192 for three or four); every other shape runs on the tensor
cores (tcgen05 kind::f16, the codes converted to bf16 in shared memory, K
split over the SMs).  Llama-3.1-8B shapes, Qwen3-8B block shapes, ragged
shapes, workspace reuse across calls, and the argument limits.
"""
import numpy as np
import pytest
import torch

import fp8_linear_layers_b200 as ql
import oracle
from fp8_linear_layers_b200 import synthetic
from tests._util import assert_y_close, bf16_dev, bits, f32_dev, oracle_wo_par, u8_dev

pytestmark = pytest.mark.gpu

def _run(scheme, M, N, K, seed=0, outliers=None):
    if outliers is None:
        outliers = synthetic.outlier_count(K)
    x = synthetic.make_x(M, K, seed=seed, tag=f"fwo-x{M}", outliers=outliers)
    w = synthetic.make_w(N, K, seed=seed, tag="fwo-w")
    wq, sw = oracle.quantize_weight(scheme, w)
    ypad = torch.full((M * N + 64,), -12345.0, dtype=torch.bfloat16, device="cuda")
    y = ypad[:M * N].view(M, N)
    nb = ql.weight_only_workspace_bytes(scheme, M, N, K)
    ws = ql.new_workspace(nb) if nb else None
    ref = oracle_wo_par(scheme, x, wq, sw)
    for call in range(2):  # the workspace is left ready for the next call of this shape
        ql.forward_weight_only(scheme, bf16_dev(x), u8_dev(wq), f32_dev(sw), y=y, workspace=ws)
        assert ql.device_status()[0] == 0
        assert np.all(bits(ypad[M * N:]) == bits(torch.tensor([-12345.0], dtype=torch.bfloat16))[0])
        assert_y_close(bits(y), ref, f"weight-only M={M} scheme {scheme} {N}x{K} call {call}")


@pytest.mark.parametrize("M", [2, 3, 4, 8, 16, 32])
@pytest.mark.parametrize("scheme", [ql.W8A8_INT8_ROW, ql.FP8_E4M3_ROW])
@pytest.mark.parametrize("name,N,K", synthetic.LLAMA31_8B)
def test_forward_weight_only_llama(cuda, M, scheme, name, N, K):
    _run(scheme, M, N, K)


@pytest.mark.parametrize("M", [2, 4, 5, 32])
@pytest.mark.parametrize("name,N,K", synthetic.QWEN3_8B)
def test_forward_weight_only_qwen_block(cuda, M, name, N, K):
    _run(ql.FP8_E4M3_BLOCK128, M, N, K, outliers=0)


@pytest.mark.parametrize("M,N,K", [(2, 37, 256), (3, 129, 4112), (4, 5, 6144), (2, 300, 16384),
                                   (3, 150, 8192), (1, 1000, 1024), (5, 37, 272), (7, 1000, 4112),
                                   (3, 150, 8208), (1, 130, 20000), (17, 300, 2064), (32, 128, 128),
                                   (2, 64, 16400)])
@pytest.mark.parametrize("scheme", [ql.W8A8_INT8_ROW, ql.FP8_E4M3_ROW])
def test_forward_weight_only_odd_shapes(cuda, M, N, K, scheme):
    _run(scheme, M, N, K, outliers=min(3, K))


def test_forward_weight_only_limits(cuda):
    # the GEMV route's K limits, as the library reports them through the workspace size
    for M, K in ((1, 16384), (2, 16384), (3, 8192), (4, 8192)):
        assert ql.weight_only_workspace_bytes(ql.FP8_E4M3_ROW, M, 256, K) == 0
        assert ql.weight_only_workspace_bytes(ql.FP8_E4M3_ROW, M, 256, K + 16) > 0
    assert ql.weight_only_workspace_bytes(ql.FP8_E4M3_ROW, 5, 256, 256) > 0
    for M, K, status in ((33, 256, 2), (8, 256, 7)):
        x = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
        wq = torch.zeros((16, K), dtype=torch.uint8, device="cuda")
        sw = torch.ones(16, dtype=torch.float32, device="cuda")
        y = torch.empty((M, 16), dtype=torch.bfloat16, device="cuda")
        st = ql.lib().qlinear_forward_weight_only(ql.FP8_E4M3_ROW, x.data_ptr(), wq.data_ptr(), sw.data_ptr(),
                                                  M, 16, K, y.data_ptr(), None, 0,
                                                  torch.cuda.current_stream().cuda_stream)
        assert st == status  # too many tokens / no workspace
