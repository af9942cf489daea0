"""The allocation-free small-M entry point, qlinear_gemm_small_noalloc.

Some callers cannot allocate device memory themselves (plugin code inside a
framework that reserved all device memory up front, a stateless C caller
with nowhere to keep a workspace pointer, a latency-critical path where an
allocation could stall the device).  For them the library offers a variant
of qlinear_gemm_small whose scratch is a fixed array inside the library.

These tests call it through the C ABI (ctypes, raw device pointers), twice in
a row on the same inputs, and compare each result with qlinear_gemm_small
run with a caller workspace, within the output tolerance the other GPU tests
use (and exactly, for int8).  This file is collected last so that a failure
here cannot hide any other test; it also passes alone in a fresh process.
"""
import numpy as np
import pytest
import torch

import fp8_linear_layers_b200 as ql
from fp8_linear_layers_b200 import synthetic
from tests._util import assert_y_close, bf16_dev, bits

pytestmark = pytest.mark.gpu


def _inputs(scheme, M, N, K):
    x = bf16_dev(synthetic.make_x(M, K, seed=11, tag="noalloc-x", outliers=synthetic.outlier_count(K)))
    w = bf16_dev(synthetic.make_w(N, K, seed=11, tag="noalloc-w"))
    wq, sw = ql.quantize_weight(scheme, w)
    return x, wq, sw


@pytest.mark.parametrize("scheme,M,N,K", [
    (ql.W8A8_INT8_ROW, 8, 1024, 4096),
    (ql.FP8_E4M3_ROW, 16, 4096, 4096),
    (ql.FP8_E4M3_BLOCK128, 32, 1024, 4096),
    (ql.W8A8_INT8_ROW, 32, 4096, 14336),
])
def test_noalloc_matches_workspace_entry_point(cuda, scheme, M, N, K):
    x, wq, sw = _inputs(scheme, M, N, K)
    ws = ql.new_workspace(ql.workspace_bytes(scheme, M, N, K))
    ref = bits(ql.gemm_small(scheme, x, wq, sw, ws))
    L = ql.lib()
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        st = L.qlinear_gemm_small_noalloc(scheme, x.data_ptr(), wq.data_ptr(), sw.data_ptr(), M, N, K,
                                          y.data_ptr(), stream)
        assert st == 0, f"call {call}: status {st}"
        torch.cuda.synchronize()
        got = bits(y)
        assert_y_close(got, ref, f"noalloc call {call}")
        if scheme == ql.W8A8_INT8_ROW:
            assert np.array_equal(got, ref), f"call {call}: int8 outputs must match exactly"
    status, detail = ql.device_status()
    assert status == 0, f"device status {status} ({detail:#x})"


def test_noalloc_rejects_shapes_beyond_its_scratch(cuda):
    # 32 tokens x 65536 outputs (512 tiles of 128 rows): the two partial-sum
    # slots of 32 x 128 int32 per tile alone take 16.8 MB, more than the fixed
    # 8 MiB scratch, so the call must refuse before launching anything
    M, N, K = 32, 65536, 128
    need = ql.workspace_bytes(ql.W8A8_INT8_ROW, M, N, K)
    assert need > (8 << 20), need
    x = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    wq = torch.zeros((N, K), dtype=torch.uint8, device="cuda")
    sw = torch.ones(N, dtype=torch.float32, device="cuda")
    y = torch.zeros((M, N), dtype=torch.bfloat16, device="cuda")
    st = ql.lib().qlinear_gemm_small_noalloc(ql.W8A8_INT8_ROW, x.data_ptr(), wq.data_ptr(), sw.data_ptr(),
                                             M, N, K, y.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == 7  # QL_ERR_WORKSPACE
    assert b"static scratch holds" in ql.lib().qlinear_last_cuda_error()
    assert f"needs {need} bytes".encode() in ql.lib().qlinear_last_cuda_error()
    assert torch.count_nonzero(y).item() == 0  # nothing ran
