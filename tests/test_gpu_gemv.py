"""GPU parity: the M = 1 GEMV (activation quantization fused) vs the oracle.

Full-size: every output of one Llama-3.1-8B layer's seven projections (W8A8
and FP8 per-row) and one Qwen3-8B layer's (FP8 block), with the fused
quantization's codes, scales and (int8) int32 accumulators captured through
the debug hook and compared bit-exactly.  bf16 outputs: bit-exact for int8
(same int32 sum, same two f32 multiplies), 2^-7 |y| + 1e-3 for E4M3.  Plus
odd and ragged shapes and a canary check that nothing is written past y.
"""
import numpy as np
import pytest
import torch

import fp8_linear_layers_b200 as ql
import oracle
from fp8_linear_layers_b200 import synthetic
from tests._util import assert_y_close, bf16_dev, bits, f32_dev, u8_dev

pytestmark = pytest.mark.gpu


def _run(scheme, N, K, seed=0, outliers=None, canary=True):
    if outliers is None:
        outliers = synthetic.outlier_count(K)
    x = synthetic.make_x(1, K, seed=seed, tag="gemv-x", outliers=outliers)
    w = synthetic.make_w(N, K, seed=seed, tag="gemv-w")
    wq, sw = oracle.quantize_weight(scheme, w)
    dev = "cuda"
    ypad = torch.full((N + 64,), -12345.0, dtype=torch.bfloat16, device=dev)
    y = ypad[:N].view(1, N)
    dbg = ql.Debug(qx=torch.empty((1, K), dtype=torch.uint8, device=dev),
                   sx=torch.empty(ql.act_scale_shape(scheme, 1, K), dtype=torch.float32, device=dev),
                   acc_i32=torch.empty((1, N), dtype=torch.int32, device=dev),
                   acc_f32=torch.empty((1, N), dtype=torch.float32, device=dev))
    ql.gemv(scheme, bf16_dev(x), u8_dev(wq), f32_dev(sw), y=y, debug=dbg)
    st, _ = ql.device_status()
    assert st == 0
    rqx, rsx = oracle.quantize_act(scheme, x)
    ry, racc_i, racc_d = oracle.linear(scheme, rqx, rsx, wq, sw, want_acc=True)
    assert np.array_equal(dbg.qx.cpu().numpy(), rqx)
    assert np.array_equal(dbg.sx.cpu().numpy().view(np.uint32), rsx.view(np.uint32))
    gy = bits(y)
    if scheme == ql.W8A8_INT8_ROW:
        assert np.array_equal(dbg.acc_i32.cpu().numpy(), racc_i)
        assert np.array_equal(gy, ry), "int8 outputs must be bit-exact"
    else:
        assert_y_close(gy, ry, f"gemv scheme {scheme} {N}x{K}")
        if scheme == ql.FP8_E4M3_ROW:
            acc = dbg.acc_f32.cpu().numpy().astype(np.float64)
            assert np.all(np.abs(acc - racc_d) <= 1e-5 * np.abs(racc_d).max() + 1e-6)
    if canary:
        tail = bits(ypad[N:])
        assert np.all(tail == bits(torch.tensor([-12345.0], dtype=torch.bfloat16))[0]), \
            "gemv wrote past the end of y"


@pytest.mark.parametrize("scheme", [ql.W8A8_INT8_ROW, ql.FP8_E4M3_ROW])
@pytest.mark.parametrize("name,N,K", synthetic.LLAMA31_8B)
def test_gemv_llama_layer_full(cuda, scheme, name, N, K):
    _run(scheme, N, K)


@pytest.mark.parametrize("name,N,K", synthetic.QWEN3_8B)
def test_gemv_qwen_layer_block_full(cuda, name, N, K):
    _run(ql.FP8_E4M3_BLOCK128, N, K, outliers=0)


@pytest.mark.parametrize("scheme", [ql.W8A8_INT8_ROW, ql.FP8_E4M3_ROW])
@pytest.mark.parametrize("N,K", [(1, 16), (3, 48), (37, 256), (129, 4112), (1000, 1024),
                                 (300, 8208), (150, 32768), (5, 6144), (149, 12288)])
def test_gemv_odd_shapes(cuda, scheme, N, K):
    _run(scheme, N, K, outliers=min(3, K))


@pytest.mark.parametrize("N,K", [(128, 128), (256, 384), (128, 32768), (384, 6144)])
def test_gemv_block_odd_shapes(cuda, N, K):
    _run(ql.FP8_E4M3_BLOCK128, N, K, outliers=2)


def test_gemv_rejects_k_beyond_limit(cuda):
    K = 32784
    x = torch.zeros((1, K), dtype=torch.bfloat16, device="cuda")
    wq = torch.zeros((16, K), dtype=torch.uint8, device="cuda")
    sw = torch.ones(16, dtype=torch.float32, device="cuda")
    with pytest.raises(ql.QLinearError) as e:
        ql.gemv(ql.W8A8_INT8_ROW, x, wq, sw)
    assert e.value.status == 2


def test_gemv_zero_token(cuda):
    K, N = 4096, 256
    w = synthetic.make_w(N, K, seed=3)
    for scheme in (0, 1, 2):
        wq, sw = oracle.quantize_weight(scheme, w)
        y = ql.gemv(scheme, torch.zeros((1, K), dtype=torch.bfloat16, device="cuda"), u8_dev(wq),
                    f32_dev(sw))
        assert torch.count_nonzero(y.float()) == 0


@pytest.mark.parametrize("scheme", [ql.W8A8_INT8_ROW, ql.FP8_E4M3_ROW, ql.FP8_E4M3_BLOCK128])
def test_gemv_side_by_side_weights_equal_separate(cuda, scheme):
    """Every output row depends only on its own weight row and scale, so the
    q|k|v weights stored side by side along N give, in one launch, exactly
    the bits of the three separate products on the same token."""
    K = 4096
    parts = [(4096, "q"), (1024, "k"), (1024, "v")]
    x = bf16_dev(synthetic.make_x(1, K, seed=5, tag="fused-x", outliers=synthetic.outlier_count(K)))
    wqs, sws, ys = [], [], []
    for N, tag in parts:
        w = synthetic.make_w_device(N, K, seed=5, tag="fused-" + tag)
        wq, sw = ql.quantize_weight(scheme, w)
        wqs.append(wq)
        sws.append(sw)
        ys.append(ql.gemv(scheme, x, wq, sw))
    y_fused = ql.gemv(scheme, x, torch.cat(wqs, 0).contiguous(), torch.cat(sws, 0).contiguous())
    assert ql.device_status()[0] == 0
    assert torch.equal(y_fused.view(torch.int16), torch.cat(ys, 1).view(torch.int16))
