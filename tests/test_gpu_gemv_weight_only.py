"""GPU parity: the M = 1 weight-only ("equivalent" numerics) GEMV vs the oracle.

The activations stay bf16 and only the weights are quantized (the pages'
loader option that never rounds the input; W8A16 / FP8 weight-only).  Every
output of one Llama-3.1-8B layer's seven projections (int8 and FP8 per-row
weights) and one Qwen3-8B layer's (FP8 block weights) is compared with the
oracle's exact value rounded once: within 2^-7 |y| + 1e-3, and at least 95%
of them within one bf16 ulp (the kernel's f32 sums of exact products).  Plus
odd and ragged shapes, zero and extreme-range tokens, exact scale invariance
under powers of two, and a canary check that nothing is written past y.
"""
import numpy as np
import pytest
import torch

import fp8_linear_layers_b200 as ql
import oracle
from fp8_linear_layers_b200 import synthetic
from tests._util import assert_y_close, bf16_dev, bits, f32_dev, u8_dev

pytestmark = pytest.mark.gpu

CANARY = -12345.0


def _gpu(scheme, x, wq, sw):
    N, K = wq.shape
    ypad = torch.full((N + 64,), CANARY, dtype=torch.bfloat16, device="cuda")
    y = ypad[:N].view(1, N)
    ql.gemv_weight_only(scheme, bf16_dev(x), u8_dev(wq), f32_dev(sw), y=y)
    assert ql.device_status()[0] == 0
    tail = bits(ypad[N:])
    assert np.all(tail == bits(torch.tensor([CANARY], dtype=torch.bfloat16))[0]), \
        "weight-only gemv wrote past the end of y"
    return bits(y)


def _ulps(g_bits, r_bits):
    """Distance in bf16 steps between two arrays of finite bf16 values."""
    def ordered(b):
        b = b.astype(np.int64)
        return np.where(b & 0x8000, -(b & 0x7FFF), b)
    return np.abs(ordered(g_bits) - ordered(r_bits))


def _run(scheme, N, K, seed=0, outliers=None):
    if outliers is None:
        outliers = synthetic.outlier_count(K)
    x = synthetic.make_x(1, K, seed=seed, tag="gemv-wo-x", outliers=outliers)
    w = synthetic.make_w(N, K, seed=seed, tag="gemv-wo-w")
    wq, sw = oracle.quantize_weight(scheme, w)
    gy = _gpu(scheme, x, wq, sw)
    ry = oracle.linear_weight_only(scheme, x, wq, sw)
    assert_y_close(gy, ry, f"weight-only gemv scheme {scheme} {N}x{K}")
    assert np.mean(_ulps(gy, ry) <= 1) >= 0.95
    return x, wq, sw, gy


@pytest.mark.parametrize("scheme", [ql.W8A8_INT8_ROW, ql.FP8_E4M3_ROW])
@pytest.mark.parametrize("name,N,K", synthetic.LLAMA31_8B)
def test_gemv_weight_only_llama_layer_full(cuda, scheme, name, N, K):
    _run(scheme, N, K)


@pytest.mark.parametrize("name,N,K", synthetic.QWEN3_8B)
def test_gemv_weight_only_qwen_layer_block_full(cuda, name, N, K):
    _run(ql.FP8_E4M3_BLOCK128, N, K, outliers=0)


@pytest.mark.parametrize("scheme", [ql.W8A8_INT8_ROW, ql.FP8_E4M3_ROW])
@pytest.mark.parametrize("N,K", [(1, 16), (3, 48), (37, 256), (129, 4112), (1000, 1024),
                                 (300, 8208), (150, 16384), (5, 6144), (149, 12288)])
def test_gemv_weight_only_odd_shapes(cuda, scheme, N, K):
    _run(scheme, N, K, outliers=min(3, K))


@pytest.mark.parametrize("N,K", [(128, 128), (256, 384), (128, 16384), (384, 6144)])
def test_gemv_weight_only_block_odd_shapes(cuda, N, K):
    _run(ql.FP8_E4M3_BLOCK128, N, K, outliers=2)


@pytest.mark.parametrize("scheme", [ql.W8A8_INT8_ROW, ql.FP8_E4M3_ROW, ql.FP8_E4M3_BLOCK128])
def test_gemv_weight_only_power_of_two_scaling_is_exact(cuda, scheme):
    """x 2^j stages the same f16 values as x (the staging exponent moves by -j),
    so every output is y(x) 2^j bit for bit while nothing under- or overflows."""
    N, K = 1024, 4096
    x, wq, sw, gy = _run(scheme, N, K, seed=4)
    gy64 = oracle.bf16_bits_to_f64(gy)
    for j in (-60, -7, 9, 60):
        xs = oracle.f64_to_bf16_n(oracle.bf16_bits_to_f64(x) * 2.0 ** j).reshape(x.shape)
        assert np.array_equal(oracle.bf16_bits_to_f64(xs), oracle.bf16_bits_to_f64(x) * 2.0 ** j)
        gys = oracle.bf16_bits_to_f64(_gpu(scheme, xs, wq, sw))
        assert np.array_equal(gys, gy64 * 2.0 ** j), j


@pytest.mark.parametrize("scheme", [ql.W8A8_INT8_ROW, ql.FP8_E4M3_ROW, ql.FP8_E4M3_BLOCK128])
def test_gemv_weight_only_wide_dynamic_range(cuda, scheme):
    """One element 2^20 above the rest: the small ones still count (they are
    within the 2^31 the staging carries exactly)."""
    N, K = 512, 2048
    x = synthetic.make_x(1, K, seed=6, tag="gemv-wo-range", outliers=0)
    xv = oracle.bf16_bits_to_f64(x)
    xv[0, 5] = 2.0 ** 20
    x = oracle.f64_to_bf16_n(xv).reshape(x.shape)
    w = synthetic.make_w(N, K, seed=6, tag="gemv-wo-range-w")
    wq, sw = oracle.quantize_weight(scheme, w)
    gy = _gpu(scheme, x, wq, sw)
    ry = oracle.linear_weight_only(scheme, x, wq, sw)
    assert_y_close(gy, ry, "wide range")


def test_gemv_weight_only_zero_token(cuda):
    K, N = 4096, 256
    w = synthetic.make_w(N, K, seed=3)
    for scheme in (0, 1, 2):
        wq, sw = oracle.quantize_weight(scheme, w)
        y = ql.gemv_weight_only(scheme, torch.zeros((1, K), dtype=torch.bfloat16, device="cuda"),
                                u8_dev(wq), f32_dev(sw))
        assert torch.count_nonzero(y.float()) == 0


def test_gemv_weight_only_rejects_k_beyond_limit(cuda):
    K = 16400
    x = torch.zeros((1, K), dtype=torch.bfloat16, device="cuda")
    wq = torch.zeros((16, K), dtype=torch.uint8, device="cuda")
    sw = torch.ones(16, dtype=torch.float32, device="cuda")
    with pytest.raises(ql.QLinearError) as e:
        ql.gemv_weight_only(ql.W8A8_INT8_ROW, x, wq, sw)
    assert e.value.status == 2
