"""GPU parity: activation and weight quantization kernels vs the oracle, bit-exact.

Quantized codes and scales are integer / bit-pattern results, so the bar is
bit equality: the same IEEE f32 division on both sides, the same rounding.
Covers the three schemes, ragged K, the register-cached and re-read paths of
the row kernel, zero / tiny / huge / negative-zero inputs, and sweeps of every
bf16 value through the int8 and E4M3 rounding with the scale pinned to 1.
"""
import numpy as np
import pytest
import torch

import fp8_linear_layers_b200 as ql
import oracle
from fp8_linear_layers_b200 import synthetic
from tests._util import bf16_dev

pytestmark = pytest.mark.gpu

SCHEMES = [ql.W8A8_INT8_ROW, ql.FP8_E4M3_ROW, ql.FP8_E4M3_BLOCK128]


def _act_case(scheme, M, K, seed=0, outliers=None):
    if outliers is None:
        outliers = synthetic.outlier_count(K)
    return synthetic.make_x(M, K, seed=seed, tag=f"qa{scheme}", outliers=outliers)


def _check_act(scheme, x_bits):
    qx, sx = ql.quantize_act(scheme, bf16_dev(x_bits))
    torch.cuda.synchronize()
    rq, rs = oracle.quantize_act(scheme, x_bits)
    g_q, g_s = qx.cpu().numpy(), sx.cpu().numpy()
    assert np.array_equal(g_s.view(np.uint32), rs.view(np.uint32)), "scales differ"
    bad = np.nonzero(g_q != rq)
    assert bad[0].size == 0, f"{bad[0].size} codes differ, first at {list(zip(*bad))[:4]}"


@pytest.mark.parametrize("scheme", SCHEMES)
@pytest.mark.parametrize("M,K", [(1, 128), (3, 256), (5, 4096), (2, 14336), (33, 12288),
                                 (1, 32768), (2, 40960), (4, 1152)])
def test_quantize_act_matches_oracle(cuda, scheme, M, K):
    _check_act(scheme, _act_case(scheme, M, K))


@pytest.mark.parametrize("scheme", [ql.W8A8_INT8_ROW, ql.FP8_E4M3_ROW])
@pytest.mark.parametrize("M,K", [(1, 16), (3, 48), (7, 4112), (2, 2064)])
def test_quantize_act_ragged_row_schemes(cuda, scheme, M, K):
    _check_act(scheme, _act_case(scheme, M, K))


def _special_rows(K):
    rows = np.zeros((6, K), np.float32)
    rows[1, 5] = -0.0
    rows[1, 7] = 3.0                       # a single nonzero
    rows[2, :] = -0.0                      # all negative zeros
    rows[3, :] = np.float32(2.0 ** -130) * np.arange(1, K + 1, dtype=np.float32) % 7  # subnormals
    rows[4, :] = np.float32(3.0e38) * np.sin(np.arange(K, dtype=np.float32))       # huge
    rows[5, ::2] = 1.0
    rows[5, 1::2] = -1.0
    b = torch.from_numpy(rows).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    return b


@pytest.mark.parametrize("scheme", SCHEMES)
def test_quantize_act_special_values(cuda, scheme):
    _check_act(scheme, _special_rows(256))


def _all_bf16_with_pin(limit, pin):
    """Every finite bf16 value with |v| <= limit, laid out in rows of K=4096 that
    each also hold +pin, so the per-token absmax (and the scale) is pinned."""
    v = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    f = (v.astype(np.uint32) << 16).view(np.float32)
    keep = np.isfinite(f) & (np.abs(f) <= limit)
    vals = v[keep]
    K = 4096
    per = K - 1
    n = (vals.size + per - 1) // per
    pad = np.zeros(n * per, np.uint16)
    pad[:vals.size] = vals
    pin_bits = (np.array([pin], np.float32).view(np.uint32) >> 16).astype(np.uint16)[0]
    return np.concatenate([pad.reshape(n, per), np.full((n, 1), pin_bits, np.uint16)], axis=1)


def test_int8_rounding_every_bf16_value(cuda):
    # absmax 127 -> s = 1 exactly, so q = clamp(rne(x)) for every bf16 x in [-127, 127]
    _check_act(ql.W8A8_INT8_ROW, _all_bf16_with_pin(127.0, 127.0))


@pytest.mark.parametrize("pin", [448.0, 1.0, 3.0e-3, 0.7, 1.37, 5.9, 123.4, 1.1e4, 7.3e-20, 2.2e25,
                                 3.3e29, 1.0e-35])
def test_e4m3_rounding_every_bf16_value(cuda, pin):
    # pin 448 -> s = 1: the hardware E4M3 conversion meets the oracle's encoder on
    # every bf16 value; other pins push every value through a non-trivial quotient
    # (scales on both sides of the kernels' reciprocal fast path, 2^-100..2^100)
    _check_act(ql.FP8_E4M3_ROW, _all_bf16_with_pin(pin, pin))


@pytest.mark.parametrize("pin", [1.0, 0.37, 9.9, 300.5, 7.3e-20, 2.2e25, 3.3e29, 1.0e-35])
def test_int8_quotient_every_bf16_value(cuda, pin):
    # s = pin / 127: every bf16 x with |x| <= pin through rne(x / s), with the
    # rounding ties and the clamp decided by the correctly rounded quotient
    _check_act(ql.W8A8_INT8_ROW, _all_bf16_with_pin(pin, pin))


@pytest.mark.parametrize("scheme", SCHEMES)
@pytest.mark.parametrize("N,K", [(128, 128), (384, 256), (1024, 4096), (14336, 4096), (4096, 14336),
                                 (4096, 12288)])
def test_quantize_weight_matches_oracle(cuda, scheme, N, K):
    w = synthetic.make_w(N, K, seed=1, tag="qw")
    wq, sw = ql.quantize_weight(scheme, bf16_dev(w))
    torch.cuda.synchronize()
    rq, rs = oracle.quantize_weight(scheme, w)
    assert np.array_equal(sw.cpu().numpy().view(np.uint32), rs.view(np.uint32))
    assert np.array_equal(wq.cpu().numpy(), rq)


@pytest.mark.parametrize("scheme", [ql.W8A8_INT8_ROW, ql.FP8_E4M3_ROW])
def test_quantize_weight_special_rows(cuda, scheme):
    w = _special_rows(512)
    wq, sw = ql.quantize_weight(scheme, bf16_dev(w))
    torch.cuda.synchronize()
    rq, rs = oracle.quantize_weight(scheme, w)
    assert np.array_equal(sw.cpu().numpy().view(np.uint32), rs.view(np.uint32))
    assert np.array_equal(wq.cpu().numpy(), rq)
