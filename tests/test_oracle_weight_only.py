"""Pins for the oracle's weight-only ("equivalent" numerics) product (CPU only).

The pages' loader option that never rounds the input ("Llama 3.1 8B Instruct
W8A8" and "Qwen3 8B FP8", "Against bf16") and the W8A16 contrast in the W8A8
model page's "Context": X stays bf16, only W is quantized.

* exact rationals (``fractions``) rounded by a brute-force rational rounder,
  for every scheme, with E4M3 values from torch's ``float8_e4m3fn``;
* unit activations that select one dequantized weight (row and column
  indexing, which block scale applies);
* numpy's f64 matmul of X and the dequantized weights (a library routine);
* the W8A8 result on inputs that per-token quantization reproduces exactly;
* agreement with the unquantized X . W^T within the weight-rounding bound;
* sign symmetry and argument checks;
* the hand-worked example in ``tests/golden/weight_only_worked_example.txt``
  (two ties rounded to even).
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from fp8_linear_layers_b200 import synthetic
from test_oracle_linear import _bf16, _bf16_of_fraction, _e4m3_values

INT8, FP8R, FP8B = oracle.INT8_ROW, oracle.FP8_ROW, oracle.FP8_BLOCK


def _codes_f64(scheme, wq):
    if scheme == INT8:
        return wq.view(np.int8).astype(np.float64)
    return _e4m3_values()[wq]


def _dequant_f64(scheme, wq, sw):
    """Dequantized weights in f64 (every element exact: code x scale)."""
    c = _codes_f64(scheme, wq)
    N, K = wq.shape
    if scheme == FP8B:
        s = np.repeat(np.repeat(sw.astype(np.float64), 128, axis=0), 128, axis=1)
        return c * s
    return c * sw.astype(np.float64)[:, None]


def _case(scheme, M, N, K, seed, outliers=0):
    w = synthetic.make_w(N, K, seed=seed, tag=f"wo.w.{scheme}")
    x = synthetic.make_x(M, K, seed=seed, tag=f"wo.x.{scheme}", outliers=outliers)
    wq, sw = oracle.quantize_weight(scheme, w)
    return x, w, wq, sw


@pytest.mark.parametrize("scheme", [INT8, FP8R, FP8B])
def test_weight_only_exact_fractions(scheme):
    M, N, K = 2, 128, 256
    x, _, wq, sw = _case(scheme, M, N, K, seed=11, outliers=3)
    y = oracle.linear_weight_only(scheme, x, wq, sw)
    xv = oracle.bf16_bits_to_f64(x)
    c = _codes_f64(scheme, wq)
    rng = np.random.default_rng(5)
    for n in rng.choice(N, 12, replace=False):
        for m in range(M):
            total = Fraction(0)
            for k in range(K):
                s = sw[(n // 128), k // 128] if scheme == FP8B else sw[n]
                total += Fraction(xv[m, k]) * Fraction(c[n, k]) * Fraction(float(s))
            assert oracle.bf16_bits_to_f64(y[m, n:n + 1])[0] == _bf16_of_fraction(total), (m, n)


@pytest.mark.parametrize("scheme", [INT8, FP8R, FP8B])
def test_weight_only_unit_inputs_select_one_weight(scheme):
    """x = e_j: y[n] must be bf16(code[n, j] * its scale) for every n."""
    N, K = 256, 384
    _, _, wq, sw = _case(scheme, 1, N, K, seed=12)
    deq = _dequant_f64(scheme, wq, sw)
    for j in (0, 1, 127, 128, 300, K - 1):
        x = np.zeros((1, K), np.uint16)
        x[0, j] = 0x3F80  # 1.0
        y = oracle.linear_weight_only(scheme, x, wq, sw)
        want = np.array([_bf16_of_fraction(Fraction(v)) for v in deq[:, j]])
        assert np.array_equal(oracle.bf16_bits_to_f64(y[0]), want), j


@pytest.mark.parametrize("scheme", [INT8, FP8R, FP8B])
def test_weight_only_matches_numpy_f64_matmul(scheme):
    M, N, K = 3, 256, 512
    x, _, wq, sw = _case(scheme, M, N, K, seed=13, outliers=5)
    y, acc = oracle.linear_weight_only(scheme, x, wq, sw, want_acc=True)
    ref = oracle.bf16_bits_to_f64(x) @ _dequant_f64(scheme, wq, sw).T
    # two f64 sums of the same exact products in different orders
    bound = K * 2.0 ** -52 * (np.abs(oracle.bf16_bits_to_f64(x)) @ np.abs(_dequant_f64(scheme, wq, sw)).T)
    assert np.all(np.abs(acc - ref) <= bound)
    assert np.array_equal(y, oracle.f64_to_bf16_n(acc).reshape(y.shape))


def test_weight_only_row_range_matches_full():
    x, _, wq, sw = _case(FP8B, 2, 384, 256, seed=14)
    full = oracle.linear_weight_only(FP8B, x, wq, sw)
    part = oracle.linear_weight_only(FP8B, x, wq, sw, n0=128, n1=384)
    assert np.array_equal(full[:, 128:], part)


@pytest.mark.parametrize("scheme", [INT8, FP8R])
def test_weight_only_equals_w8a8_on_losslessly_quantized_inputs(scheme):
    """Per-token quantization of x = codes * 2^-4 (a full-range code present) is
    exact with scale 2^-4, so both products are the same exact sum times the
    scales; the only difference is where they round."""
    rng = np.random.default_rng(15)
    M, N, K = 2, 128, 256
    qmax = 127 if scheme == INT8 else 448
    # small codes keep the exact sums short; one full-range code per token
    codes = rng.integers(-3, 4, (M, K)).astype(np.float64)
    if scheme == FP8R:
        codes *= 0.5
    codes[:, 7] = qmax
    x = _bf16(codes * 2.0 ** -4)
    w = synthetic.make_w(N, K, seed=15, tag=f"wo.lossless.{scheme}")
    wq, sw = oracle.quantize_weight(scheme, w)
    if scheme == FP8R:  # make the row scales bf16 values too, so every product is short
        sw = oracle.bf16_bits_to_f64(oracle.f32_to_bf16_n(sw)).astype(np.float32)
    qx, sx = oracle.quantize_act(scheme, x)
    assert np.all(sx == np.float32(2.0 ** -4))
    y8, _, acc = oracle.linear(scheme, qx, sx, wq, sw, want_acc=True)
    ywo = oracle.linear_weight_only(scheme, x, wq, sw)
    # Both are the correctly rounded bf16 of the same exact value acc 2^-4 s_w
    # wherever that value is an f32 (the W8A8 epilogue's f32 multiplies are then
    # exact); those outputs are compared.
    exact = np.array([[Fraction(acc[m, n]) * Fraction(2) ** -4 * Fraction(float(sw[n]))
                       for n in range(N)] for m in range(M)], dtype=object)
    f32_exact = np.vectorize(lambda v: float(np.float32(float(v))) == v)(exact)
    assert f32_exact.sum() >= 30, f32_exact.sum()
    assert np.array_equal(y8[f32_exact], ywo[f32_exact])


@pytest.mark.parametrize("scheme", [INT8, FP8R, FP8B])
def test_weight_only_close_to_unquantized(scheme):
    """|y - X W^T| <= sum_k |x| |w - w_hat| + half a bf16 ulp of y (+ the f64 sum)."""
    M, N, K = 2, 256, 1024
    x, w, wq, sw = _case(scheme, M, N, K, seed=16, outliers=10)
    y = oracle.bf16_bits_to_f64(oracle.linear_weight_only(scheme, x, wq, sw))
    xv = oracle.bf16_bits_to_f64(x)
    wv = oracle.bf16_bits_to_f64(w)
    deq = _dequant_f64(scheme, wq, sw)
    err_bound = np.abs(xv) @ np.abs(wv - deq).T
    exact = xv @ wv.T
    assert np.all(np.abs(y - exact) <= err_bound + 2.0 ** -8 * np.abs(y) + 1e-30)
    # and the weight rounding is small: the bound itself is a few % of |X| |W|
    assert np.median(err_bound / (np.abs(xv) @ np.abs(wv).T)) < 0.05


@pytest.mark.parametrize("scheme", [INT8, FP8R, FP8B])
def test_weight_only_sign_symmetry(scheme):
    x, _, wq, sw = _case(scheme, 2, 128, 256, seed=17)
    y = oracle.linear_weight_only(scheme, x, wq, sw)
    yn = oracle.linear_weight_only(scheme, x ^ np.uint16(0x8000), wq, sw)
    assert np.array_equal(oracle.bf16_bits_to_f64(yn), -oracle.bf16_bits_to_f64(y))


def test_weight_only_rejects_bad_shapes():
    x = np.zeros((1, 200), np.uint16)
    with pytest.raises(ValueError):
        oracle.linear_weight_only(FP8B, x, np.zeros((128, 200), np.uint8), np.zeros((1, 1), np.float32))
    x = np.zeros((1, 128), np.uint16)
    with pytest.raises(ValueError):
        oracle.linear_weight_only(INT8, x, np.zeros((4, 128), np.uint8), np.ones(4, np.float32),
                                  n0=2, n1=5)


def test_weight_only_worked_example_golden():
    import os
    from test_oracle_linear import GOLDEN, _read_worked
    d = _read_worked(os.path.join(GOLDEN, "weight_only_worked_example.txt"))
    x = _bf16(np.array([[float(v) for v in d["x"]]]))
    w = np.array([[float(v) for v in d[f"w{i}"]] for i in range(3)]) * 2.0 ** int(d["w_exp"][0])
    wq, sw = oracle.quantize_weight(INT8, _bf16(w))
    assert np.all(sw == np.float32(2.0 ** int(d["w_exp"][0])))
    y, acc = oracle.linear_weight_only(INT8, x, wq, sw, want_acc=True)
    scale = 2.0 ** int(d["w_exp"][0])
    assert (acc[0] / scale).tolist() == [float(v) for v in d["sum"]]
    assert oracle.bf16_bits_to_f64(y)[0].tolist() == [float(v) for v in d["y"]]
