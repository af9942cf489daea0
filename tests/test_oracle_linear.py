"""Pins for the oracle's products and epilogues (CPU only).

* closed forms for the exact int32 accumulation (all ones, cancelling +-127,
  unit rows that select one input channel);
* exact rational sums (``fractions``) for the E4M3 accumulation;
* the hand-worked W8A8 example in ``tests/golden/w8a8_worked_example.txt``;
* lossless planted end-to-end cases whose exact answer is a rational number,
  rounded by a brute-force rational rounder;
* the dequantize-then-matmul identity against numpy's f64 matmul;
* agreement with the unquantized X . W^T within the quantization error bound.
"""
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from fp8_linear_layers_b200 import synthetic

INT8, FP8R, FP8B = oracle.INT8_ROW, oracle.FP8_ROW, oracle.FP8_BLOCK
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _e4m3_values() -> np.ndarray:
    return torch.arange(256, dtype=torch.int32).to(torch.uint8).view(
        torch.float8_e4m3fn).to(torch.float64).numpy()


def _bf16(v: np.ndarray) -> np.ndarray:
    f = v.astype(np.float32)
    assert np.array_equal(f.astype(np.float64), v)
    b = (f.view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal((b.astype(np.uint32) << 16).view(np.float32), f)
    return b


def _round_fraction(v: Fraction, sig_bits: int, min_exp: int) -> Fraction:
    """Round an exact rational to ``sig_bits`` significant bits, half to even,
    with spacing never below 2^min_exp (subnormals)."""
    if v == 0:
        return Fraction(0)
    a = abs(v)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    ulp_exp = max(e - (sig_bits - 1), min_exp)
    ulp = Fraction(2) ** ulp_exp
    q, r = divmod(a, ulp)
    if r * 2 > ulp or (r * 2 == ulp and q % 2 == 1):
        q += 1
    out = q * ulp
    return out if v > 0 else -out


def _bf16_of_fraction(v: Fraction) -> float:
    return float(_round_fraction(v, 8, -133))


def _f32_of_fraction(v: Fraction) -> Fraction:
    return _round_fraction(v, 24, -149)


def _y_f64(y_bits: np.ndarray) -> np.ndarray:
    return oracle.bf16_bits_to_f64(y_bits)


# ---- exact accumulation -------------------------------------------------------

def test_int8_accumulation_closed_forms():
    K = 4096
    ones = np.ones((1, K), np.int8).view(np.uint8)
    alt = np.tile(np.array([127, -127], np.int8), K // 2)[None, :].view(np.uint8)
    s1 = np.ones(1, np.float32)
    _, acc, _ = oracle.linear(INT8, ones, s1, ones, s1, want_acc=True)
    assert acc[0, 0] == K
    _, acc, _ = oracle.linear(INT8, alt, s1, alt, s1, want_acc=True)
    assert acc[0, 0] == K * 127 * 127  # 66,064,384: large, exact in int32
    _, acc, _ = oracle.linear(INT8, alt, s1, ones, s1, want_acc=True)
    assert acc[0, 0] == 0


def test_int8_unit_rows_select_channels():
    """W rows are unit vectors e_{j_n}: acc[m, n] must be q_x[m, j_n]."""
    rng = np.random.default_rng(3)
    M, N, K = 3, 5, 64
    qx = rng.integers(-127, 128, (M, K)).astype(np.int8)
    j = rng.permutation(K)[:N]
    wq = np.zeros((N, K), np.int8)
    wq[np.arange(N), j] = 1
    _, acc, _ = oracle.linear(INT8, qx.view(np.uint8), np.ones(M, np.float32),
                              wq.view(np.uint8), np.ones(N, np.float32), want_acc=True)
    assert np.array_equal(acc, qx[:, j].astype(np.int32))


def test_e4m3_accumulation_exact_vs_fractions():
    rng = np.random.default_rng(4)
    M, N, K = 2, 3, 96
    vals = _e4m3_values()
    qx = rng.integers(0, 256, (M, K)).astype(np.uint8)
    wq = rng.integers(0, 256, (N, K)).astype(np.uint8)
    for a in (qx, wq):
        a[(a & 0x7F) == 0x7F] ^= 1
    _, _, acc = oracle.linear(FP8R, qx, np.ones(M, np.float32), wq, np.ones(N, np.float32),
                              want_acc=True)
    for m in range(M):
        for n in range(N):
            exact = sum(Fraction(vals[qx[m, k]]) * Fraction(vals[wq[n, k]]) for k in range(K))
            assert Fraction(acc[m, n]) == exact


# ---- hand-worked example --------------------------------------------------------

def _read_worked(path):
    d = {}
    with open(path) as f:
        for line in f:
            if not line.strip() or line.startswith("#"):
                continue
            k, *v = line.split()
            d[k] = v
    return d


def test_w8a8_worked_example_golden():
    d = _read_worked(os.path.join(GOLDEN, "w8a8_worked_example.txt"))
    x = np.array([[float(v) for v in d["x"]]]) * 2.0 ** int(d["x_exp"][0])
    w = np.array([[float(v) for v in d[f"w{i}"]] for i in range(3)]) * 2.0 ** int(d["w_exp"][0])
    wq, sw = oracle.quantize_weight(INT8, _bf16(w))
    qx, sx = oracle.quantize_act(INT8, _bf16(x))
    y, acc, _ = oracle.linear(INT8, qx, sx, wq, sw, want_acc=True)
    assert acc[0].tolist() == [int(v) for v in d["acc"]]
    assert _y_f64(y)[0].tolist() == [float(v) for v in d["y"]]


# ---- lossless planted end-to-end cases ----------------------------------------------

def _planted_case(scheme, rng, M, N, K):
    """X and W built as codes x powers of two (full-range code present in each
    scale unit), so that quantization returns those codes and scales exactly."""
    vals = _e4m3_values()
    if scheme == INT8:
        cx = rng.integers(-127, 128, (M, K))
        cx[np.arange(M), rng.integers(0, K, M)] = 127
        cw = rng.integers(-127, 128, (N, K))
        cw[np.arange(N), rng.integers(0, K, N)] = -127
        ex = rng.integers(-8, 4, M)
        ew = rng.integers(-10, -2, N)
        return (cx * np.exp2(ex)[:, None], cw * np.exp2(ew)[:, None], cx, cw, ex, ew)
    cx = rng.integers(0, 256, (M, K)).astype(np.uint8)
    cw = rng.integers(0, 256, (N, K)).astype(np.uint8)
    for a in (cx, cw):
        a[(a & 0x7F) == 0x7F] ^= 1
    if scheme == FP8R:
        cx[np.arange(M), rng.integers(0, K, M)] = 0x7E
        cw[np.arange(N), rng.integers(0, K, N)] = 0xFE
        ex = rng.integers(-12, 0, M)
        ew = rng.integers(-14, -6, N)
        return (vals[cx] * np.exp2(ex)[:, None], vals[cw] * np.exp2(ew)[:, None], cx, cw, ex, ew)
    G, NB = K // 128, N // 128
    for m in range(M):
        for g in range(G):
            cx[m, g * 128 + rng.integers(0, 128)] = 0x7E
    for nb in range(NB):
        for g in range(G):
            blk = cw[nb * 128:(nb + 1) * 128, g * 128:(g + 1) * 128]
            blk[(blk & 0x7F) == 0x7E] ^= 2
            blk[rng.integers(0, 128), rng.integers(0, 128)] = 0xFE
    ex = rng.integers(-12, 0, (M, G))
    ew = rng.integers(-14, -6, (NB, G))
    xs = vals[cx] * np.repeat(np.exp2(ex), 128, axis=1)
    ws = vals[cw] * np.kron(np.exp2(ew), np.ones((128, 128)))
    return xs, ws, cx, cw, ex, ew


@pytest.mark.parametrize("scheme,M,N,K", [(INT8, 3, 5, 48), (FP8R, 4, 3, 64), (FP8B, 3, 256, 384)])
def test_planted_end_to_end_exact(scheme, M, N, K):
    rng = np.random.default_rng(10 + scheme)
    x, w, cx, cw, ex, ew = _planted_case(scheme, rng, M, N, K)
    wq, sw = oracle.quantize_weight(scheme, _bf16(w))
    y = oracle.forward(scheme, _bf16(x), wq, sw)
    yv = _y_f64(y)
    vals = _e4m3_values()
    cols = range(N) if N <= 8 else list(range(0, N, 37)) + [N - 1]
    for m in range(M):
        for n in cols:
            if scheme == INT8:
                acc = sum(int(cx[m, k]) * int(cw[n, k]) for k in range(K))
                ref = _bf16_of_fraction(Fraction(acc) * Fraction(2) ** int(ex[m] + ew[n]))
            elif scheme == FP8R:
                acc = sum(Fraction(vals[cx[m, k]]) * Fraction(vals[cw[n, k]]) for k in range(K))
                # the method rounds the f32 accumulator before the scale epilogue
                ref = _bf16_of_fraction(_f32_of_fraction(acc) * Fraction(2) ** int(ex[m] + ew[n]))
            else:
                tot = Fraction(0)
                for g in range(K // 128):
                    p = sum(Fraction(vals[cx[m, k]]) * Fraction(vals[cw[n, k]])
                            for k in range(g * 128, g * 128 + 128))
                    tot += p * Fraction(2) ** int(ex[m, g] + ew[n // 128, g])
                ref = _bf16_of_fraction(tot)
            assert yv[m, n] == ref, (m, n)


# ---- dequantize-then-matmul identity ---------------------------------------------------

def _dequant(scheme, q, s, rows, K, weight):
    vals = _e4m3_values()
    d = q.view(np.int8).astype(np.float64) if scheme == INT8 else vals[q]
    if scheme == FP8B:
        if weight:
            return d * np.kron(s.astype(np.float64), np.ones((128, 128)))
        return d * np.repeat(s.astype(np.float64), 128, axis=1)
    return d * s.astype(np.float64)[:, None]


@pytest.mark.parametrize("scheme", [INT8, FP8R, FP8B])
def test_dequantize_then_matmul_identity(scheme):
    M, N, K = 4, 256, 512
    x = synthetic.make_x(M, K, seed=21, outliers=5)
    w = synthetic.make_w(N, K, seed=22)
    wq, sw = oracle.quantize_weight(scheme, w)
    qx, sx = oracle.quantize_act(scheme, x)
    y, _, acc = oracle.linear(scheme, qx, sx, wq, sw, want_acc=True)
    ref = _dequant(scheme, qx, sx, M, K, False) @ _dequant(scheme, wq, sw, N, K, True).T
    if scheme == FP8B:
        pre = acc  # exact f64 value before the final rounding
    else:
        pre = acc * sx.astype(np.float64)[:, None] * sw.astype(np.float64)[None, :]
    assert np.allclose(pre, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    # the bf16 output is within one bf16 step (plus the f32 epilogue roundings) of it
    yv = _y_f64(y)
    assert np.all(np.abs(yv - ref) <= np.abs(ref) * 2.0**-8 * (1 + 2.0**-20) + 1e-30)


@pytest.mark.parametrize("scheme", [INT8, FP8R, FP8B])
def test_agrees_with_unquantized_within_quantization_bound(scheme):
    """The pages' accuracy reference is the unrounded product ("equivalent"
    numerics never round the input).  Per output, the quantized result must be
    within sum_k |x| dw + |w| dx + dx dw of X.W^T, where dx, dw are the largest
    errors round-to-nearest can make with the scales used."""
    M, N, K = 3, 128, 1024
    x = synthetic.make_x(M, K, seed=31, outliers=10)
    w = synthetic.make_w(N, K, seed=32)
    wq, sw = oracle.quantize_weight(scheme, w)
    y = oracle.forward(scheme, x, wq, sw)
    qx, sx = oracle.quantize_act(scheme, x)
    xf, wf = oracle.bf16_bits_to_f64(x), oracle.bf16_bits_to_f64(w)
    ref = xf @ wf.T
    if scheme == INT8:
        dx = np.broadcast_to(sx.astype(np.float64)[:, None] / 2, (M, K))
        dw = np.broadcast_to(sw.astype(np.float64)[:, None] / 2, (N, K))
    else:
        sxe = (np.repeat(sx.astype(np.float64), 128, axis=1) if scheme == FP8B
               else np.broadcast_to(sx.astype(np.float64)[:, None], (M, K)))
        swe = (np.kron(sw.astype(np.float64), np.ones((128, 128))) if scheme == FP8B
               else np.broadcast_to(sw.astype(np.float64)[:, None], (N, K)))
        dx = np.maximum(np.abs(xf) * 2.0**-4, sxe * 2.0**-10)
        dw = np.maximum(np.abs(wf) * 2.0**-4, swe * 2.0**-10)
    dx, dw = dx * (1 + 1e-6), dw * (1 + 1e-6)
    bound = np.abs(xf) @ dw.T + dx @ np.abs(wf).T + dx @ dw.T
    yv = _y_f64(y)
    assert np.all(np.abs(yv - ref) <= bound + np.abs(yv) * 2.0**-8 + 1e-6)
    # and the bound is not vacuous: the error is much smaller than |y| overall
    assert np.median(np.abs(yv - ref)) < 0.1 * np.median(np.abs(ref))


# ---- consistency of the sampled and sliced forms (infrastructure) ----------------------

@pytest.mark.parametrize("scheme", [INT8, FP8R, FP8B])
def test_sampled_and_rows_match_full(scheme):
    M, N, K = 3, 256, 256
    x = synthetic.make_x(M, K, seed=41)
    w = synthetic.make_w(N, K, seed=42)
    wq, sw = oracle.quantize_weight(scheme, w)
    qx, sx = oracle.quantize_act(scheme, x)
    y = oracle.linear(scheme, qx, sx, wq, sw)
    rng = np.random.default_rng(0)
    pm, pn = rng.integers(0, M, 50), rng.integers(0, N, 50)
    ys = oracle.linear_sampled(scheme, qx, sx, wq, sw, pm, pn)
    assert np.array_equal(ys, y[pm, pn])
    assert np.array_equal(oracle.linear_rows(scheme, qx, sx, wq, sw, 128, 256), y[:, 128:256])
