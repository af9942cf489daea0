"""Pins for the oracle's weight and activation quantizers (CPU only).

Pins used here, none of which runs the oracle's own formulas:
* lossless planted inputs: every row / token / group / block is a set of codes
  times a power of two with the largest code at full range, so the scale must
  come out as that exact power of two and the codes must come back unchanged;
* the absmax invariant (the largest element of each token maps to exactly
  +-127 or +-448);
* per-element error bounds of round-to-nearest;
* shapes chosen non-square (M != N != K/128 != groups) so a transposed or
  mis-strided index cannot pass.
"""
import numpy as np
import pytest
import torch

import oracle
from fp8_linear_layers_b200 import synthetic

INT8, FP8R, FP8B = oracle.INT8_ROW, oracle.FP8_ROW, oracle.FP8_BLOCK


def _bf16(v: np.ndarray) -> np.ndarray:
    """f64 values that are exactly representable in bf16 -> bf16 bits."""
    f = v.astype(np.float32)
    assert np.array_equal(f.astype(np.float64), v), "value not exact in f32"
    b = (f.view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal((b.astype(np.uint32) << 16).view(np.float32), f), "value not exact in bf16"
    return b


def _e4m3_values() -> np.ndarray:
    return torch.arange(256, dtype=torch.int32).to(torch.uint8).view(
        torch.float8_e4m3fn).to(torch.float64).numpy()


def _planted_int8(rng, shape, pos_axis_len):
    """int codes in [-127, 127] with one +-127 per row (last axis)."""
    q = rng.integers(-127, 128, size=shape)
    idx = rng.integers(0, pos_axis_len, size=shape[:-1])
    np.put_along_axis(q, idx[..., None], rng.choice([-127, 127], size=shape[:-1])[..., None], -1)
    return q


def _planted_e4m3(rng, shape):
    """finite E4M3 codes (no NaN) with one +-448 (0x7E / 0xFE) per row."""
    codes = rng.integers(0, 256, size=shape).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] ^= 0x01  # NaN -> 0x7E / 0xFE
    idx = rng.integers(0, shape[-1], size=shape[:-1])
    np.put_along_axis(codes, idx[..., None], rng.choice([0x7E, 0xFE], size=shape[:-1])[..., None].astype(np.uint8), -1)
    return codes


# ---- activations --------------------------------------------------------------

def test_act_int8_per_token_lossless():
    rng = np.random.default_rng(1)
    M, K = 5, 48
    q = _planted_int8(rng, (M, K), K)
    e = rng.integers(-20, 6, size=M)
    x = q * np.exp2(e)[:, None]
    qx, sx = oracle.quantize_act(INT8, _bf16(x))
    assert np.array_equal(sx, np.exp2(e).astype(np.float32))
    assert np.array_equal(qx.view(np.int8).astype(np.int64), q)


def test_act_e4m3_per_token_lossless():
    rng = np.random.default_rng(2)
    M, K = 6, 40
    c = _planted_e4m3(rng, (M, K))
    e = rng.integers(-30, 10, size=M)
    x = _e4m3_values()[c] * np.exp2(e)[:, None]
    qx, sx = oracle.quantize_act(FP8R, _bf16(x))
    assert np.array_equal(sx, np.exp2(e).astype(np.float32))
    assert np.array_equal(qx, c)  # includes -0 -> 0x80


def test_act_e4m3_per_group_lossless():
    rng = np.random.default_rng(3)
    M, G = 3, 5
    K = 128 * G
    c = _planted_e4m3(rng, (M, G, 128))
    e = rng.integers(-25, 8, size=(M, G))
    x = (_e4m3_values()[c] * np.exp2(e)[:, :, None]).reshape(M, K)
    qx, sx = oracle.quantize_act(FP8B, _bf16(x))
    assert sx.shape == (M, G)
    assert np.array_equal(sx, np.exp2(e).astype(np.float32))
    assert np.array_equal(qx, c.reshape(M, K))


def test_act_zero_token_and_group():
    x = np.zeros((2, 256), np.uint16)
    x[1, 200] = _bf16(np.array([3.0]))[0]
    for scheme in (INT8, FP8R, FP8B):
        qx, sx = oracle.quantize_act(scheme, x)
        assert np.all(sx.ravel()[: (1 if scheme != FP8B else 2)] == 0)
        assert np.all(qx[0] == 0)
        assert np.count_nonzero(qx[1]) == 1


@pytest.mark.parametrize("scheme", [INT8, FP8R, FP8B])
def test_act_absmax_maps_to_full_range(scheme):
    K = 4096
    x = synthetic.make_x(16, K, seed=5, outliers=41)
    qx, sx = oracle.quantize_act(scheme, x)
    xf = oracle.bf16_bits_to_f64(x)
    top = 448.0 if scheme != INT8 else 127.0
    width = 128 if scheme == FP8B else K
    xs = np.abs(xf).reshape(16, K // width, width)
    arg = xs.argmax(-1)
    deq = (qx.view(np.int8).astype(np.float64) if scheme == INT8
           else _e4m3_values()[qx]).reshape(16, K // width, width)
    picked = np.take_along_axis(deq, arg[..., None], -1)[..., 0]
    assert np.array_equal(np.abs(picked), np.full_like(picked, top))


@pytest.mark.parametrize("scheme", [INT8, FP8R, FP8B])
def test_act_rounding_error_bound(scheme):
    """|deq(q) * s - x| within half a code step (plus one f32 rounding of x/s)."""
    K = 1024
    x = synthetic.make_x(8, K, seed=6, outliers=10)
    qx, sx = oracle.quantize_act(scheme, x)
    xf = oracle.bf16_bits_to_f64(x)
    width = 128 if scheme == FP8B else K
    s = np.repeat(sx.astype(np.float64).reshape(8, -1), width, axis=1)
    t = xf / s
    if scheme == INT8:
        q = qx.view(np.int8).astype(np.float64)
        assert np.all(np.abs(q - t) <= 0.5 + np.abs(t) * 2.0**-23)
    else:
        q = _e4m3_values()[qx]
        step_half = np.maximum(np.abs(t) * 2.0**-4, 2.0**-10)
        assert np.all(np.abs(q - t) <= step_half * (1 + 2.0**-20) + np.abs(t) * 2.0**-23)


# ---- weights --------------------------------------------------------------

def test_weight_int8_per_row_lossless():
    rng = np.random.default_rng(4)
    N, K = 7, 80
    q = _planted_int8(rng, (N, K), K)
    e = rng.integers(-12, 2, size=N)
    w = q * np.exp2(e)[:, None]
    wq, sw = oracle.quantize_weight(INT8, _bf16(w))
    assert np.array_equal(sw, np.exp2(e).astype(np.float32))
    assert np.array_equal(wq.view(np.int8).astype(np.int64), q)


def test_weight_int8_scale_is_bf16_rounded():
    """s_w is one bf16 number per row: a/127 rounded to bf16 (torch's RNE)."""
    w = synthetic.make_w(64, 512, seed=8)
    wq, sw = oracle.quantize_weight(INT8, w)
    a = np.abs(oracle.bf16_bits_to_f64(w)).max(1).astype(np.float32)
    ref = torch.from_numpy(a / np.float32(127)).to(torch.bfloat16).float().numpy()
    assert np.array_equal(sw, ref)
    assert np.all(np.abs(wq.view(np.int8)) <= 127)


def test_weight_e4m3_per_row_lossless():
    rng = np.random.default_rng(5)
    N, K = 9, 64
    c = _planted_e4m3(rng, (N, K))
    e = rng.integers(-15, 3, size=N)
    w = _e4m3_values()[c] * np.exp2(e)[:, None]
    wq, sw = oracle.quantize_weight(FP8R, _bf16(w))
    assert np.array_equal(sw, np.exp2(e).astype(np.float32))
    assert np.array_equal(wq, c)


def test_weight_e4m3_per_block_lossless():
    """N=256, K=384: 2 x 3 blocks, each with its own power-of-two scale."""
    rng = np.random.default_rng(6)
    NB, KB = 2, 3
    c = np.zeros((NB, 128, KB, 128), np.uint8)
    e = rng.integers(-20, 4, size=(NB, KB))
    for nb in range(NB):
        for kb in range(KB):
            blk = rng.integers(0, 256, size=(128, 128)).astype(np.uint8)
            blk[(blk & 0x7F) == 0x7F] ^= 1
            blk[(blk & 0x7F) == 0x7E] ^= 2  # keep 448 for the planted maximum only
            i, j = rng.integers(0, 128, 2)
            blk[i, j] = rng.choice([0x7E, 0xFE])
            c[nb, :, kb, :] = blk
    w = _e4m3_values()[c] * np.exp2(e)[:, None, :, None]
    wq, sw = oracle.quantize_weight(FP8B, _bf16(w.reshape(NB * 128, KB * 128)))
    assert sw.shape == (NB, KB)
    assert np.array_equal(sw, np.exp2(e).astype(np.float32))
    assert np.array_equal(wq, c.reshape(NB * 128, KB * 128))


def test_weight_shape_errors():
    w = np.zeros((100, 128), np.uint16)
    with pytest.raises(ValueError):
        oracle.quantize_weight(FP8B, w)
    with pytest.raises(ValueError):
        oracle.quantize_act(FP8B, np.zeros((2, 100), np.uint16))
