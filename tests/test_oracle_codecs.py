"""Pins for the oracle's number codecs (CPU only).

Each check compares the oracle with something that does not share its code:
torch's own bf16 / float8_e4m3fn conversions (library routines), numpy's
round-half-even ``rint``, exact rational brute force (``fractions``), and the
hand-worked fixtures under ``tests/golden/``.
"""
import os
from fractions import Fraction

import numpy as np
import torch

import oracle
from fp8_linear_layers_b200 import synthetic

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _finite_f32(bits: np.ndarray) -> np.ndarray:
    v = bits.astype(np.uint32).view(np.float32)
    return v[np.isfinite(v)]


# ---- bf16 -------------------------------------------------------------------

def test_bf16_from_f32_matches_torch_rne():
    bits = synthetic.make_uniform_bits(1 << 20, seed=1, tag="bf16")
    v = np.concatenate([_finite_f32(bits), np.array(
        [0.0, -0.0, 1.0, -1.0, 3.3895313e38, 3.4028235e38, 1e-45, -1e-45, 1.00390625, 1.01171875,
         1.0078125, 1.00390637], np.float32)])
    mine = oracle.f32_to_bf16_n(v)
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(mine, ref)


def test_bf16_to_f32_is_exact():
    h = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ref = torch.from_numpy(h.view(np.int16)).view(torch.bfloat16).float().numpy()
    keep = np.isfinite(ref)  # NaN payloads are not preserved through a ctypes float return
    h, ref = h[keep], ref[keep]
    mine = np.array([oracle.bf16_to_f32(int(c)) for c in h[::37]], np.float32)
    assert np.array_equal(mine.view(np.uint32), ref[::37].view(np.uint32))


def _bf16_value(bits: int) -> Fraction:
    f = np.array([bits << 16], np.uint32).view(np.float32)[0]
    return Fraction(float(f))


def _nearest_bf16_brute(v: float) -> int:
    """Nearest bf16 to the f64 value v by exact rational comparison, ties to the
    even code; candidates are the bf16 codes next to the truncation of v."""
    fv = Fraction(v)
    a = abs(fv)
    sign = 0x8000 if np.signbit(v) else 0
    t = int(np.array([abs(np.float32(v))], np.float32).view(np.uint32)[0] >> 16)
    best = None
    for c in range(max(t - 2, 0), min(t + 3, 0x7F80)):
        d = abs(_bf16_value(c) - a)
        if best is None or d < best[0] or (d == best[0] and c % 2 == 0):
            best = (d, c)
    return sign | best[1]


def test_bf16_from_f64_single_rounding_brute_force():
    rng = np.random.default_rng(7)
    # values with more than 24 significant bits, near ties, tiny and subnormal
    base = rng.standard_normal(3000) * np.exp2(rng.integers(-140, 100, 3000))
    ties = np.array([1.0 + 2.0**-8, 1.0 + 3 * 2.0**-8, 1.0 + 2.0**-8 + 2.0**-40, 2.0**-130 * 1.5,
                     2.0**-134, 2.0**-134 * 3, -(1.0 + 2.0**-8), 7.875 + 2.0**-9])
    vals = np.concatenate([base, ties, -ties])
    mine = oracle.f64_to_bf16_n(vals)
    ref = np.array([_nearest_bf16_brute(float(v)) for v in vals], np.uint16)
    assert np.array_equal(mine, ref)


# ---- E4M3 -------------------------------------------------------------------

def _torch_e4m3_table() -> np.ndarray:
    return torch.arange(256, dtype=torch.int32).to(torch.uint8).view(
        torch.float8_e4m3fn).to(torch.float64).numpy()


def test_e4m3_decode_all_codes_match_torch():
    ref = _torch_e4m3_table()
    mine = np.array([oracle.e4m3_decode(c) for c in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(mine), nan)
    assert np.array_equal(mine[~nan], ref[~nan])
    assert np.array_equal(np.signbit(mine[~nan]), np.signbit(ref[~nan]))


def test_e4m3_decode_golden_ocp_table():
    n = 0
    with open(os.path.join(GOLDEN, "e4m3_ocp_values.txt")) as f:
        for line in f:
            if not line.strip() or line.startswith("#"):
                continue
            code, val = line.split()[:2]
            got = oracle.e4m3_decode(int(code, 16))
            if val == "nan":
                assert np.isnan(got), code
            else:
                assert got == float(val) and np.signbit(got) == val.startswith("-"), code
            n += 1
    assert n >= 18


def _e4m3_brute(v: np.ndarray) -> np.ndarray:
    """Nearest finite E4M3 code to each f32 value, ties to the even code,
    saturating at 448, sign kept (exact comparisons in f64)."""
    table = _torch_e4m3_table()
    pos = table[:127]  # codes 0x00..0x7E, increasing
    a = np.abs(v.astype(np.float64))
    idx = np.clip(np.searchsorted(pos, a, side="right") - 1, 0, 125)
    lo, hi = pos[idx], pos[idx + 1]
    twice = 2.0 * a                      # exact
    mid = lo + hi                        # exact: both multiples of 2^-9 below 2^10
    code = np.where(twice < mid, idx, np.where(twice > mid, idx + 1,
                    np.where(idx % 2 == 0, idx, idx + 1)))
    code = np.where(a >= 448.0, 126, code)
    return (code | np.where(np.signbit(v), 0x80, 0)).astype(np.uint8)


def _e4m3_sweep_values() -> np.ndarray:
    # every f32 exponent from subnormal up to 2^9, every top-8-bit mantissa,
    # and low-bit patterns that make the value exact, a tie or one ulp off it
    exps = np.arange(0, 137, dtype=np.uint32)
    hi = np.arange(256, dtype=np.uint32)
    lo = np.array([0, 1, 0x3FFF, 0x4000, 0x4001, 0x7FFF], np.uint32)
    b = (exps[:, None, None] << 23) | (hi[None, :, None] << 15) | lo[None, None, :]
    b = b.ravel()
    structured = np.concatenate([b, b | 0x80000000]).view(np.float32)
    table = _torch_e4m3_table()[:127]
    mids = ((table[:-1] + table[1:]) / 2).astype(np.float32)  # exact in f32
    near = np.concatenate([mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(1e9)),
                           table.astype(np.float32)])
    rand = _finite_f32(synthetic.make_uniform_bits(1 << 20, seed=3, tag="e4m3"))
    extra = np.array([0.0, -0.0, 448.0, 449.0, 464.0, 1e30, -1e30, 2.0**-10, -(2.0**-10),
                      3 * 2.0**-10, 2.0**-6 - 2.0**-10], np.float32)
    return np.concatenate([structured, near, -near, rand, extra])


def test_e4m3_encode_matches_brute_force_nearest():
    v = _e4m3_sweep_values()
    mine = oracle.e4m3_encode_n(v)
    ref = _e4m3_brute(v)
    bad = np.nonzero(mine != ref)[0]
    assert bad.size == 0, [(float(v[i]), hex(mine[i]), hex(ref[i])) for i in bad[:10]]


def test_e4m3_encode_matches_torch_in_range():
    v = _e4m3_sweep_values()
    v = v[np.abs(v) <= 448.0]
    mine = oracle.e4m3_encode_n(v)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(mine, ref)


def test_e4m3_all_codes_round_trip():
    for c in range(256):
        if c in (0x7F, 0xFF):
            continue
        assert oracle.e4m3_encode(oracle.e4m3_decode(c)) == c


# ---- int8 rounding ------------------------------------------------------------

def test_int8_round_golden_cases():
    n = 0
    with open(os.path.join(GOLDEN, "int8_rne_cases.txt")) as f:
        for line in f:
            if not line.strip() or line.startswith("#"):
                continue
            t, q = line.split()
            assert oracle.int8_round(np.float32(t)) == int(q), t
            n += 1
    assert n >= 20


def test_int8_round_matches_numpy_rint():
    rng = np.random.default_rng(11)
    t = np.concatenate([(rng.standard_normal(200000) * 80).astype(np.float32),
                        (np.arange(-300, 300) + 0.5).astype(np.float32),
                        np.arange(-300, 300).astype(np.float32)])
    ref = np.clip(np.rint(t), -127, 127).astype(np.int32)
    assert np.array_equal(oracle.int8_round_n(t), ref)
