"""Pins for the division steps of the oracle's quantizers (CPU only).

The quantizers take two divisions that decide codes bit for bit: the scale
s = absmax / 127 (int8) or absmax / 448 (E4M3), and the quotient x / s that
is then rounded to a code.  The reading taken for both (the pages say only
"symmetric", per token / per channel / per 128 block) is one correctly
rounded f32 division each, not a product with a rounded reciprocal; the two
differ in the last bit for some operands, and that bit moves codes at
rounding ties.

Everything expected here is computed with exact rationals (``fractions``) and
an explicit round-to-nearest-even onto the f32 (and bf16) grid, written out
below; nothing goes through the oracle's own arithmetic.  The cases:

* every positive finite bf16 absmax -> the scale, for 127 and for 448;
* synthetic tokens with outlier channels, all three schemes -> scales and codes;
* the weight quantizer's row and 128x128 block scales and codes;
* hand-worked cases (``tests/golden/division_cases.txt``) where x / s and
  x * (1 / s) round to different f32 quotients and different codes.
"""
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from fp8_linear_layers_b200 import synthetic

INT8, FP8R, FP8B = oracle.INT8_ROW, oracle.FP8_ROW, oracle.FP8_BLOCK
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
HALF = Fraction(1, 2)


# ---- exact rounding onto a binary floating-point grid --------------------------

def round_to_grid(v: Fraction, precision: int, emin: int) -> Fraction:
    """v rounded to the nearest value with `precision` significant bits and
    exponent >= emin (subnormal spacing 2^(emin - precision + 1) below
    2^emin), ties to the even significand.  No overflow handling: the values
    used here stay far below the largest f32."""
    if v == 0:
        return Fraction(0)
    a = abs(v)
    e = a.numerator.bit_length() - a.denominator.bit_length()  # 2^e <= a < 2^(e+1) after fix-up
    if Fraction(2) ** e > a:
        e -= 1
    elif Fraction(2) ** (e + 1) <= a:
        e += 1
    ulp = Fraction(2) ** (max(e, emin) - precision + 1)
    q = a / ulp
    n = q.numerator // q.denominator
    r = q - n
    if r > HALF or (r == HALF and n % 2 == 1):
        n += 1
    out = n * ulp
    return out if v > 0 else -out


def rn_f32(v: Fraction) -> Fraction:
    return round_to_grid(v, 24, -126)


def rn_bf16(v: Fraction) -> Fraction:
    return round_to_grid(v, 8, -126)


def f32_bits(v: Fraction) -> int:
    """Bit pattern of an f32-representable rational (|v| in the normal or subnormal range)."""
    f = np.float32(float(v))
    assert Fraction(float(f)) == v, "not an f32 value"
    return int(np.array([f], np.float32).view(np.uint32)[0])


# ---- codes from an exact f32 quotient ------------------------------------------

def int8_code(t: Fraction) -> int:
    """Nearest integer, ties to even, clamped to [-127, 127]."""
    n = t.numerator // t.denominator
    r = t - n
    if r > HALF or (r == HALF and n % 2 == 1):
        n += 1
    return max(-127, min(127, n))


def _e4m3_positive_values():
    """(value, code) of the 127 non-negative finite E4M3 codes, from the OCP
    field definition: exponent field 0 is m * 2^-9, else (1 + m/8) 2^(e-7)."""
    out = []
    for c in range(0x7F):
        e, m = c >> 3, c & 7
        v = Fraction(m, 512) if e == 0 else (1 + Fraction(m, 8)) * Fraction(2) ** (e - 7)
        out.append((v, c))
    return out


E4M3_POS = _e4m3_positive_values()


def e4m3_code(t: Fraction, negative: bool) -> int:
    """Nearest E4M3 value to t by exhaustive search, ties to the even code,
    saturating at 448; the sign bit follows the sign of the quotient."""
    a = abs(t)
    best = None
    for v, c in E4M3_POS:
        d = abs(v - a)
        if best is None or d < best[0] or (d == best[0] and c % 2 == 0):
            best = (d, c)
    return (0x80 if negative else 0) | best[1]


def bf16_value(bits: int) -> Fraction:
    return Fraction(float(np.array([int(bits) << 16], np.uint32).view(np.float32)[0]))


def expected_quant(xbits: np.ndarray, qmax: int, bf16_scale: bool = False):
    """Scale and codes of one token / row / group / block (bf16 bits, any
    shape) under the reading: s = RN_f32(absmax / qmax) (then RN_bf16 for the
    W8A8 weight scale), t = RN_f32(x / s), code = nearest code to t."""
    vals = [bf16_value(b) for b in xbits.ravel()]
    a = max(abs(v) for v in vals)
    s = rn_f32(a / qmax)
    if bf16_scale:
        s = rn_bf16(s)
    codes, seen = [], {}  # one exact computation per distinct bf16 value (same scale)
    for b, v in zip(xbits.ravel(), vals):
        b = int(b)
        if b not in seen:
            if s == 0:
                seen[b] = 0
            elif qmax == 127:
                seen[b] = int8_code(rn_f32(v / s)) & 0xFF
            else:
                seen[b] = e4m3_code(rn_f32(v / s), negative=bool(b & 0x8000))
        codes.append(seen[b])
    return s, np.array(codes, np.uint8).reshape(xbits.shape)


# ---- self-checks of the exact helpers (closed forms) ----------------------------

def test_rounder_closed_forms():
    # 1/3 = 0.010101...b: the bits after the 24th significant one read 1010... > 1/2 ulp,
    # so the last kept bit rounds up: 0x3EAAAAAB
    assert f32_bits(rn_f32(Fraction(1, 3))) == 0x3EAAAAAB
    assert f32_bits(rn_f32(Fraction(1, 127))) == int(np.array([np.float32(1) / np.float32(127)]).view(np.uint32)[0])
    # ties: 1 + 2^-24 is halfway between 1 and 1 + 2^-23 -> even (1); 1 + 3 2^-24 -> 1 + 2^-22
    assert rn_f32(1 + Fraction(1, 2**24)) == 1
    assert rn_f32(1 + Fraction(3, 2**24)) == 1 + Fraction(1, 2**22)
    # subnormal spacing 2^-149: 2^-150 ties to 0, 3 2^-150 to 2^-148
    assert rn_f32(Fraction(1, 2**150)) == 0
    assert rn_f32(Fraction(3, 2**150)) == Fraction(1, 2**148)
    # bf16: 1 + 2^-8 ties to 1, 1 + 3 2^-8 to 1 + 2^-6
    assert rn_bf16(1 + Fraction(1, 2**8)) == 1
    assert rn_bf16(1 + Fraction(3, 2**8)) == 1 + Fraction(1, 2**6)
    assert int8_code(Fraction(5, 2)) == 2 and int8_code(Fraction(-7, 2)) == -4
    assert int8_code(Fraction(300)) == 127 and int8_code(Fraction(-300)) == -127
    # E4M3: 17 lies between 16 (0x58) and 18 (0x59): tie to the even code 0x58
    assert e4m3_code(Fraction(17), False) == 0x58
    assert e4m3_code(Fraction(449), True) == 0xFE
    assert e4m3_code(Fraction(1, 1024), False) == 0x00  # half of the smallest subnormal: tie to 0


def test_rounder_matches_numpy_division_on_random_operands():
    """IEEE f32 division (numpy, a library routine) is the correctly rounded
    quotient; the exact rounder must agree on random operands."""
    rng = np.random.default_rng(11)
    a = (rng.standard_normal(400) * np.exp2(rng.integers(-30, 30, 400))).astype(np.float32)
    b = (rng.standard_normal(400) * np.exp2(rng.integers(-30, 30, 400))).astype(np.float32)
    q = a / b
    for x, y, z in zip(a, b, q):
        assert rn_f32(Fraction(float(x)) / Fraction(float(y))) == Fraction(float(z))


# ---- the scale: every positive finite bf16 absmax -------------------------------

@pytest.mark.parametrize("scheme", [INT8, FP8R])
def test_act_scale_is_one_correctly_rounded_division_for_every_bf16_absmax(scheme):
    """Token i holds one element, the i-th positive finite bf16 value; its
    scale must be RN_f32(a / 127) or RN_f32(a / 448) for every a."""
    a_bits = np.arange(1, 0x7F80, dtype=np.uint16)  # positive finite bf16
    K = 16
    x = np.zeros((a_bits.size, K), np.uint16)
    x[:, 5] = a_bits
    _, sx = oracle.quantize_act(scheme, x)
    qmax = 127 if scheme == INT8 else 448
    # the exact quotient's rounding, computed per distinct value
    want = np.array([f32_bits(rn_f32(bf16_value(b) / qmax)) for b in a_bits], np.uint32)
    got = sx.view(np.uint32)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, f"{bad.size} scales differ; first absmax bits {a_bits[bad[:5]]}"


# ---- tokens with outliers: scales and codes, all schemes -------------------------

@pytest.mark.parametrize("scheme", [INT8, FP8R, FP8B])
@pytest.mark.parametrize("seed", [0, 1])
def test_act_codes_from_exact_quotients(scheme, seed):
    M, K = 6, 1024
    x = synthetic.make_x(M, K, seed=seed, tag="division-pin", outliers=10)
    qx, sx = oracle.quantize_act(scheme, x)
    qmax = 127 if scheme == INT8 else 448
    width = 128 if scheme == FP8B else K
    G = K // width
    for m in range(M):
        for g in range(G):
            xs = x[m, g * width:(g + 1) * width]
            s, codes = expected_quant(xs, qmax)
            assert sx.reshape(M, G)[m, g] == np.float32(float(s)), (m, g)
            got = qx[m, g * width:(g + 1) * width]
            diff = np.nonzero(got != codes)[0]
            assert diff.size == 0, f"token {m} group {g}: {diff.size} codes differ at {diff[:5]}"


@pytest.mark.parametrize("scheme", [INT8, FP8R])
def test_act_codes_dense_sweep_at_several_scales(scheme):
    """Every bf16 x in [-a, a] at a few absmax values a (denser than random
    tokens, so that many quotients sit next to a rounding boundary)."""
    qmax = 127 if scheme == INT8 else 448
    for a_val in (3.0, 0.7109375, 1.0e-3, 213.0):
        a_bits = int(np.array([np.float32(a_val)], np.float32).view(np.uint32)[0] >> 16)
        xs = np.arange(0, a_bits + 1, 7, dtype=np.uint32)
        xs = np.concatenate([xs, xs | 0x8000, [a_bits]]).astype(np.uint16)
        K = (xs.size + 15) // 16 * 16
        row = np.zeros(K, np.uint16)
        row[:xs.size] = xs
        qx, sx = oracle.quantize_act(scheme, row[None, :])
        s, codes = expected_quant(row, qmax)
        assert sx[0] == np.float32(float(s))
        diff = np.nonzero(qx[0] != codes)[0]
        assert diff.size == 0, f"absmax {a_val}: {diff.size} codes differ, first x bits {row[diff[:5]]}"


# ---- the weight quantizer's scales and codes -------------------------------------

@pytest.mark.parametrize("scheme", [INT8, FP8R])
def test_weight_rows_from_exact_quotients(scheme):
    N, K = 24, 512
    w = synthetic.make_w(N, K, seed=3, tag="division-pin-w")
    wq, sw = oracle.quantize_weight(scheme, w)
    qmax = 127 if scheme == INT8 else 448
    for n in range(N):
        s, codes = expected_quant(w[n], qmax, bf16_scale=(scheme == INT8))
        assert sw[n] == np.float32(float(s)), n
        diff = np.nonzero(wq[n] != codes)[0]
        assert diff.size == 0, f"row {n}: {diff.size} codes differ at {diff[:5]}"


def test_weight_blocks_from_exact_quotients():
    N, K = 256, 384
    w = synthetic.make_w(N, K, seed=4, tag="division-pin-wb")
    wq, sw = oracle.quantize_weight(FP8B, w)
    for nb in range(N // 128):
        for kb in range(K // 128):
            blk = w[nb * 128:(nb + 1) * 128, kb * 128:(kb + 1) * 128]
            s, codes = expected_quant(blk, 448)
            assert sw[nb, kb] == np.float32(float(s)), (nb, kb)
            got = wq[nb * 128:(nb + 1) * 128, kb * 128:(kb + 1) * 128]
            assert np.array_equal(got, codes), (nb, kb, int((got != codes).sum()))


# ---- hand-worked cases where the reciprocal product rounds differently ----------

def _load_cases():
    cases = []
    with open(os.path.join(GOLDEN, "division_cases.txt")) as f:
        for ln in f:
            ln = ln.split("#", 1)[0].strip()
            if not ln:
                continue
            kind, a_hex, x_hex, s_hex, t_hex, code_hex, r_hex, rcode_hex = ln.split()
            cases.append((kind, int(a_hex, 16), int(x_hex, 16), int(s_hex, 16), int(t_hex, 16),
                          int(code_hex, 16), int(r_hex, 16), int(rcode_hex, 16)))
    return cases


CASES = _load_cases()


def test_golden_division_cases_restate_exactly():
    """The fixture's scale, quotient and code follow from the exact rationals;
    the reciprocal route's quotient and code follow too, and differ."""
    assert len(CASES) >= 6
    for kind, a, x, s_bits, t_bits, code, r_bits, rcode in CASES:
        qmax = 127 if kind == "int8" else 448
        s = rn_f32(bf16_value(a) / qmax)
        assert f32_bits(s) == s_bits
        t = rn_f32(bf16_value(x) / s)
        assert f32_bits(t) == t_bits
        r = rn_f32(rn_f32(Fraction(1) / s) * bf16_value(x))  # x * (1 / s), two roundings
        assert f32_bits(r) == r_bits and r != t
        if kind == "int8":
            assert int8_code(t) & 0xFF == code and int8_code(r) & 0xFF == rcode
        else:
            assert e4m3_code(t, x & 0x8000 != 0) == code and e4m3_code(r, x & 0x8000 != 0) == rcode
        assert code != rcode


@pytest.mark.parametrize("case", CASES, ids=[f"{c[0]}-{c[1]:04x}-{c[2]:04x}" for c in CASES])
def test_golden_division_cases_through_the_oracle(case):
    kind, a, x, s_bits, t_bits, code, r_bits, rcode = case
    scheme = INT8 if kind == "int8" else FP8R
    row = np.zeros((1, 16), np.uint16)
    row[0, 0], row[0, 1] = a, x
    qx, sx = oracle.quantize_act(scheme, row)
    assert int(sx.view(np.uint32)[0]) == s_bits
    assert int(qx[0, 1]) == code, f"oracle code {qx[0, 1]:#x}, exact {code:#x}, reciprocal {rcode:#x}"
