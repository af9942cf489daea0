"""CPU oracle for the quantized decoder projection -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product (the CUDA library and its
Python binding) never does, and shares no code with it.

The arithmetic lives in ``oracle.c`` (plain scalar C, exact integer
accumulation, IEEE f32 where the method computes scales and quotients); this
module only marshals numpy arrays through ctypes.  Each function names the
page passage it follows:

* "Llama 3.1 8B Instruct W8A8" model page, intro and "Loading": int8 weights
  with a bf16 scale for each output row, per-token int8 activations, int32 sums.
* "Meta-Llama-3.1-8B-Instruct-FP8-dynamic" README, "Model Optimizations" and
  the "Creation" recipe: E4M3 weights per output channel (static, symmetric),
  E4M3 activations per token (dynamic, symmetric).
* "Qwen3 8B FP8" model page, intro and "Loading": a multiplying scale for each
  128x128 weight block, activations quantized in groups of 128 along K.
* The same pages' "Against bf16" sections: a loader option that never rounds
  the input (weight-only products, ``linear_weight_only``).

Every function has pins in ``tests/test_oracle_*.py`` that do not go through
the oracle's own formulas (brute force, closed forms, library routines).
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from .build import build as _build, LIB_PATH

INT8_ROW = 0
FP8_ROW = 1
FP8_BLOCK = 2
SCHEMES = (INT8_ROW, FP8_ROW, FP8_BLOCK)

_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        path = os.environ.get("QL_ORACLE_LIB")
        if not path:
            _build()
            path = LIB_PATH
        L = ctypes.CDLL(path)
        u8p = ctypes.POINTER(ctypes.c_uint8)
        u16p = ctypes.POINTER(ctypes.c_uint16)
        f32p = ctypes.POINTER(ctypes.c_float)
        f64p = ctypes.POINTER(ctypes.c_double)
        i32p = ctypes.POINTER(ctypes.c_int32)
        i64p = ctypes.POINTER(ctypes.c_int64)
        i64 = ctypes.c_int64
        L.oracle_bf16_to_f32.argtypes = [ctypes.c_uint16]
        L.oracle_bf16_to_f32.restype = ctypes.c_float
        L.oracle_f32_to_bf16.argtypes = [ctypes.c_float]
        L.oracle_f32_to_bf16.restype = ctypes.c_uint16
        L.oracle_f64_to_bf16.argtypes = [ctypes.c_double]
        L.oracle_f64_to_bf16.restype = ctypes.c_uint16
        L.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_decode.restype = ctypes.c_double
        L.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        L.oracle_e4m3_encode.restype = ctypes.c_uint8
        L.oracle_int8_round.argtypes = [ctypes.c_float]
        L.oracle_int8_round.restype = ctypes.c_int32
        L.oracle_quantize_weight.argtypes = [ctypes.c_int, u16p, i64, i64, u8p, f32p]
        L.oracle_quantize_act.argtypes = [ctypes.c_int, u16p, i64, i64, u8p, f32p]
        L.oracle_linear.argtypes = [ctypes.c_int, u8p, f32p, u8p, f32p, i64, i64, i64, u16p, i32p,
                                    f64p]
        L.oracle_linear_sampled.argtypes = [ctypes.c_int, u8p, f32p, u8p, f32p, i64, i64, i64,
                                            i64p, i64p, i64, u16p, i32p, f64p]
        L.oracle_linear_rows.argtypes = [ctypes.c_int, u8p, f32p, u8p, f32p, i64, i64, i64, i64,
                                         i64, u16p, i32p, f64p]
        L.oracle_linear_wo_rows.argtypes = [ctypes.c_int, u16p, u8p, f32p, i64, i64, i64, i64,
                                            i64, u16p, f64p]
        L.oracle_e4m3_encode_n.argtypes = [f32p, i64, u8p]
        L.oracle_f32_to_bf16_n.argtypes = [f32p, i64, u16p]
        L.oracle_int8_round_n.argtypes = [f32p, i64, i32p]
        L.oracle_f64_to_bf16_n.argtypes = [f64p, i64, u16p]
        L.oracle_rounding_is_nearest.restype = ctypes.c_int
        for name in ("oracle_quantize_weight", "oracle_quantize_act", "oracle_linear",
                     "oracle_linear_sampled", "oracle_linear_rows", "oracle_linear_wo_rows"):
            getattr(L, name).restype = ctypes.c_int
        if not L.oracle_rounding_is_nearest():
            raise RuntimeError("oracle: FPU is not rounding to nearest")
        _lib = L
    return _lib


def _p(a: np.ndarray, ct):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.POINTER(ct))


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("bf16 tensors cross the oracle boundary as uint16 bit patterns")
    return a


def scale_shape(scheme: int, rows: int, K: int, weight: bool, N: int | None = None):
    if scheme == FP8_BLOCK:
        return ((N // 128) if weight else rows, K // 128)
    return ((N if weight else rows),)


# ---- codecs ----------------------------------------------------------------

def bf16_to_f32(h: int) -> float:
    return lib().oracle_bf16_to_f32(int(h))


def f32_to_bf16(f: float) -> int:
    return lib().oracle_f32_to_bf16(float(np.float32(f)))


def f64_to_bf16(v: float) -> int:
    return lib().oracle_f64_to_bf16(float(v))


def e4m3_decode(c: int) -> float:
    return lib().oracle_e4m3_decode(int(c))


def e4m3_encode(v: float) -> int:
    return lib().oracle_e4m3_encode(float(np.float32(v)))


def int8_round(t: float) -> int:
    return lib().oracle_int8_round(float(np.float32(t)))


def e4m3_encode_n(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, np.float32).ravel()
    out = np.empty(v.shape[0], np.uint8)
    lib().oracle_e4m3_encode_n(_p(v, ctypes.c_float), v.shape[0], _p(out, ctypes.c_uint8))
    return out


def f32_to_bf16_n(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, np.float32).ravel()
    out = np.empty(v.shape[0], np.uint16)
    lib().oracle_f32_to_bf16_n(_p(v, ctypes.c_float), v.shape[0], _p(out, ctypes.c_uint16))
    return out


def f64_to_bf16_n(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, np.float64).ravel()
    out = np.empty(v.shape[0], np.uint16)
    lib().oracle_f64_to_bf16_n(_p(v, ctypes.c_double), v.shape[0], _p(out, ctypes.c_uint16))
    return out


def int8_round_n(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, np.float32).ravel()
    out = np.empty(v.shape[0], np.int32)
    lib().oracle_int8_round_n(_p(v, ctypes.c_float), v.shape[0], _p(out, ctypes.c_int32))
    return out


# ---- quantizers --------------------------------------------------------------

def quantize_weight(scheme: int, w_bf16: np.ndarray):
    """W [N,K] bf16 bits -> (W_q [N,K] uint8 bytes, s_w f32 [N] or [N/128,K/128])."""
    w = _u16(w_bf16)
    N, K = w.shape
    wq = np.empty((N, K), np.uint8)
    sw = np.empty(scale_shape(scheme, N, K, True, N), np.float32)
    if lib().oracle_quantize_weight(scheme, _p(w, ctypes.c_uint16), N, K, _p(wq, ctypes.c_uint8),
                                    _p(sw, ctypes.c_float)):
        raise ValueError(f"oracle_quantize_weight: bad shape {N}x{K} for scheme {scheme}")
    return wq, sw


def quantize_act(scheme: int, x_bf16: np.ndarray):
    """X [M,K] bf16 bits -> (q_x [M,K] uint8 bytes, s_x f32 [M] or [M,K/128])."""
    x = _u16(x_bf16)
    M, K = x.shape
    qx = np.empty((M, K), np.uint8)
    sx = np.empty(scale_shape(scheme, M, K, False), np.float32)
    if lib().oracle_quantize_act(scheme, _p(x, ctypes.c_uint16), M, K, _p(qx, ctypes.c_uint8),
                                 _p(sx, ctypes.c_float)):
        raise ValueError(f"oracle_quantize_act: bad shape {M}x{K} for scheme {scheme}")
    return qx, sx


# ---- products ------------------------------------------------------------------

def linear(scheme: int, qx, sx, wq, sw, want_acc: bool = False):
    """Full product from quantized operands -> y [M,N] bf16 bits (uint16).

    With want_acc, also returns (acc_i32 or None, acc_f64): the exact int32
    accumulators (int8 scheme) and the exact pre-scale accumulators (row
    schemes) or the exact f64 value before the final rounding (block)."""
    qx = np.ascontiguousarray(qx, np.uint8)
    wq = np.ascontiguousarray(wq, np.uint8)
    sx = np.ascontiguousarray(sx, np.float32)
    sw = np.ascontiguousarray(sw, np.float32)
    M, K = qx.shape
    N = wq.shape[0]
    y = np.empty((M, N), np.uint16)
    acc_i = np.empty((M, N), np.int32) if (want_acc and scheme == INT8_ROW) else None
    acc_d = np.empty((M, N), np.float64) if want_acc else None
    if lib().oracle_linear(scheme, _p(qx, ctypes.c_uint8), _p(sx, ctypes.c_float),
                           _p(wq, ctypes.c_uint8), _p(sw, ctypes.c_float), M, N, K,
                           _p(y, ctypes.c_uint16), _p(acc_i, ctypes.c_int32),
                           _p(acc_d, ctypes.c_double)):
        raise ValueError("oracle_linear: bad shape")
    return (y, acc_i, acc_d) if want_acc else y


def linear_sampled(scheme: int, qx, sx, wq, sw, pm, pn, want_acc: bool = False):
    """Only the outputs (pm[i], pn[i]); for full-size cases."""
    qx = np.ascontiguousarray(qx, np.uint8)
    wq = np.ascontiguousarray(wq, np.uint8)
    sx = np.ascontiguousarray(sx, np.float32)
    sw = np.ascontiguousarray(sw, np.float32)
    pm = np.ascontiguousarray(pm, np.int64)
    pn = np.ascontiguousarray(pn, np.int64)
    M, K = qx.shape
    N = wq.shape[0]
    P = pm.shape[0]
    y = np.empty(P, np.uint16)
    acc_i = np.empty(P, np.int32) if (want_acc and scheme == INT8_ROW) else None
    acc_d = np.empty(P, np.float64) if want_acc else None
    if lib().oracle_linear_sampled(scheme, _p(qx, ctypes.c_uint8), _p(sx, ctypes.c_float),
                                   _p(wq, ctypes.c_uint8), _p(sw, ctypes.c_float), M, N, K,
                                   _p(pm, ctypes.c_int64), _p(pn, ctypes.c_int64), P,
                                   _p(y, ctypes.c_uint16), _p(acc_i, ctypes.c_int32),
                                   _p(acc_d, ctypes.c_double)):
        raise ValueError("oracle_linear_sampled: bad shape or index")
    return (y, acc_i, acc_d) if want_acc else y


def linear_rows(scheme: int, qx, sx, wq, sw, n0: int, n1: int):
    """Output columns [n0, n1) of the full product -> y [M, n1-n0] bf16 bits."""
    qx = np.ascontiguousarray(qx, np.uint8)
    wq = np.ascontiguousarray(wq, np.uint8)
    sx = np.ascontiguousarray(sx, np.float32)
    sw = np.ascontiguousarray(sw, np.float32)
    M, K = qx.shape
    N = wq.shape[0]
    y = np.empty((M, n1 - n0), np.uint16)
    if lib().oracle_linear_rows(scheme, _p(qx, ctypes.c_uint8), _p(sx, ctypes.c_float),
                                _p(wq, ctypes.c_uint8), _p(sw, ctypes.c_float), M, N, K, n0, n1,
                                _p(y, ctypes.c_uint16), None, None):
        raise ValueError("oracle_linear_rows: bad shape")
    return y


def linear_weight_only(scheme: int, x_bf16, wq, sw, n0: int = 0, n1: int | None = None,
                       want_acc: bool = False):
    """Weight-only ("equivalent" numerics, W8A16 / FP8 weight-only) product:
    X stays bf16, each weight is its code times its row or block scale, the
    sum is taken in f64 and rounded once -> y [M, n1-n0] bf16 bits.  The
    loader option that never rounds the input ("Llama 3.1 8B Instruct W8A8",
    "Against bf16"; "Qwen3 8B FP8", "Against bf16") and the W8A16 contrast in
    the W8A8 model page's "Context".  With want_acc also returns the f64 value
    before the final rounding."""
    x = _u16(x_bf16)
    wq = np.ascontiguousarray(wq, np.uint8)
    sw = np.ascontiguousarray(sw, np.float32)
    M, K = x.shape
    N = wq.shape[0]
    n1 = N if n1 is None else n1
    y = np.empty((M, n1 - n0), np.uint16)
    acc = np.empty((M, n1 - n0), np.float64) if want_acc else None
    if lib().oracle_linear_wo_rows(scheme, _p(x, ctypes.c_uint16), _p(wq, ctypes.c_uint8),
                                   _p(sw, ctypes.c_float), M, N, K, n0, n1,
                                   _p(y, ctypes.c_uint16), _p(acc, ctypes.c_double)):
        raise ValueError("oracle_linear_wo_rows: bad shape")
    return (y, acc) if want_acc else y


def forward(scheme: int, x_bf16, wq, sw):
    """The whole method from bf16 X: quantize X per call, multiply, scale."""
    qx, sx = quantize_act(scheme, x_bf16)
    return linear(scheme, qx, sx, wq, sw)


# ---- helpers for checks (decoding only; no method arithmetic) -------------------

def e4m3_table() -> np.ndarray:
    """Value of each of the 256 E4M3 codes (NaN for 0x7F/0xFF), as f64."""
    return np.array([e4m3_decode(c) for c in range(256)], np.float64)


def bf16_bits_to_f64(h: np.ndarray) -> np.ndarray:
    h = np.ascontiguousarray(h, np.uint16)
    return (h.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
