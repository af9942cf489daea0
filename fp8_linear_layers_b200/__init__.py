"""Quantized decoder projections on B200: Python binding of ``libqlinear.so``.

This module only marshals arguments: it checks dtypes, devices and
contiguity, allocates outputs with torch when the caller does not pass them,
and calls the C ABI declared in ``include/qlinear.h``.  Every step of the
computation runs in the library's CUDA kernels; there is no fallback.  If the
library is not built, importing the functions raises.

Schemes (see the header for the exact numerics):
    W8A8_INT8_ROW      int8 weights, one bf16 scale per output row, per-token int8 activations
    FP8_E4M3_ROW       E4M3 weights per output row, per-token dynamic E4M3 activations
    FP8_E4M3_BLOCK128  E4M3 weights per 128x128 block, E4M3 activations per 128-input group

Tensors: bf16 activations/outputs as ``torch.bfloat16``; quantized codes as
``torch.uint8`` (view them as ``torch.int8`` / ``torch.float8_e4m3fn``);
scales as ``torch.float32``.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

W8A8_INT8_ROW = 0
FP8_E4M3_ROW = 1
FP8_E4M3_BLOCK128 = 2
SCHEMES = (W8A8_INT8_ROW, FP8_E4M3_ROW, FP8_E4M3_BLOCK128)
SCHEME_NAMES = {W8A8_INT8_ROW: "w8a8_int8_row", FP8_E4M3_ROW: "fp8_e4m3_row",
                FP8_E4M3_BLOCK128: "fp8_e4m3_block128"}

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libqlinear.so")

STATUS = {0: "QL_OK", 1: "QL_ERR_INVALID_ARG", 2: "QL_ERR_UNSUPPORTED_SHAPE", 3: "QL_ERR_MISALIGNED",
          4: "QL_ERR_CUDA", 5: "QL_ERR_TIMEOUT", 6: "QL_ERR_DEVICE", 7: "QL_ERR_WORKSPACE"}

# Every function the C ABI exports (kept in step with include/qlinear.h by a test).
EXPORTS = ("qlinear_quantize_weight", "qlinear_quantize_act", "qlinear_gemv", "qlinear_gemm_small",
           "qlinear_gemm", "qlinear_forward", "qlinear_workspace_bytes",
           "qlinear_forward_workspace_bytes", "qlinear_get_device_status", "qlinear_status_string",
           "qlinear_last_cuda_error", "qlinear_gemm_small_noalloc", "qlinear_gemv_weight_only",
           "qlinear_debug_gemv_stalled", "qlinear_forward_weight_only", "qlinear_gemv_grouped",
           "qlinear_gemv_prequant", "qlinear_gemm_small_prequant",
           "qlinear_gemm_quant_out", "qlinear_weight_only_workspace_bytes", "qlinear_gemm_grouped",
           "qlinear_gemm_grouped_workspace_bytes", "qlinear_gemm_small_grouped",
           "qlinear_gemm_small_grouped_workspace_bytes")


class QLinearError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str = ""):
        self.status = status
        msg = f"{where}: {STATUS.get(status, status)}"
        if detail:
            msg += f" ({detail})"
        super().__init__(msg)


class _Debug(ctypes.Structure):
    _fields_ = [("qx", ctypes.c_void_p), ("sx", ctypes.c_void_p), ("acc_i32", ctypes.c_void_p),
                ("acc_f32", ctypes.c_void_p)]


@dataclass
class Debug:
    """Optional capture buffers (device tensors) for bit-exact checks."""
    qx: torch.Tensor | None = None
    sx: torch.Tensor | None = None
    acc_i32: torch.Tensor | None = None
    acc_f32: torch.Tensor | None = None

    def _c(self):
        p = lambda t: None if t is None else t.data_ptr()
        return ctypes.byref(_Debug(p(self.qx), p(self.sx), p(self.acc_i32), p(self.acc_f32)))


_lib = None


def lib() -> ctypes.CDLL:
    """Load libqlinear.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m fp8_linear_layers_b200.build` (nvcc, sm_100a)")
        L = ctypes.CDLL(LIB_PATH)
        vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
        L.qlinear_quantize_weight.argtypes = [i32, vp, i64, i64, vp, vp, vp]
        L.qlinear_quantize_act.argtypes = [i32, vp, i64, i64, vp, vp, vp]
        L.qlinear_gemv.argtypes = [i32, vp, vp, vp, i64, i64, vp, vp, vp]
        L.qlinear_gemv_weight_only.argtypes = [i32, vp, vp, vp, i64, i64, vp, vp]
        L.qlinear_debug_gemv_stalled.argtypes = [i32, vp, vp, vp, i64, i64, vp, vp]
        L.qlinear_forward_weight_only.argtypes = [i32, vp, vp, vp, i64, i64, i64, vp, vp, sz, vp]
        L.qlinear_weight_only_workspace_bytes.argtypes = [i32, i64, i64, i64]
        L.qlinear_weight_only_workspace_bytes.restype = sz
        L.qlinear_gemv_grouped.argtypes = [i32, vp, i32, i64, vp]
        L.qlinear_gemv_prequant.argtypes = [i32, vp, vp, vp, vp, i64, i64, vp, vp]
        L.qlinear_gemm_small_prequant.argtypes = [i32, vp, vp, vp, vp, i64, i64, i64, vp, vp, sz, vp]
        L.qlinear_gemm_quant_out.argtypes = [i32, vp, vp, vp, vp, i64, i64, i64, vp, vp, vp, vp, sz, vp]
        L.qlinear_gemm_small.argtypes = [i32, vp, vp, vp, i64, i64, i64, vp, vp, sz, vp, vp]
        L.qlinear_gemm.argtypes = [i32, vp, vp, vp, vp, i64, i64, i64, vp, vp, sz, vp, vp]
        L.qlinear_gemm_grouped.argtypes = [i32, vp, vp, vp, i32, i64, i64, vp, sz, vp]
        L.qlinear_gemm_grouped_workspace_bytes.argtypes = [i32, vp, i32, i64, i64]
        L.qlinear_gemm_grouped_workspace_bytes.restype = sz
        L.qlinear_gemm_small_grouped.argtypes = [i32, vp, vp, vp, vp, i32, i64, i64, vp, sz, vp]
        L.qlinear_gemm_small_grouped_workspace_bytes.argtypes = [i32, vp, i32, i64, i64]
        L.qlinear_gemm_small_grouped_workspace_bytes.restype = sz
        L.qlinear_forward.argtypes = [i32, vp, vp, vp, i64, i64, i64, vp, vp, sz, vp]
        L.qlinear_gemm_small_noalloc.argtypes = [i32, vp, vp, vp, i64, i64, i64, vp, vp]
        L.qlinear_workspace_bytes.argtypes = [i32, i64, i64, i64]
        L.qlinear_workspace_bytes.restype = sz
        L.qlinear_forward_workspace_bytes.argtypes = [i32, i64, i64, i64]
        L.qlinear_forward_workspace_bytes.restype = sz
        L.qlinear_get_device_status.argtypes = [vp, ctypes.POINTER(ctypes.c_uint32)]
        L.qlinear_status_string.argtypes = [i32]
        L.qlinear_status_string.restype = ctypes.c_char_p
        L.qlinear_last_cuda_error.restype = ctypes.c_char_p
        for name in ("qlinear_quantize_weight", "qlinear_quantize_act", "qlinear_gemv",
                     "qlinear_gemm_small", "qlinear_gemm", "qlinear_forward",
                     "qlinear_get_device_status", "qlinear_gemm_small_noalloc",
                     "qlinear_gemv_weight_only", "qlinear_debug_gemv_stalled",
                     "qlinear_forward_weight_only", "qlinear_gemv_grouped",
                     "qlinear_gemv_prequant", "qlinear_gemm_small_prequant",
                     "qlinear_gemm_quant_out"):
            getattr(L, name).restype = i32
        _lib = L
    return _lib


def _check(status: int, where: str):
    if status != 0:
        detail = ""
        if status == 4:
            detail = lib().qlinear_last_cuda_error().decode(errors="replace")
        raise QLinearError(status, where, detail)


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dev(t: torch.Tensor, dtype, name: str) -> int:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def weight_scale_shape(scheme: int, N: int, K: int) -> tuple:
    return (N // 128, K // 128) if scheme == FP8_E4M3_BLOCK128 else (N,)


def act_scale_shape(scheme: int, M: int, K: int) -> tuple:
    return (M, K // 128) if scheme == FP8_E4M3_BLOCK128 else (M,)


def quantize_weight(scheme: int, w: torch.Tensor, stream=None):
    """W bf16 [N,K] -> (W_q uint8 [N,K], s_w f32 [N] or [N/128,K/128])."""
    N, K = w.shape
    wq = torch.empty((N, K), dtype=torch.uint8, device=w.device)
    sw = torch.empty(weight_scale_shape(scheme, N, K), dtype=torch.float32, device=w.device)
    _check(lib().qlinear_quantize_weight(scheme, _dev(w, torch.bfloat16, "w"), N, K, wq.data_ptr(),
                                         sw.data_ptr(), _stream(stream)), "qlinear_quantize_weight")
    return wq, sw


def quantize_act(scheme: int, x: torch.Tensor, qx=None, sx=None, stream=None):
    """X bf16 [M,K] -> (q_x uint8 [M,K], s_x f32 [M] or [M,K/128])."""
    M, K = x.shape
    if qx is None:
        qx = torch.empty((M, K), dtype=torch.uint8, device=x.device)
    if sx is None:
        sx = torch.empty(act_scale_shape(scheme, M, K), dtype=torch.float32, device=x.device)
    _check(lib().qlinear_quantize_act(scheme, _dev(x, torch.bfloat16, "x"), M, K,
                                      _dev(qx, torch.uint8, "qx"), _dev(sx, torch.float32, "sx"),
                                      _stream(stream)), "qlinear_quantize_act")
    return qx, sx


def gemv(scheme: int, x: torch.Tensor, wq: torch.Tensor, sw: torch.Tensor, y=None,
         debug: Debug | None = None, stream=None) -> torch.Tensor:
    """M = 1: x bf16 [1,K] (or [K]) -> y bf16 [1,N]."""
    K = x.shape[-1]
    N = wq.shape[0]
    if x.numel() != K:
        raise ValueError("gemv takes a single token")
    if y is None:
        y = torch.empty((1, N), dtype=torch.bfloat16, device=x.device)
    _check(lib().qlinear_gemv(scheme, _dev(x, torch.bfloat16, "x"), _dev(wq, torch.uint8, "wq"),
                              _dev(sw, torch.float32, "sw"), N, K, _dev(y, torch.bfloat16, "y"),
                              debug._c() if debug else None, _stream(stream)), "qlinear_gemv")
    return y


GEMV_MAX_GROUP = 8  # QL_GEMV_MAX_GROUP


class _GemvProblem(ctypes.Structure):
    _fields_ = [("x", ctypes.c_void_p), ("qx", ctypes.c_void_p), ("sx", ctypes.c_void_p),
                ("wq", ctypes.c_void_p), ("sw", ctypes.c_void_p), ("y", ctypes.c_void_p),
                ("N", ctypes.c_int64)]


def gemv_grouped(scheme: int, problems, stream=None) -> list:
    """Several M = 1 products of one K in one launch.  `problems` is a list of
    (x, wq [N,K], sw, y or None) tuples, x a bf16 [1,K] tensor or a pair
    (q_x [1,K] uint8, s_x f32) already quantized; returns the outputs [1,N]."""
    if not 1 <= len(problems) <= GEMV_MAX_GROUP:
        raise ValueError(f"1 to {GEMV_MAX_GROUP} products per grouped launch")
    K = problems[0][1].shape[1]
    table = (_GemvProblem * len(problems))()
    ys = []
    for j, (x, wq, sw, y) in enumerate(problems):
        qx, sx = (x if isinstance(x, tuple) else (None, None))
        xin = qx if qx is not None else x
        if xin.numel() != K or xin.shape[-1] != K or wq.shape[1] != K:
            raise ValueError("every product of a grouped launch takes one token of the same K")
        N = wq.shape[0]
        if y is None:
            y = torch.empty((1, N), dtype=torch.bfloat16, device=xin.device)
        if qx is None:
            table[j] = _GemvProblem(_dev(x, torch.bfloat16, "x"), None, None, _dev(wq, torch.uint8, "wq"),
                                    _dev(sw, torch.float32, "sw"), _dev(y, torch.bfloat16, "y"), N)
        else:
            table[j] = _GemvProblem(None, _dev(qx, torch.uint8, "qx"), _dev(sx, torch.float32, "sx"),
                                    _dev(wq, torch.uint8, "wq"), _dev(sw, torch.float32, "sw"),
                                    _dev(y, torch.bfloat16, "y"), N)
        ys.append(y)
    _check(lib().qlinear_gemv_grouped(scheme, ctypes.cast(table, ctypes.c_void_p), len(problems), K,
                                      _stream(stream)), "qlinear_gemv_grouped")
    return ys


def gemv_prequant(scheme: int, qx: torch.Tensor, sx: torch.Tensor, wq: torch.Tensor, sw: torch.Tensor,
                  y=None, stream=None) -> torch.Tensor:
    """M = 1 on an input already quantized: q_x uint8 [1,K], s_x f32 -> y bf16 [1,N]."""
    K = qx.shape[-1]
    N = wq.shape[0]
    if qx.numel() != K:
        raise ValueError("gemv_prequant takes a single token")
    if y is None:
        y = torch.empty((1, N), dtype=torch.bfloat16, device=qx.device)
    _check(lib().qlinear_gemv_prequant(scheme, _dev(qx, torch.uint8, "qx"), _dev(sx, torch.float32, "sx"),
                                       _dev(wq, torch.uint8, "wq"), _dev(sw, torch.float32, "sw"), N, K,
                                       _dev(y, torch.bfloat16, "y"), _stream(stream)),
           "qlinear_gemv_prequant")
    return y


def gemv_weight_only(scheme: int, x: torch.Tensor, wq: torch.Tensor, sw: torch.Tensor, y=None,
                     stream=None) -> torch.Tensor:
    """M = 1 weight-only product ("equivalent" numerics, W8A16 / FP8 weight-only):
    x bf16 [1,K] (or [K]) is not rounded -> y bf16 [1,N]."""
    K = x.shape[-1]
    N = wq.shape[0]
    if x.numel() != K:
        raise ValueError("gemv_weight_only takes a single token")
    if y is None:
        y = torch.empty((1, N), dtype=torch.bfloat16, device=x.device)
    _check(lib().qlinear_gemv_weight_only(scheme, _dev(x, torch.bfloat16, "x"),
                                          _dev(wq, torch.uint8, "wq"), _dev(sw, torch.float32, "sw"),
                                          N, K, _dev(y, torch.bfloat16, "y"), _stream(stream)),
           "qlinear_gemv_weight_only")
    return y


def debug_gemv_stalled(scheme: int, x: torch.Tensor, wq: torch.Tensor, sw: torch.Tensor, y=None,
                       stream=None) -> torch.Tensor:
    """Test hook: gemv with its weight copies held back, so its bounded waits run
    out (about 2 s) and the kernel records QL_ERR_TIMEOUT in the status word."""
    K = x.shape[-1]
    N = wq.shape[0]
    if y is None:
        y = torch.empty((1, N), dtype=torch.bfloat16, device=x.device)
    _check(lib().qlinear_debug_gemv_stalled(scheme, _dev(x, torch.bfloat16, "x"),
                                            _dev(wq, torch.uint8, "wq"), _dev(sw, torch.float32, "sw"),
                                            N, K, _dev(y, torch.bfloat16, "y"), _stream(stream)),
           "qlinear_debug_gemv_stalled")
    return y


def forward_weight_only(scheme: int, x: torch.Tensor, wq: torch.Tensor, sw: torch.Tensor, y=None,
                        workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """1 <= M <= 32 weight-only product: x bf16 [M,K] is not rounded -> y bf16 [M,N].
    A zero-filled workspace of weight_only_workspace_bytes(...) is made if none is given."""
    M, K = x.shape
    N = wq.shape[0]
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    if workspace is None:
        nb = weight_only_workspace_bytes(scheme, M, N, K)
        workspace = new_workspace(nb) if nb else None
    wp, wn = _ws(workspace)
    _check(lib().qlinear_forward_weight_only(scheme, _dev(x, torch.bfloat16, "x"),
                                             _dev(wq, torch.uint8, "wq"),
                                             _dev(sw, torch.float32, "sw"), M, N, K,
                                             _dev(y, torch.bfloat16, "y"), wp, wn, _stream(stream)),
           "qlinear_forward_weight_only")
    return y


def weight_only_workspace_bytes(scheme: int, M: int, N: int, K: int) -> int:
    return int(lib().qlinear_weight_only_workspace_bytes(scheme, M, N, K))


def workspace_bytes(scheme: int, M: int, N: int, K: int) -> int:
    return int(lib().qlinear_workspace_bytes(scheme, M, N, K))


def forward_workspace_bytes(scheme: int, M: int, N: int, K: int) -> int:
    return int(lib().qlinear_forward_workspace_bytes(scheme, M, N, K))


def new_workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """A zero-filled workspace buffer (the library keeps it zero-filled after each call)."""
    return torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=device)


def _ws(workspace):
    if workspace is None:
        return None, 0
    return _dev(workspace, torch.uint8, "workspace"), workspace.numel()


def gemm_small(scheme: int, x: torch.Tensor, wq: torch.Tensor, sw: torch.Tensor,
               workspace: torch.Tensor, y=None, debug: Debug | None = None, stream=None):
    """1 <= M <= 32 on the tensor cores: x bf16 [M,K] -> y bf16 [M,N]."""
    M, K = x.shape
    N = wq.shape[0]
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    wp, wn = _ws(workspace)
    _check(lib().qlinear_gemm_small(scheme, _dev(x, torch.bfloat16, "x"), _dev(wq, torch.uint8, "wq"),
                                    _dev(sw, torch.float32, "sw"), M, N, K,
                                    _dev(y, torch.bfloat16, "y"), wp, wn,
                                    debug._c() if debug else None, _stream(stream)),
           "qlinear_gemm_small")
    return y


def gemm_small_prequant(scheme: int, qx: torch.Tensor, sx: torch.Tensor, wq: torch.Tensor,
                        sw: torch.Tensor, workspace: torch.Tensor, y=None, stream=None):
    """1 <= M <= 32 on an input already quantized: q_x uint8 [M,K], s_x f32 -> y bf16 [M,N]."""
    M, K = qx.shape
    N = wq.shape[0]
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=qx.device)
    wp, wn = _ws(workspace)
    _check(lib().qlinear_gemm_small_prequant(scheme, _dev(qx, torch.uint8, "qx"), _dev(sx, torch.float32, "sx"),
                                             _dev(wq, torch.uint8, "wq"), _dev(sw, torch.float32, "sw"),
                                             M, N, K, _dev(y, torch.bfloat16, "y"), wp, wn, _stream(stream)),
           "qlinear_gemm_small_prequant")
    return y


def gemm_small_noalloc(scheme: int, x: torch.Tensor, wq: torch.Tensor, sw: torch.Tensor, y=None,
                       stream=None):
    """Same as ``gemm_small`` with the library's fixed device scratch instead of a
    caller workspace (for callers that cannot allocate; calls must not overlap)."""
    M, K = x.shape
    N = wq.shape[0]
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    status = lib().qlinear_gemm_small_noalloc(scheme, _dev(x, torch.bfloat16, "x"),
                                              _dev(wq, torch.uint8, "wq"), _dev(sw, torch.float32, "sw"),
                                              M, N, K, _dev(y, torch.bfloat16, "y"), _stream(stream))
    if status == 7:  # the shape needs more than the fixed scratch; the library says how much
        raise QLinearError(status, "qlinear_gemm_small_noalloc",
                           lib().qlinear_last_cuda_error().decode(errors="replace"))
    _check(status, "qlinear_gemm_small_noalloc")
    return y


def gemm(scheme: int, qx: torch.Tensor, sx: torch.Tensor, wq: torch.Tensor, sw: torch.Tensor,
         workspace: torch.Tensor | None = None, y=None, debug: Debug | None = None, stream=None):
    """Large M on pre-quantized activations: q_x [M,K], s_x -> y bf16 [M,N]."""
    M, K = qx.shape
    N = wq.shape[0]
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=qx.device)
    wp, wn = _ws(workspace)
    _check(lib().qlinear_gemm(scheme, _dev(qx, torch.uint8, "qx"), _dev(sx, torch.float32, "sx"),
                              _dev(wq, torch.uint8, "wq"), _dev(sw, torch.float32, "sw"), M, N, K,
                              _dev(y, torch.bfloat16, "y"), wp, wn, debug._c() if debug else None,
                              _stream(stream)), "qlinear_gemm")
    return y


GEMM_MAX_GROUP = 4  # QL_GEMM_MAX_GROUP


class _GemmProblem(ctypes.Structure):
    _fields_ = [("wq", ctypes.c_void_p), ("sw", ctypes.c_void_p), ("y", ctypes.c_void_p), ("qy", ctypes.c_void_p),
                ("sy", ctypes.c_void_p), ("N", ctypes.c_int64)]


def gemm_grouped_workspace_bytes(scheme: int, Ns, M: int, K: int) -> int:
    arr = (ctypes.c_int64 * len(Ns))(*Ns)
    return int(lib().qlinear_gemm_grouped_workspace_bytes(scheme, ctypes.cast(arr, ctypes.c_void_p), len(Ns),
                                                          M, K))


def gemm_grouped(scheme: int, qx: torch.Tensor, sx: torch.Tensor, problems, workspace: torch.Tensor | None = None,
                 stream=None) -> list:
    """Several large-M products on one quantized input in one launch.
    `problems` is a list of (wq [N,K], sw, y or None) or, block scheme, of
    (wq, sw, y or None, qy [M,N] uint8, sy [M,N/128] f32) to also write each
    output's codes and scales (y may then be False: codes only); returns the
    outputs [M,N] (None where not written)."""
    if not 1 <= len(problems) <= GEMM_MAX_GROUP:
        raise ValueError(f"1 to {GEMM_MAX_GROUP} products per grouped launch")
    M, K = qx.shape
    table = (_GemmProblem * len(problems))()
    ys = []
    for j, prob in enumerate(problems):
        wq, sw, y = prob[:3]
        qy, sy = prob[3:5] if len(prob) > 3 else (None, None)
        if wq.shape[1] != K:
            raise ValueError("every product of a grouped launch reads the same [M,K] input")
        N = wq.shape[0]
        if y is None:
            y = torch.empty((M, N), dtype=torch.bfloat16, device=qx.device)
        elif y is False:
            y = None
        table[j] = _GemmProblem(_dev(wq, torch.uint8, "wq"), _dev(sw, torch.float32, "sw"),
                                _dev(y, torch.bfloat16, "y") if y is not None else None,
                                _dev(qy, torch.uint8, "qy") if qy is not None else None,
                                _dev(sy, torch.float32, "sy") if sy is not None else None, N)
        ys.append(y)
    wp, wn = _ws(workspace)
    _check(lib().qlinear_gemm_grouped(scheme, _dev(qx, torch.uint8, "qx"), _dev(sx, torch.float32, "sx"),
                                      ctypes.cast(table, ctypes.c_void_p), len(problems), M, K, wp, wn,
                                      _stream(stream)), "qlinear_gemm_grouped")
    return ys


def gemm_small_grouped_workspace_bytes(scheme: int, Ns, M: int, K: int) -> int:
    arr = (ctypes.c_int64 * len(Ns))(*Ns)
    return int(lib().qlinear_gemm_small_grouped_workspace_bytes(scheme, ctypes.cast(arr, ctypes.c_void_p),
                                                                len(Ns), M, K))


def gemm_small_grouped(scheme: int, x, problems, workspace: torch.Tensor, stream=None) -> list:
    """Several 1 <= M <= 32 products on the same tokens in one launch.  x is a
    bf16 [M,K] tensor or a pair (q_x [M,K] uint8, s_x f32) already quantized;
    `problems` a list of (wq [N,K], sw, y or None); returns the outputs [M,N]."""
    if not 1 <= len(problems) <= GEMM_MAX_GROUP:
        raise ValueError(f"1 to {GEMM_MAX_GROUP} products per grouped launch")
    qx, sx = x if isinstance(x, tuple) else (None, None)
    xin = qx if qx is not None else x
    M, K = xin.shape
    table = (_GemmProblem * len(problems))()
    ys = []
    for j, (wq, sw, y) in enumerate(problems):
        if wq.shape[1] != K:
            raise ValueError("every product of a grouped launch reads the same [M,K] tokens")
        N = wq.shape[0]
        if y is None:
            y = torch.empty((M, N), dtype=torch.bfloat16, device=xin.device)
        table[j] = _GemmProblem(_dev(wq, torch.uint8, "wq"), _dev(sw, torch.float32, "sw"),
                                _dev(y, torch.bfloat16, "y"), None, None, N)
        ys.append(y)
    wp, wn = _ws(workspace)
    if qx is None:
        args = (_dev(x, torch.bfloat16, "x"), None, None)
    else:
        args = (None, _dev(qx, torch.uint8, "qx"), _dev(sx, torch.float32, "sx"))
    _check(lib().qlinear_gemm_small_grouped(scheme, *args, ctypes.cast(table, ctypes.c_void_p), len(problems), M, K,
                                            wp, wn, _stream(stream)), "qlinear_gemm_small_grouped")
    return ys


def gemm_quant_out(scheme: int, qx: torch.Tensor, sx: torch.Tensor, wq: torch.Tensor, sw: torch.Tensor,
                   workspace: torch.Tensor | None = None, y=None, want_y: bool = True, qy=None, sy=None,
                   stream=None):
    """Block scheme, large M: q_x, s_x -> (y bf16 [M,N] or None, q_y uint8 [M,N], s_y f32 [M,N/128]),
    the output quantized in the same kernel for the product that reads it next."""
    M, K = qx.shape
    N = wq.shape[0]
    if want_y and y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=qx.device)
    if qy is None:
        qy = torch.empty((M, N), dtype=torch.uint8, device=qx.device)
    if sy is None:
        sy = torch.empty((M, N // 128), dtype=torch.float32, device=qx.device)
    wp, wn = _ws(workspace)
    _check(lib().qlinear_gemm_quant_out(scheme, _dev(qx, torch.uint8, "qx"), _dev(sx, torch.float32, "sx"),
                                        _dev(wq, torch.uint8, "wq"), _dev(sw, torch.float32, "sw"), M, N, K,
                                        _dev(y, torch.bfloat16, "y") if y is not None else None,
                                        _dev(qy, torch.uint8, "qy"), _dev(sy, torch.float32, "sy"), wp, wn,
                                        _stream(stream)), "qlinear_gemm_quant_out")
    return y, qy, sy


def forward(scheme: int, x: torch.Tensor, wq: torch.Tensor, sw: torch.Tensor,
            workspace: torch.Tensor | None = None, y=None, stream=None) -> torch.Tensor:
    """The projection as a model calls it (dispatch on M: GEMV / small-M / large-M)."""
    M, K = x.shape
    N = wq.shape[0]
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    wp, wn = _ws(workspace)
    _check(lib().qlinear_forward(scheme, _dev(x, torch.bfloat16, "x"), _dev(wq, torch.uint8, "wq"),
                                 _dev(sw, torch.float32, "sw"), M, N, K,
                                 _dev(y, torch.bfloat16, "y"), wp, wn, _stream(stream)),
           "qlinear_forward")
    return y


def device_status(stream=None) -> tuple[int, int]:
    """Synchronise and read (then clear) the device status word: (status, detail)."""
    d = ctypes.c_uint32(0)
    s = lib().qlinear_get_device_status(_stream(stream), ctypes.byref(d))
    return int(s), int(d.value)
