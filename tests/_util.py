"""Helpers shared by the GPU parity tests (marshalling and the tolerance only)."""
import numpy as np
import torch

import oracle

# bf16 outputs of fp32-accumulated products: |y_gpu - y_oracle| <= 2^-7 |y_oracle| + 1e-3
REL_TOL = 2.0 ** -7
ABS_TOL = 1e-3


def bf16_dev(bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits, np.uint16).view(np.int16)).to(device).view(torch.bfloat16)


def u8_dev(a: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, np.uint8)).to(device)


def f32_dev(a: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(device)


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> uint16 bit patterns (host)."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def assert_y_close(y_gpu_bits: np.ndarray, y_ref_bits: np.ndarray, what=""):
    g = oracle.bf16_bits_to_f64(y_gpu_bits)
    r = oracle.bf16_bits_to_f64(y_ref_bits)
    err = np.abs(g - r)
    lim = REL_TOL * np.abs(r) + ABS_TOL
    bad = np.nonzero(err > lim)
    assert bad[0].size == 0, (f"{what}: {bad[0].size} outputs out of tolerance; first "
                              f"{[(tuple(int(i) for i in idx), g[idx], r[idx]) for idx in zip(*bad)][:5]}")
    return float(err.max()) if err.size else 0.0


def oracle_forward_par(scheme: int, x: np.ndarray, wq: np.ndarray, sw: np.ndarray, chunks: int = 0):
    """oracle.forward split over output-row ranges on threads (the oracle's C
    calls release the GIL), for full-size layers.  Block-scheme ranges are
    whole 128-row blocks.  The same values as oracle.forward."""
    import concurrent.futures
    import os
    qx, sx = oracle.quantize_act(scheme, x)
    N = wq.shape[0]
    chunks = chunks or min(32, os.cpu_count() or 4)
    step = -(-N // chunks)
    if scheme == oracle.FP8_BLOCK:
        step = -(-step // 128) * 128
    bounds = [(n0, min(N, n0 + step)) for n0 in range(0, N, step)]
    with concurrent.futures.ThreadPoolExecutor(max_workers=len(bounds)) as ex:
        parts = list(ex.map(lambda b: oracle.linear_rows(scheme, qx, sx, wq, sw, b[0], b[1]), bounds))
    return np.concatenate(parts, axis=1)


def oracle_wo_par(scheme: int, x: np.ndarray, wq: np.ndarray, sw: np.ndarray, chunks: int = 0):
    """oracle.linear_weight_only split over output-row ranges on threads."""
    import concurrent.futures
    import os
    N = wq.shape[0]
    chunks = chunks or min(32, os.cpu_count() or 4)
    step = -(-N // chunks)
    if scheme == oracle.FP8_BLOCK:
        step = -(-step // 128) * 128
    bounds = [(n0, min(N, n0 + step)) for n0 in range(0, N, step)]
    with concurrent.futures.ThreadPoolExecutor(max_workers=len(bounds)) as ex:
        parts = list(ex.map(lambda b: oracle.linear_weight_only(scheme, x, wq, sw, b[0], b[1]), bounds))
    return np.concatenate(parts, axis=1)
