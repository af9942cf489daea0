"""Seeded synthetic inputs shaped like Llama-3.1-8B and Qwen3-8B projections.

This module only draws random numbers and rounds them to bf16 storage; it
holds none of the quantized-linear arithmetic, so both the CUDA path and the
CPU oracle can take their inputs from it without sharing any computation.

Recipe (stand-ins for the checkpoints and prompts the model pages use, none
of which exist here):

* X ~ N(0, 1) per element, with ``outliers`` channels (the first entries of a
  seeded permutation of [0, K)) multiplied by 20 for every token.
* W ~ N(0, 0.02) per element.
* Each tensor has its own stream, derived from (seed, tag), so any tensor can
  be regenerated alone.
* Values are drawn in f32 (numpy's PCG64 normal sampler) and rounded to bf16
  by torch's round-to-nearest-even conversion; tensors are returned as uint16
  bit patterns (the bf16 storage).
"""
from __future__ import annotations

import zlib

import numpy as np
import torch

OUTLIER_GAIN = 20.0
WEIGHT_STD = 0.02

# (name, N = output features, K = input features), nn.Linear [out, in] layout.
LLAMA31_8B = (
    ("q_proj", 4096, 4096),
    ("k_proj", 1024, 4096),
    ("v_proj", 1024, 4096),
    ("o_proj", 4096, 4096),
    ("gate_proj", 14336, 4096),
    ("up_proj", 14336, 4096),
    ("down_proj", 4096, 14336),
)
QWEN3_8B = (
    ("q_proj", 4096, 4096),
    ("k_proj", 1024, 4096),
    ("v_proj", 1024, 4096),
    ("o_proj", 4096, 4096),
    ("gate_proj", 12288, 4096),
    ("up_proj", 12288, 4096),
    ("down_proj", 4096, 12288),
)
LLAMA31_8B_PREFILL = (
    ("gate_proj", 14336, 4096),
    ("up_proj", 14336, 4096),
    ("down_proj", 4096, 14336),
    ("qkv_proj", 6144, 4096),
)
# The same layer with the projections that read one input stored side by side
# along N (q|k|v and gate|up, the serving layout): four products instead of seven.
LLAMA31_8B_FUSED = (
    ("qkv_proj", 6144, 4096),
    ("o_proj", 4096, 4096),
    ("gate_up_proj", 28672, 4096),
    ("down_proj", 4096, 14336),
)


def outlier_count(K: int, fraction: float = 0.01) -> int:
    """1% of the input channels, rounded (41 for K=4096, 143 for K=14336)."""
    return int(round(fraction * K))


def _rng(seed: int, tag: str) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, zlib.crc32(tag.encode())])))


def _to_bf16_bits(a: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def make_x(M: int, K: int, seed: int = 0, tag: str = "X", outliers: int = 0,
           std: float = 1.0) -> np.ndarray:
    """Activations [M, K] as bf16 bits: N(0, std) with ``outliers`` channels x20."""
    g = _rng(seed, f"{tag}:{M}x{K}")
    x = g.standard_normal((M, K), dtype=np.float32) * np.float32(std)
    if outliers:
        cols = g.permutation(K)[:outliers]
        x[:, cols] *= np.float32(OUTLIER_GAIN)
    return _to_bf16_bits(x)


def outlier_channels(M: int, K: int, seed: int = 0, tag: str = "X", outliers: int = 0) -> np.ndarray:
    """The channel indices ``make_x`` scales, for tests that check them."""
    g = _rng(seed, f"{tag}:{M}x{K}")
    g.standard_normal((M, K), dtype=np.float32)
    return np.sort(g.permutation(K)[:outliers])


def make_w(N: int, K: int, seed: int = 0, tag: str = "W", std: float = WEIGHT_STD) -> np.ndarray:
    """Weights [N, K] as bf16 bits: N(0, std)."""
    g = _rng(seed, f"{tag}:{N}x{K}")
    return _to_bf16_bits(g.standard_normal((N, K), dtype=np.float32) * np.float32(std))


def make_uniform_bits(n: int, seed: int = 0, tag: str = "bits") -> np.ndarray:
    """n uniformly random 32-bit patterns (for codec sweeps)."""
    return _rng(seed, tag).integers(0, 2**32, size=n, dtype=np.uint64).astype(np.uint32)


def _torch_gen(seed: int, tag: str, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(np.random.SeedSequence([seed, zlib.crc32(tag.encode())]).generate_state(1)[0]))
    return g


def make_x_device(M: int, K: int, seed: int = 0, tag: str = "X", outliers: int = 0,
                  device="cuda") -> torch.Tensor:
    """Same recipe as ``make_x`` drawn by torch's generator on ``device`` (for
    large benchmark inputs); returns a bf16 tensor."""
    g = _torch_gen(seed, f"{tag}:{M}x{K}", device)
    x = torch.randn((M, K), generator=g, device=device, dtype=torch.float32)
    if outliers:
        cols = torch.randperm(K, generator=g, device=device)[:outliers]
        x[:, cols] *= OUTLIER_GAIN
    return x.to(torch.bfloat16)


def make_w_device(N: int, K: int, seed: int = 0, tag: str = "W", std: float = WEIGHT_STD,
                  device="cuda") -> torch.Tensor:
    """Same recipe as ``make_w`` drawn by torch's generator on ``device``."""
    g = _torch_gen(seed, f"{tag}:{N}x{K}", device)
    return (torch.randn((N, K), generator=g, device=device, dtype=torch.float32) * std).to(torch.bfloat16)
