"""Seeded synthetic inputs for the MiniKV hot path.

This module draws random numbers and nothing else: it holds none of the
method's arithmetic, so both the CUDA path and the CPU oracle may take their
inputs from it.

Recipe (shapes of the LLaMA2-7B/13B and Mistral-7B models that the MiniKV
LongBench table evaluates; LongBench itself is not used):
  * q, K, V ~ N(0, 1), drawn in fp32 and rounded to fp16;
  * the first ``OUTLIER_CHANNELS`` channels of every KV head's keys are scaled
    by ``OUTLIER_SCALE`` in fp32 before rounding (the per-channel key outliers
    that make sub-channel key quantization worthwhile);
  * every tensor slice has its own seed, a fixed function of
    (workload id, layer, tensor id, step, batch row), so any slice can be drawn
    again on its own.
"""
from __future__ import annotations

import torch

OUTLIER_CHANNELS = 4
OUTLIER_SCALE = 10.0

# tensor ids inside a seed
T_Q, T_K, T_V, T_QDEC, T_KNEW, T_VNEW = 1, 2, 3, 4, 5, 6


def seed_of(workload: int, layer: int, tensor: int, step: int = 0, b: int = 0) -> int:
    """Deterministic 63-bit seed for one slice."""
    s = workload
    for part, mult in ((layer, 1009), (tensor, 101), (step, 1_000_003), (b, 65_537)):
        s = (s * mult + part + 1) % (2 ** 61 - 1)
    return s


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def normal_fp16(shape, seed: int, device="cpu") -> torch.Tensor:
    """N(0,1) drawn in fp32, rounded to fp16."""
    x = torch.randn(shape, generator=_gen(seed, device), device=device, dtype=torch.float32)
    return x.to(torch.float16)


def keys_fp16(shape, seed: int, device="cpu") -> torch.Tensor:
    """Keys [..., D]: N(0,1) with the first OUTLIER_CHANNELS channels x OUTLIER_SCALE (fp32), then fp16."""
    x = torch.randn(shape, generator=_gen(seed, device), device=device, dtype=torch.float32)
    x[..., :OUTLIER_CHANNELS] *= OUTLIER_SCALE
    return x.to(torch.float16)
