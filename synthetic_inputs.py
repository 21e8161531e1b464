"""Seeded synthetic inputs shared by the CPU oracle and the CUDA path.

This module holds random-number recipes only (no quantization arithmetic):
both sides consume the identical bf16 bytes it produces.  There is no
dataset or checkpoint here; the shapes stand in for the Qwen2.5-VL-7B
language backbone projections named in the workload list, and the value
distributions are the stated synthetic ones:

* tiny:   X [16, 256] ~ N(0, 1) with channels 5 and 133 scaled x20,
          W [128, 256] ~ N(0, 0.02^2), seed 0.
* prefill / decode projections (qkv 3584->4608, o 3584->3584,
  gate_up 3584->37888, down 18944->3584, seeds 1..4):
          c_k = exp(N(0, 1)) per input channel, X = bf16(N(0, 1) * c),
          W = bf16(N(0, 1) / sqrt(K)).
* fused-prologue path: gain ~ U(0.5, 1.5), residual R ~ N(0, 1) [M, N]
  drawn from seed + 100.
* 28-layer stack: 7 unfused projections per layer, seed 1000 + 7 l + p.

Every tensor has its own generator (seed * 16 + stream id), so the weights
of a projection do not depend on M and decode / prefill share weights.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch

# name -> (K, N, seed)
PROJECTIONS = {
    "qkv": (3584, 4608, 1),
    "o": (3584, 3584, 2),
    "gate_up": (3584, 37888, 3),
    "down": (18944, 3584, 4),
}

# 28-layer stack: 7 unfused projections (K, N)
STACK_PROJECTIONS = [
    ("q", 3584, 3584),
    ("k", 3584, 512),
    ("v", 3584, 512),
    ("o", 3584, 3584),
    ("gate", 3584, 18944),
    ("up", 3584, 18944),
    ("down", 18944, 3584),
]
STACK_LAYERS = 28

_S_CHAN, _S_X, _S_W, _S_GAMMA, _S_RES = 0, 1, 2, 3, 4


def _gen(seed: int, stream: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed * 16 + stream)
    return g


def to_bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> numpy uint16 bit patterns (no copy of values)."""
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def tiny_inputs(seed: int = 0):
    """X [16, 256] with two x20 outlier channels, W [128, 256] ~ N(0, 0.02^2)."""
    gx = _gen(seed, _S_X)
    X = torch.randn(16, 256, generator=gx, dtype=torch.float32)
    X[:, 5] *= 20.0
    X[:, 133] *= 20.0
    gw = _gen(seed, _S_W)
    W = torch.randn(128, 256, generator=gw, dtype=torch.float32) * 0.02
    return X.to(torch.bfloat16), W.to(torch.bfloat16)


def projection_activations(K: int, M: int, seed: int) -> torch.Tensor:
    """X = bf16(N(0,1) * c), c_k = exp(N(0,1)) per channel; [M, K]."""
    c = torch.exp(torch.randn(K, generator=_gen(seed, _S_CHAN), dtype=torch.float32))
    X = torch.randn(M, K, generator=_gen(seed, _S_X), dtype=torch.float32) * c
    return X.to(torch.bfloat16)


def projection_weight(K: int, N: int, seed: int) -> torch.Tensor:
    """W = bf16(N(0,1) / sqrt(K)); [N, K]."""
    W = torch.randn(N, K, generator=_gen(seed, _S_W), dtype=torch.float32)
    W.mul_(1.0 / math.sqrt(K))
    return W.to(torch.bfloat16)


def norm_gain(K: int, seed: int) -> torch.Tensor:
    """gamma ~ U(0.5, 1.5), bf16 [K]."""
    u = torch.rand(K, generator=_gen(seed, _S_GAMMA), dtype=torch.float32)
    return (0.5 + u).to(torch.bfloat16)


def residual(M: int, N: int, seed: int) -> torch.Tensor:
    """R ~ N(0, 1), bf16 [M, N], drawn from seed + 100."""
    return torch.randn(M, N, generator=_gen(seed + 100, _S_RES), dtype=torch.float32).to(torch.bfloat16)


@dataclass
class FusedCase:
    """One projection of the fused-prologue workload."""
    name: str
    K: int
    N: int
    seed: int
    rmsnorm: bool      # RMSNorm(gain) before the rotation (qkv, gate_up)
    residual: bool     # residual add in the epilogue (o, down)


FUSED_CASES = [
    FusedCase("qkv", 3584, 4608, 1, True, False),
    FusedCase("o", 3584, 3584, 2, False, True),
    FusedCase("gate_up", 3584, 37888, 3, True, False),
    FusedCase("down", 18944, 3584, 4, False, True),
]


def stack_seed(layer: int, proj: int) -> int:
    return 1000 + 7 * layer + proj
