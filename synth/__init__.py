"""Seeded synthetic workloads for the NF4 codec and the QLoRA linear layer.

This module only draws random numbers and casts them to bfloat16; it holds none of the
method's arithmetic.  Both the oracle-side tests and the CUDA-side tests / benchmark
take their inputs from here, so both see identical bf16 bits.

Draws use numpy's PCG64 generator seeded per tensor (``seed_for``), in float32, scaled,
then rounded to bfloat16 by torch's nearest-even cast.  ``device="cuda"`` instead draws
with torch's CUDA generator (a different stream of numbers, used only where no oracle
comparison needs the same values, e.g. timing runs).

Workloads (shapes are the LLaMA-style linears named beside each):

1. ``single``  W 1024x1024 ~ N(0, 0.02^2), seed 0; x 128x1024 ~ N(0,1); r=16, alpha=16
   (s = 1); A ~ N(0, 1/r); B ~ N(0, 0.01^2).
2. ``llama7b_512``  seven linears of a LLaMA-7B block (q,k,v,o 4096x4096; gate,up
   11008x4096; down 4096x11008), 512 tokens, r=64, alpha=16.
3. ``llama13b_8192``  seven linears of a LLaMA-13B block (q,k,v,o 5120x5120; gate,up
   13824x5120; down 5120x13824), 8192 tokens, r=64, alpha=16.
4. ``stack65b``  80 layers x (4 x 8192x8192, 3 x 22016x8192), W ~ N(0, 0.015^2), drawn
   per layer (codec only).
5. ``robust``  W 4000x3000, Student-t(3) scaled to std 0.02, 1% of the input columns
   multiplied by 20, then 5% of entries set to exactly zero; r in {8, 64, 256};
   M in {1, 16, 512, 16384}.

For every linear set, A ~ N(0, 1/r), B ~ N(0, 0.01^2), x and dY ~ N(0, 1).
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch


@dataclass(frozen=True)
class Linear:
    name: str
    N: int      # out features
    K: int      # in features


LLAMA7B = (Linear("q", 4096, 4096), Linear("k", 4096, 4096), Linear("v", 4096, 4096),
           Linear("o", 4096, 4096), Linear("gate", 11008, 4096), Linear("up", 11008, 4096),
           Linear("down", 4096, 11008))
LLAMA13B = (Linear("q", 5120, 5120), Linear("k", 5120, 5120), Linear("v", 5120, 5120),
            Linear("o", 5120, 5120), Linear("gate", 13824, 5120), Linear("up", 13824, 5120),
            Linear("down", 5120, 13824))
STACK65B_LAYER = (Linear("q", 8192, 8192), Linear("k", 8192, 8192), Linear("v", 8192, 8192),
                  Linear("o", 8192, 8192), Linear("gate", 22016, 8192), Linear("up", 22016, 8192),
                  Linear("down", 8192, 22016))

WORKLOADS = {
    "single": {"linears": (Linear("w", 1024, 1024),), "M": 128, "r": 16, "alpha": 16.0,
               "w_std": 0.02, "config": 1},
    "llama7b_512": {"linears": LLAMA7B, "M": 512, "r": 64, "alpha": 16.0, "w_std": 0.02,
                    "config": 2},
    "llama13b_8192": {"linears": LLAMA13B, "M": 8192, "r": 64, "alpha": 16.0, "w_std": 0.02,
                      "config": 3},
    "stack65b": {"linears": STACK65B_LAYER, "layers": 80, "w_std": 0.015, "config": 4},
    "robust": {"linears": (Linear("w", 4000, 3000),), "Ms": (1, 16, 512, 16384),
               "rs": (8, 64, 256), "alpha": 16.0, "w_std": 0.02, "config": 5},
}


def seed_for(config: int, tensor_index: int) -> int:
    """Per-tensor seed: 0 for the single-weight workload's weight, else 1000*config + index."""
    if config == 1 and tensor_index == 0:
        return 0
    return 1000 * config + tensor_index


def _to_bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def normal_bf16(shape, std: float, seed: int, device: str = "cpu") -> torch.Tensor:
    """N(0, std^2) draws rounded to bf16."""
    if device != "cpu":
        g = torch.Generator(device=device)
        g.manual_seed(seed)
        return (torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std).to(torch.bfloat16)
    rng = np.random.default_rng(seed)
    return _to_bf16(rng.standard_normal(size=shape, dtype=np.float32) * np.float32(std))


def robust_weight_bf16(N: int, K: int, seed: int, std: float = 0.02,
                       outlier_frac: float = 0.01, outlier_gain: float = 20.0,
                       zero_frac: float = 0.05) -> torch.Tensor:
    """Student-t(3) weights scaled to std ``std``; ``outlier_frac`` of the input columns
    scaled by ``outlier_gain``; then a Bernoulli(``zero_frac``) mask of exact zeros."""
    rng = np.random.default_rng(seed)
    w = rng.standard_t(3, size=(N, K)).astype(np.float32) * np.float32(std / math.sqrt(3.0))
    n_out = max(1, int(round(outlier_frac * K)))
    cols = rng.choice(K, size=n_out, replace=False)
    w[:, cols] *= np.float32(outlier_gain)
    w[rng.random(size=(N, K)) < zero_frac] = 0.0
    return _to_bf16(w)


def linear_inputs(M: int, N: int, K: int, r: int, seed: int, device: str = "cpu") -> dict:
    """x, dY ~ N(0,1), A ~ N(0, 1/r), B ~ N(0, 0.01^2), all bf16, from four sub-seeds."""
    return {
        "x": normal_bf16((M, K), 1.0, seed * 16 + 1, device),
        "A": normal_bf16((r, K), 1.0 / math.sqrt(r), seed * 16 + 2, device),
        "B": normal_bf16((N, r), 0.01, seed * 16 + 3, device),
        "dY": normal_bf16((M, N), 1.0, seed * 16 + 4, device),
    }


def bf16_to_f32_numpy(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> float32 numpy array holding the same (exact) values."""
    return t.detach().to("cpu").float().numpy()


def bf16_bits_numpy(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> its 16-bit patterns as a uint16 numpy array."""
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)
