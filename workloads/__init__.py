"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module only draws numbers: it holds no quantization or matrix-product
arithmetic.  Every tensor comes from numpy's PCG64 generator seeded from a
fixed tuple (the workload's base seed, a tag and the shape), is drawn in
float32, and is then rounded to its storage dtype by torch (round to nearest
even).  Nothing here touches a GPU.

Workloads (shapes of the 7B / 70B LLaMA-style layers the quantization write-ups
use as examples):

* tiny      -- W fp32 [256, 512] ~ N(0, 0.02) with 4 random input columns x20;
               INT4 asymmetric g=128; X bf16 [1, 512] ~ N(0, 1).
* 7b-decode -- W bf16 [4096,4096], [11008,4096], [4096,11008] ~ N(0, 0.02) with
               0.1% of input columns x30; INT4 symmetric g=128; X bf16 [M, K]
               ~ N(0, 1), M in {1, 4, 16}.
* 70b-decode-- W bf16 [28672,8192], [8192,28672] ~ N(0, 0.015) with 0.1% of
               input columns x50; INT4 asymmetric g=128 (fp16 scale and zero);
               X bf16 M in {1, 8, 16}.
* prefill   -- W bf16 [11008, 4096] ~ N(0, 0.02), INT4 symmetric g=128;
               X bf16 [2048, 4096] ~ N(0, 1) with 6 fixed hidden dims whose
               entries are +-U(50, 100) (systematic activation outliers).
* w8a8      -- W bf16 [4096, 4096] ~ N(0, 0.02) -> int8 per output channel;
               X bf16 [4096, 4096] ~ N(0, 1) with the same 6-dim outlier rule ->
               int8 per token.

The outlier column count for weights is round(0.001 * K) (at least 1); the
columns are drawn without replacement after the Gaussian matrix.
"""
from dataclasses import dataclass, field
from typing import List, Optional, Tuple

import numpy as np
import torch

_TAGS = {"w": 1, "x": 2}


def _rng(seed: int, tag: str, *shape: int) -> np.random.Generator:
    ss = np.random.SeedSequence([int(seed), _TAGS[tag], *[int(s) for s in shape]])
    return np.random.Generator(np.random.PCG64(ss))


def make_weight(N: int, K: int, sigma: float, seed: int,
                outlier_frac: float = 0.0, outlier_scale: float = 1.0,
                dtype: torch.dtype = torch.bfloat16) -> torch.Tensor:
    """Gaussian weight [N, K] with a few scaled input columns (CPU tensor)."""
    rng = _rng(seed, "w", N, K)
    W = rng.standard_normal((N, K), dtype=np.float32)
    W *= np.float32(sigma)
    if outlier_frac > 0.0:
        count = max(1, int(round(outlier_frac * K)))
        cols = rng.choice(K, size=count, replace=False)
        W[:, cols] *= np.float32(outlier_scale)
    t = torch.from_numpy(W)
    return t if dtype == torch.float32 else t.to(dtype)


def make_activation(M: int, K: int, seed: int, outlier_dims: int = 0,
                    lo: float = 50.0, hi: float = 100.0,
                    dtype: torch.dtype = torch.bfloat16) -> torch.Tensor:
    """Gaussian activation [M, K]; `outlier_dims` fixed hidden dims are
    replaced by +-U(lo, hi) with a random sign (CPU tensor)."""
    rng = _rng(seed, "x", M, K)
    X = rng.standard_normal((M, K), dtype=np.float32)
    if outlier_dims > 0:
        dims = rng.choice(K, size=outlier_dims, replace=False)
        mag = rng.uniform(lo, hi, size=(M, outlier_dims)).astype(np.float32)
        sign = np.where(rng.random((M, outlier_dims)) < 0.5, -1.0, 1.0).astype(np.float32)
        X[:, dims] = mag * sign
    return torch.from_numpy(X).to(dtype)


@dataclass
class Workload:
    name: str
    shapes: List[Tuple[int, int]]          # weight shapes [N, K]
    ms: List[int]                          # activation rows M
    sigma: float
    outlier_frac: float
    outlier_scale: float
    sym: bool
    seed: int
    w_dtype: torch.dtype = torch.bfloat16
    act_outlier_dims: int = 0
    bits: int = 4
    group_size: int = 128
    notes: str = ""

    def weight(self, i: int) -> torch.Tensor:
        N, K = self.shapes[i]
        return make_weight(N, K, self.sigma, self.seed + 100 * i,
                           self.outlier_frac, self.outlier_scale, self.w_dtype)

    def activation(self, M: int, K: int) -> torch.Tensor:
        return make_activation(M, K, self.seed + 1, self.act_outlier_dims)


WORKLOADS = {
    "tiny": Workload("tiny", [(256, 512)], [1], 0.02, 4 / 512, 20.0, sym=False,
                     seed=1, w_dtype=torch.float32),
    "7b-decode": Workload("7b-decode", [(4096, 4096), (11008, 4096), (4096, 11008)],
                          [1, 4, 16], 0.02, 0.001, 30.0, sym=True, seed=7),
    "70b-decode": Workload("70b-decode", [(28672, 8192), (8192, 28672)], [1, 8, 16],
                           0.015, 0.001, 50.0, sym=False, seed=70),
    "prefill": Workload("prefill", [(11008, 4096)], [2048], 0.02, 0.0, 1.0, sym=True,
                        seed=2048, act_outlier_dims=6),
    "w8a8": Workload("w8a8", [(4096, 4096)], [4096], 0.02, 0.0, 1.0, sym=True,
                     seed=88, act_outlier_dims=6, bits=8),
}


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """uint16 bit pattern of a bf16 CPU tensor (for the oracle's C interface)."""
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)
