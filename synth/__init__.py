"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle side.

This module holds no arithmetic of the quantized linear: it only draws numbers.
Both the CUDA path and the CPU oracle receive the same bf16 bytes from here.

Recipe (stated once, used everywhere):
  * values: numpy ``PCG64(seed)`` standard normals in float32, times ``std``;
  * outliers: a Bernoulli(``outlier_p``) mask drawn from the same generator
    multiplies the chosen entries by ``outlier_factor``;
  * the float32 values are rounded to bf16 (round-to-nearest-even) by torch.
  * tensor seeds: workload seed + {A: 0, W: 1, bias: 2, W2: 3, A2: 4}.

The workloads are the transformer linears of a rectified-flow image model
("FLUX 3 Image Klein" release notes: width and height are multiples of 16, so a
1 MP image has 4096 latent tokens and a 4096x4096 image has 65536) at hidden
size 3072 and MLP width 12288.  No trained weights exist here, so
N(0, 0.02)-style weights and N(0, 1) activations with sparse outliers stand in.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

SEED_OFFSET = {"A": 0, "W": 1, "bias": 2, "W2": 3, "A2": 4}


def bf16_normal(shape, std: float, seed: int, outlier_p: float = 0.0,
                outlier_factor: float = 1.0) -> torch.Tensor:
    """bf16 CPU tensor of N(0, std^2) draws with optional sparse outliers."""
    rng = np.random.Generator(np.random.PCG64(seed))
    v = rng.standard_normal(size=shape, dtype=np.float32)
    v *= np.float32(std)
    if outlier_p > 0.0:
        mask = rng.random(size=shape, dtype=np.float32) < np.float32(outlier_p)
        v[mask] *= np.float32(outlier_factor)
    return torch.from_numpy(v).to(torch.bfloat16)


def uniform_u8(n: int, seed: int) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64(seed))
    return rng.integers(0, 256, size=n, dtype=np.uint8)


@dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    M: int
    K: int
    N: int
    a_std: float = 1.0
    w_std: float = 0.02
    outlier_p: float = 0.0
    outlier_factor: float = 1.0
    bias: bool = False
    scheme: str = "nvfp4"
    # second GEMM of an MLP pair (config "mlp"): A2 [M, N] x W2 [K, N]
    n2: int = 0
    a2_std: float = 0.5
    w2_std: float = 0.01
    extra: dict = field(default_factory=dict)

    def A(self) -> torch.Tensor:
        return bf16_normal((self.M, self.K), self.a_std, self.seed + SEED_OFFSET["A"],
                           self.outlier_p, self.outlier_factor)

    def W(self) -> torch.Tensor:
        return bf16_normal((self.N, self.K), self.w_std, self.seed + SEED_OFFSET["W"])

    def bias_vec(self) -> torch.Tensor | None:
        if not self.bias:
            return None
        return bf16_normal((self.N,), 0.1, self.seed + SEED_OFFSET["bias"])

    def W2(self) -> torch.Tensor:
        return bf16_normal((self.K, self.N), self.w2_std, self.seed + SEED_OFFSET["W2"])

    def A2(self) -> torch.Tensor:
        return bf16_normal((self.M, self.N), self.a2_std, self.seed + SEED_OFFSET["A2"])

    def A_rows(self, M: int) -> torch.Tensor:
        """Activation of another token count with this workload's recipe."""
        return bf16_normal((M, self.K), self.a_std, self.seed + SEED_OFFSET["A"],
                           self.outlier_p, self.outlier_factor)


WORKLOADS = {
    # 128x256 activations (1 % outliers x20) against a 256x256 weight
    "nvfp4_tiny": Workload("nvfp4_tiny", 0, M=128, K=256, N=256, outlier_p=0.01,
                           outlier_factor=20.0),
    # attention projection at 1 MP: 4096 tokens, 3072 -> 3072, with bias
    "nvfp4_attn_1mp": Workload("nvfp4_attn_1mp", 10, M=4096, K=3072, N=3072,
                               outlier_p=0.005, outlier_factor=30.0, bias=True),
    # MLP up (3072 -> 12288) then down (12288 -> 3072) at 1 MP
    "nvfp4_mlp_1mp": Workload("nvfp4_mlp_1mp", 20, M=4096, K=3072, N=12288,
                              outlier_p=0.005, outlier_factor=30.0),
    # per-row FP8 at 1 MP (plus an M sweep of 256, 1024, 16384)
    "fp8r_1mp": Workload("fp8r_1mp", 30, M=4096, K=3072, N=3072, scheme="fp8r"),
    # 4K output: 65536 tokens; projections 3072 -> 3072 and 3072 -> 12288
    "nvfp4_4k": Workload("nvfp4_4k", 40, M=65536, K=3072, N=3072, outlier_p=0.005,
                         outlier_factor=30.0),
    "nvfp4_4k_up": Workload("nvfp4_4k_up", 40, M=65536, K=3072, N=12288,
                            outlier_p=0.005, outlier_factor=30.0),
}

FP8R_M_SWEEP = (256, 1024, 4096, 16384)
