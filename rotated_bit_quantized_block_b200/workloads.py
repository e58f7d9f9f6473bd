"""Seeded synthetic workloads for the ConvRot linear.

This module only draws inputs; it holds none of the method's arithmetic, so both
the CUDA path and the CPU oracle can be fed from it.  The shapes stand in for the
transformer linears the source pages quantize (SAM 3.1 image encoder, TRELLIS.2
diffusion transformer): activations are N(0, 1) with a few "outlier channels"
(input columns scaled by a large factor, the case ConvRot's rotation exists to
spread), weights are N(0, sigma).  Values are drawn in float32 with
``torch.Generator('cpu').manual_seed(seed)`` and rounded to fp16.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch


@dataclass(frozen=True)
class Linear:
    name: str
    K: int  # in-features (reduction dimension)
    N: int  # out-features
    bits: int = 0  # 8 or 4 for this linear; 0 = the workload's width


@dataclass(frozen=True)
class Workload:
    name: str
    M: int
    linears: tuple
    bits: int
    block: int
    outlier_frac: float
    outlier_factor: float
    w_sigma: float
    seed: int
    description: str = field(default="", compare=False)

    def bits_of(self, lin: Linear) -> int:
        """Code width of one linear (per-layer choice, else the workload's)."""
        return lin.bits or self.bits

    def ops(self) -> int:
        """Integer multiply-adds x2 of one pass over every linear."""
        return sum(2 * self.M * l.K * l.N for l in self.linears)


VIT_L_LINEARS = (Linear("qkv", 1024, 3072), Linear("proj", 1024, 1024),
                 Linear("fc1", 1024, 4096), Linear("fc2", 4096, 1024))
DIT_LINEARS = (Linear("qkv", 1536, 4608), Linear("fc1", 1536, 6144), Linear("fc2", 6144, 1536))

WORKLOADS = {
    "tiny_w8a8": Workload("tiny_w8a8", 64, (Linear("tiny", 256, 256),), 8, 64, 0.02, 20.0, 0.02, 0,
                          "X 64x256, W 256x256, block 64"),
    "vit_l_w8a8": Workload("vit_l_w8a8", 5184, VIT_L_LINEARS, 8, 128, 0.01, 30.0, 0.02, 1,
                           "ViT-L encoder linears, 72x72 patches"),
    "vit_l_w4a4": Workload("vit_l_w4a4", 5184, VIT_L_LINEARS, 4, 128, 0.01, 30.0, 0.02, 2,
                           "ViT-L encoder linears, W4A4"),
    "dit_w8a8": Workload("dit_w8a8", 8192, DIT_LINEARS, 8, 128, 0.005, 50.0, 0.015, 3,
                         "DiT linears, batch 2 x 4096 tokens"),
    # per-layer code width: attention linears W8A8, MLP linears W4A4
    "vit_l_mixed": Workload("vit_l_mixed", 5184,
                            (Linear("qkv", 1024, 3072, 8), Linear("proj", 1024, 1024, 8),
                             Linear("fc1", 1024, 4096, 4), Linear("fc2", 4096, 1024, 4)),
                            8, 128, 0.01, 30.0, 0.02, 5, "ViT-L encoder linears, W8A8 attention, W4A4 MLP"),
}
MSWEEP_M = (1, 16, 128, 1024, 4096, 16384)


def msweep(M: int) -> Workload:
    return Workload(f"msweep_w8a8_M{M}", M, (Linear("sq4096", 4096, 4096),), 8, 128, 0.01, 30.0,
                    0.01, 4, "M sweep at K=N=4096")


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def activations(M: int, K: int, outlier_frac: float, outlier_factor: float, seed: int) -> np.ndarray:
    """X (M x K fp16): N(0,1) with ceil(frac*K) distinct columns scaled by ``factor``."""
    g = _gen(seed)
    x = torch.randn(M, K, generator=g, dtype=torch.float32)
    n_out = int(math.ceil(outlier_frac * K))
    if n_out:
        cols = torch.randperm(K, generator=g)[:n_out]
        x[:, cols] *= outlier_factor
    return x.to(torch.float16).numpy()


def weight(N: int, K: int, sigma: float, seed: int) -> np.ndarray:
    """W (N x K fp16) ~ N(0, sigma)."""
    g = _gen(seed)
    return (torch.randn(N, K, generator=g, dtype=torch.float32) * sigma).to(torch.float16).numpy()


def bias(N: int, seed: int, sigma: float = 0.02) -> np.ndarray:
    g = _gen(seed)
    return (torch.randn(N, generator=g, dtype=torch.float32) * sigma).to(torch.float16).numpy()


def linear_inputs(w: Workload, idx: int, M: int | None = None, with_bias: bool = False, replica: int = 0):
    """(X, W, bias-or-None) for linear ``idx`` of workload ``w``.

    ``replica`` selects an independent draw of the same shapes (used for
    rotating buffer sets and for per-rank batches).
    """
    lin = w.linears[idx]
    M = w.M if M is None else M
    base = w.seed * 1_000_003 + idx * 1009 + replica * 7919
    X = activations(M, lin.K, w.outlier_frac, w.outlier_factor, base + 1)
    W = weight(lin.N, lin.K, w.w_sigma, base + 2)
    b = bias(lin.N, base + 3) if with_bias else None
    return X, W, b
