"""Seeded synthetic workloads for the SS1 layer: shapes, value distributions and generators.

This module holds no arithmetic of the layer itself -- only the layer shapes taken from the
workloads the SS1 paper summary reports on ("SS1: Accelerating Inference with Fast and
Expressive Sketch Structured Transform", section "Key results" / "Measured effects": GPT-2
Small and Large, Llama-3-8B projections, the DLRM MLPerf top MLP) and seeded random inputs
of those shapes. Both the CUDA path's tests/benchmark and the CPU oracle's tests draw
their inputs from here; nothing here calls either implementation.

Generation recipe: one torch CPU generator per layer instance, seeded with
`instance_seed(layer)`; X is drawn first, then the outlier rows (if any), then Wc, all in
float32; bf16 layers are rounded with `.to(torch.bfloat16)` (round to nearest even). The
hash tables use the workload's seed as given.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, replace
from typing import Dict, List, Tuple

import torch


@dataclass(frozen=True)
class Layer:
    """One SS1 layer instance: Y[M, N] = SS1(X[M, K]) with compressed weights Wc[N, K/c]."""
    workload: str
    M: int
    K: int
    N: int
    c: int
    BK: int
    BN: int
    dtype: str            # "bf16" or "fp32": dtype of X, Wc and Y (accumulation is fp32)
    x_dist: str           # "normal", "normal_outliers", "uniform_pm1"
    w_dist: str           # "uniform_invsqrtk", "normal_002"
    seed: int             # table seed (and base of the input seed)

    @property
    def Kc(self) -> int:
        return self.K // self.c

    @property
    def NB(self) -> int:
        return self.N // self.BN

    @property
    def tag(self) -> str:
        return f"{self.workload}:M{self.M}:K{self.K}:N{self.N}:c{self.c}"

    def with_M(self, M: int) -> "Layer":
        return replace(self, M=M)


def instance_seed(layer: Layer) -> int:
    """Seed of the input generator of one layer instance (independent per shape, c and M)."""
    return (layer.seed * 1_000_003 + layer.K * 7919 + layer.N * 104_729 + layer.c * 131 + layer.M) % (1 << 62)


def _workloads() -> Dict[int, List[Layer]]:
    w: Dict[int, List[Layer]] = {}
    # 1: single fp32 layer
    w[1] = [Layer("fp32-single", 64, 768, 768, 2, 64, 64, "fp32", "normal", "uniform_invsqrtk", 0)]
    # 2: GPT-2 Small shaped (qkv, attn proj, fc, fc proj), batch 8 x seq 1024
    w[2] = [Layer("gpt2-small", 8192, K, N, 2, 128, 128, "bf16", "normal", "uniform_invsqrtk", 1)
            for K, N in [(768, 2304), (768, 768), (768, 3072), (3072, 768)]]
    # 3: GPT-2 Large shaped, 1% outlier rows x20
    w[3] = [Layer("gpt2-large", 16384, K, N, 4, 128, 128, "bf16", "normal_outliers", "uniform_invsqrtk", 2)
            for K, N in [(1280, 3840), (1280, 1280), (1280, 5120), (5120, 1280)]]
    # 4: Llama-3-8B shaped projections, decode to prefill
    w[4] = [Layer("llama3-8b", M, K, N, c, 256, 128, "bf16", "normal", "normal_002", 3)
            for c in (2, 8) for M in (1, 16, 4096)
            for K, N in [(4096, 4096), (4096, 1024), (4096, 14336), (14336, 4096)]]
    # 5: square 4096 sweep over c and M, plus the DLRM top-MLP chain 1024 -> 1024 -> 512 -> 256
    w[5] = [Layer("sweep-4096", M, 4096, 4096, c, 128, 128, "bf16", "uniform_pm1", "uniform_invsqrtk", 4)
            for c in (1, 2, 4, 8) for M in (1, 64, 1024, 16384)]
    w[5] += [Layer("dlrm-top-mlp", 65536, K, N, 2, 128, 128, "bf16", "uniform_pm1", "uniform_invsqrtk", 4)
             for K, N in [(1024, 1024), (1024, 512), (512, 256)]]
    return w


WORKLOADS: Dict[int, List[Layer]] = _workloads()

#: The workload the benchmark times by default: the eight Llama-3-8B shaped projections at
#: M = 4096 (c = 2 and c = 8), the largest single-GPU configuration.
BENCH_WORKLOAD = 4


def make_inputs(layer: Layer, device: str = "cpu") -> Tuple[torch.Tensor, torch.Tensor]:
    """Seeded X[M, K] and Wc[N, K/c] for one layer instance (CPU generation, then moved)."""
    gen = torch.Generator(device="cpu").manual_seed(instance_seed(layer))
    M, K, N, Kc = layer.M, layer.K, layer.N, layer.Kc
    if layer.x_dist in ("normal", "normal_outliers"):
        X = torch.randn(M, K, generator=gen, dtype=torch.float32)
        if layer.x_dist == "normal_outliers":
            n_out = max(1, round(0.01 * M))
            rows = torch.randperm(M, generator=gen)[:n_out]
            X[rows] *= 20.0
    elif layer.x_dist == "uniform_pm1":
        X = torch.rand(M, K, generator=gen, dtype=torch.float32) * 2.0 - 1.0
    else:
        raise ValueError(layer.x_dist)
    if layer.w_dist == "uniform_invsqrtk":
        Wc = (torch.rand(N, Kc, generator=gen, dtype=torch.float32) * 2.0 - 1.0) / math.sqrt(K)
    elif layer.w_dist == "normal_002":
        Wc = torch.randn(N, Kc, generator=gen, dtype=torch.float32) * 0.02
    else:
        raise ValueError(layer.w_dist)
    if layer.dtype == "bf16":
        X, Wc = X.to(torch.bfloat16), Wc.to(torch.bfloat16)
    elif layer.dtype != "fp32":
        raise ValueError(layer.dtype)
    return X.to(device), Wc.to(device)


def torch_dtype(layer: Layer) -> torch.dtype:
    return torch.bfloat16 if layer.dtype == "bf16" else torch.float32
