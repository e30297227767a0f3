"""Seeded synthetic layer inputs for the rank-r W4A4 linear.

This module only draws inputs: it holds none of the quantizer's or the
forward's arithmetic, so that both the CPU oracle and the CUDA path can be fed
identical bits from it.  Every tensor is drawn in fp32 from a CPU
``torch.Generator`` and rounded once to bf16 (the activations, weights and
low-rank factors are 16-bit tensors in the layer; the smoothing vector is fp32).

Layer shapes follow the diffusion / language backbones that the H-SVDQuant
pages evaluate (Deflating the Hessian, Tables 1, 3 and 8: PixArt-Sigma,
SANA-1.6B, FLUX.1 and Qwen3-8B); value distributions are synthetic stand-ins
(Gaussian weights, Gaussian activations with a few large outlier channels, or
a log-uniform per-channel spread), because the pages print none.

The smoothing vector uses the common migration-strength-1/2 recipe
``s_k = sqrt(max_m |X[m,k]| / max_n |W[n,k]|)``, evaluated in fp64 on the
drawn data and stored as fp32.  It is an input of the layer, not something the
layer computes.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional

import torch

__all__ = ["LayerSpec", "LayerData", "make_layer", "WORKLOADS", "workload_layers"]


@dataclasses.dataclass(frozen=True)
class LayerSpec:
    """One linear layer of a synthetic workload."""

    name: str
    M: int            # tokens
    K: int            # in-features
    N: int            # out-features
    r: int            # rank of the high-precision branch
    act: str          # "outlier" | "logstd"
    outlier_frac: float = 0.0
    outlier_mult: float = 1.0
    seed: int = 0
    bias: bool = False  # the stated workloads use a zero bias; tests switch it on
    group: int = 64     # quantization group along K (the pages use 128 for Qwen3-8B)
    fmt: str = "int4"   # "int4" (the method's groups of 64/128) or "nvfp4" (the DiRotQ page's FP4 setting)


@dataclasses.dataclass
class LayerData:
    spec: LayerSpec
    X: torch.Tensor    # bf16 [M, K]
    W: torch.Tensor    # bf16 [N, K]  (torch Linear layout)
    L1: torch.Tensor   # bf16 [K, r]
    L2: torch.Tensor   # bf16 [r, N]
    bias: Optional[torch.Tensor]  # bf16 [N] or None (zero bias)
    s: torch.Tensor    # fp32 [K]


def _smoothing_vector(X: torch.Tensor, W: torch.Tensor) -> torch.Tensor:
    xmax = X.double().abs().amax(dim=0)
    wmax = W.double().abs().amax(dim=0)
    s = torch.ones_like(xmax)
    ok = (xmax > 0) & (wmax > 0)
    s[ok] = torch.sqrt(xmax[ok] / wmax[ok])
    return s.float()


def make_layer(spec: LayerSpec, with_s: bool = True) -> LayerData:
    """Draw one layer's tensors from ``spec.seed`` in a fixed order."""
    g = torch.Generator().manual_seed(spec.seed)
    M, K, N, r = spec.M, spec.K, spec.N, spec.r
    X = torch.randn(M, K, generator=g, dtype=torch.float32)
    if spec.act == "outlier":
        n_out = int(math.ceil(spec.outlier_frac * K)) if spec.outlier_frac > 0 else 0
        perm = torch.randperm(K, generator=g)
        if n_out:
            X[:, perm[:n_out]] *= spec.outlier_mult
    elif spec.act == "logstd":
        # per-channel std log-uniform in [0.1, 8]: an ~80x spread across channels
        u = torch.rand(K, generator=g, dtype=torch.float64)
        std = torch.exp(math.log(0.1) + u * (math.log(8.0) - math.log(0.1)))
        X = X * std.float()[None, :]
    else:
        raise ValueError(f"unknown activation generator {spec.act!r}")
    W = torch.randn(N, K, generator=g, dtype=torch.float32) * 0.02
    L1 = torch.randn(K, r, generator=g, dtype=torch.float32) * 0.02
    L2 = torch.randn(r, N, generator=g, dtype=torch.float32) * 0.02
    bias = None
    if spec.bias:
        bias = (torch.randn(N, generator=g, dtype=torch.float32) * 0.5).to(torch.bfloat16)
    Xb, Wb = X.to(torch.bfloat16), W.to(torch.bfloat16)
    s = _smoothing_vector(Xb, Wb) if with_s else torch.ones(K, dtype=torch.float32)
    return LayerData(spec, Xb, Wb, L1.to(torch.bfloat16), L2.to(torch.bfloat16), bias, s)


def _pixart(M, r=4, seed0=0):
    common = dict(act="outlier", outlier_frac=0.01, outlier_mult=30.0)
    return [LayerSpec("pixart_qkv", M, 1152, 3456, r, seed=seed0 + 0, **common),
            LayerSpec("pixart_fc1", M, 1152, 4608, r, seed=seed0 + 1, **common),
            LayerSpec("pixart_fc2", M, 4608, 1152, r, seed=seed0 + 2, **common)]


def _sana(r):
    common = dict(act="logstd")
    return [LayerSpec(f"sana_up_r{r}", 1024, 2240, 5600, r, seed=0, **common),
            LayerSpec(f"sana_down_r{r}", 1024, 5600, 2240, r, seed=1, **common)]


def _flux(r, fmt="int4"):
    common = dict(act="outlier", outlier_frac=0.005, outlier_mult=50.0, fmt=fmt)
    tag = "" if fmt == "int4" else f"_{fmt}"
    return [LayerSpec(f"flux_qkv_r{r}{tag}", 4608, 3072, 9216, r, seed=0, **common),
            LayerSpec(f"flux_mlp_up_r{r}{tag}", 4608, 3072, 12288, r, seed=1, **common),
            LayerSpec(f"flux_mlp_down_r{r}{tag}", 4608, 12288, 3072, r, seed=2, **common)]


def _qwen(M, group=64):
    common = dict(act="outlier", outlier_frac=0.001, outlier_mult=100.0, group=group)
    tag = "" if group == 64 else f"_g{group}"
    return [LayerSpec(f"qwen_gate_up_m{M}{tag}", M, 4096, 12288, 4, seed=0, **common),
            LayerSpec(f"qwen_down_m{M}{tag}", M, 12288, 4096, 4, seed=1, **common)]


#: Named workloads: the layer shapes of the backbones the pages evaluate.
WORKLOADS: Dict[str, List[LayerSpec]] = {
    "pixart_tiny": [LayerSpec("pixart_tiny", 256, 1152, 1152, 4, act="outlier",
                              outlier_frac=0.01, outlier_mult=30.0, seed=0)],
    "pixart_1024px": _pixart(4096),
    "sana_r4": _sana(4),
    "sana_r32": _sana(32),
    "flux_block_r4": _flux(4),
    "flux_block_r32": _flux(32),
    **{f"qwen3_8b_m{M}": _qwen(M) for M in (1, 16, 128, 1024, 8192)},
    # the pages' own Qwen3-8B setting: groups of 128 (Table 3 and Table 4 captions)
    **{f"qwen3_8b_m{M}_g128": _qwen(M, 128) for M in (1, 16, 128, 1024, 8192)},
    # the same FLUX.1 block in the NVFP4 variant (E2M1 values, E4M3 scale per 16, fp32 tensor scale)
    "flux_block_r4_nvfp4": _flux(4, "nvfp4"),
}


def workload_layers(name: str) -> List[LayerSpec]:
    return list(WORKLOADS[name])
