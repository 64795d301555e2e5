"""Seeded synthetic inputs shaped like DiT linear layers.

This module only draws random numbers.  It holds none of the quantization or
GEMM arithmetic, and it is the one module that both the CUDA path (tests,
benchmark) and the CPU oracle consume.

The pages benchmark on WebVid-10M / VGGSound / UCF-101 clips and COCO prompts
with trained DiT weights (NVFP4-DiT README, "Datasets, hardware, and metrics";
FP4DiT README, "Quantization").  None of those are used: seeded tensors with
the shapes and value structure of the corresponding transformer layers stand
in for them.

Workloads (X is the layer input [M, K] in bf16, W the weight [N, K] in bf16,
Y = X W^T):

  pr1         seed 0  M=128    one layer K=256 -> N=256
                      X ~ N(0,1), W ~ N(0, 0.02^2)
  dit_xl2     seed 1  M=2048   (256 tokens x batch 8, hidden 1152)
                      qkv 1152->3456, out 1152->1152, fc1 1152->4608, fc2 4608->1152
                      X ~ N(0,1) with round(0.01 K) channels scaled x20 (outliers)
  pixart1024  seed 2  M=8192   (4096 tokens x batch 2, hidden 1152), same four
                      layers plus cross-attention K and V from text tokens
                      (M = 2 x 300 = 600, K=4096 -> N=1152)
                      X ~ Student-t nu=3:  z / sqrt(chi2_3 / 3)
  video_dit   seed 3  M=32768  (16 frames x 2048 tokens, hidden 3072)
                      qkv 3072->9216, fc1 3072->12288, fc2 12288->3072
                      X ~ N(0,1) times a per-token factor exp(U(ln 0.1, ln 10))
  w4a16       seed 4  M=16384  (hidden 5120) fc1 5120->20480, fc2 20480->5120
                      X ~ N(0,1), W ~ N(0, 0.015^2) (weights-only NVFP4)

All weights except w4a16 are N(0, 0.02^2).  Every tensor is drawn in float32
from a torch.Generator seeded with seed * 1000 + layer index (X first, then
W) and cast to bf16 with round-to-nearest-even.  A generator lives on the
device the tensor is made on, so CPU and CUDA draws differ but each is
reproducible.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Layer:
    name: str
    M: int
    K: int
    N: int


@dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    x_dist: str          # "normal" | "outlier" | "student_t3" | "token_scaled"
    w_std: float
    layers: tuple

    def layer(self, name: str) -> Layer:
        for l in self.layers:
            if l.name == name:
                return l
        raise KeyError(name)

    def flops(self) -> int:
        return sum(2 * l.M * l.N * l.K for l in self.layers)


def _dit_layers(M: int, h: int, mlp: int):
    return (Layer("qkv", M, h, 3 * h), Layer("out", M, h, h),
            Layer("fc1", M, h, mlp), Layer("fc2", M, mlp, h))


WORKLOADS = {
    "pr1": Workload("pr1", 0, "normal", 0.02, (Layer("linear", 128, 256, 256),)),
    "dit_xl2": Workload("dit_xl2", 1, "outlier", 0.02, _dit_layers(2048, 1152, 4608)),
    "pixart1024": Workload("pixart1024", 2, "student_t3", 0.02,
                           _dit_layers(8192, 1152, 4608)
                           + (Layer("xattn_k", 600, 4096, 1152), Layer("xattn_v", 600, 4096, 1152))),
    "video_dit": Workload("video_dit", 3, "token_scaled", 0.02,
                          (Layer("qkv", 32768, 3072, 9216), Layer("fc1", 32768, 3072, 12288),
                           Layer("fc2", 32768, 12288, 3072))),
    "w4a16": Workload("w4a16", 4, "normal", 0.015,
                      (Layer("fc1", 16384, 5120, 20480), Layer("fc2", 16384, 20480, 5120))),
}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _draw_x(dist: str, M: int, K: int, gen: torch.Generator, device) -> torch.Tensor:
    x = torch.randn(M, K, generator=gen, device=device, dtype=torch.float32)
    if dist == "normal":
        pass
    elif dist == "outlier":
        n_out = int(round(0.01 * K))
        ch = torch.randperm(K, generator=gen, device=device)[:n_out]
        x[:, ch] *= 20.0
    elif dist == "student_t3":
        chi2 = torch.randn(3, M, K, generator=gen, device=device, dtype=torch.float32).square_().sum(0)
        x.div_(torch.sqrt(chi2 / 3.0))
    elif dist == "token_scaled":
        u = torch.rand(M, 1, generator=gen, device=device, dtype=torch.float32)
        lo, hi = math.log(0.1), math.log(10.0)
        x.mul_(torch.exp(lo + (hi - lo) * u))
    else:
        raise ValueError(dist)
    return x.to(torch.bfloat16)


def layer_tensors(workload: str, layer: str, device="cpu", want=("x", "w")):
    """(X [M,K] bf16, W [N,K] bf16) of one layer, seeded and reproducible."""
    wl = WORKLOADS[workload]
    idx = [l.name for l in wl.layers].index(layer)
    L = wl.layers[idx]
    gen = _gen(wl.seed * 1000 + idx, device)
    x = _draw_x(wl.x_dist, L.M, L.K, gen, device)
    w = (torch.randn(L.N, L.K, generator=gen, device=device, dtype=torch.float32)
         * wl.w_std).to(torch.bfloat16)
    out = {"x": x, "w": w}
    return tuple(out[k] for k in want)


def random_bf16(shape, seed: int, dist: str = "normal", scale: float = 1.0, device="cpu"):
    """Generic seeded bf16 tensor for tests: dist in normal | student_t3 |
    outlier | token_scaled, multiplied by ``scale``."""
    gen = _gen(seed, device)
    M, K = shape
    x = _draw_x(dist, M, K, gen, device)
    if scale != 1.0:
        x = (x.float() * scale).to(torch.bfloat16)
    return x
