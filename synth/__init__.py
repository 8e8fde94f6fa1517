"""Seeded synthetic inputs shared by the oracle tests, the GPU parity tests and bench.py.

This module holds no quantization or GEMM arithmetic. It only draws the
workloads: activations X ~ N(0, 1) with a few outlier input features scaled by
20, and weights W ~ N(0, 0.02), both rounded to bf16 by torch's own cast.

Recipe (one CPU torch.Generator per tensor, so that every consumer sees the
same bits):
  * X: randn(M, K) with generator seed `seed`; the outlier columns are chosen
    by randperm(K) with seed `seed + 2`, the first n of them, and multiplied
    by 20 before the bf16 cast; n = 2 for the tiny case, round(0.005 * K)
    otherwise.
  * W: 0.02 * randn(N, K) with seed `seed + 1`, then bf16.

The shapes are the Llama-3.x projection shapes the FP8 checkpoints on the
pages quantize: Llama-3.2-3B (hidden 3072, MLP 8192), Llama-3.1-8B (hidden
4096, 32 query / 8 KV heads of 128, MLP 14336) and Llama-3.1-70B (hidden 8192,
64 query / 8 KV heads of 128, MLP 28672).
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional

import torch

CHANNEL_TOKEN = 0  # weights per output channel, activations per token
BLOCK128 = 1       # weights per 128x128 block, activations per 128-group


def n_outliers(K: int, tiny: bool = False) -> int:
    """Number of outlier input features for a row length K."""
    return 2 if tiny else int(round(0.005 * K))


def make_x(M: int, K: int, seed: int = 0, n_out: Optional[int] = None,
           device: str = "cpu") -> torch.Tensor:
    """Activations X [M, K] bf16: N(0,1) with `n_out` outlier columns x20."""
    if n_out is None:
        n_out = n_outliers(K)
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(M, K, generator=g, dtype=torch.float32)
    if n_out > 0:
        go = torch.Generator().manual_seed(seed + 2)
        cols = torch.randperm(K, generator=go)[:n_out]
        x[:, cols] *= 20.0
    return x.to(torch.bfloat16).to(device)


def make_w(N: int, K: int, seed: int = 0, device: str = "cpu") -> torch.Tensor:
    """Weights W [N, K] bf16 (nn.Linear layout: out x in), N(0, 0.02)."""
    g = torch.Generator().manual_seed(seed + 1)
    w = 0.02 * torch.randn(N, K, generator=g, dtype=torch.float32)
    return w.to(torch.bfloat16).to(device)


def make_x_device(M: int, K: int, seed: int, n_out: Optional[int] = None,
                  device: str = "cuda") -> torch.Tensor:
    """Same distribution as make_x, drawn on the device (for timing runs whose
    inputs are never compared element by element with the oracle)."""
    if n_out is None:
        n_out = n_outliers(K)
    g = torch.Generator(device=device).manual_seed(seed)
    x = torch.randn(M, K, generator=g, device=device, dtype=torch.float32)
    if n_out > 0:
        go = torch.Generator().manual_seed(seed + 2)
        cols = torch.randperm(K, generator=go)[:n_out].to(device)
        x[:, cols] *= 20.0
    return x.to(torch.bfloat16)


def make_w_device(N: int, K: int, seed: int, device: str = "cuda") -> torch.Tensor:
    g = torch.Generator(device=device).manual_seed(seed + 1)
    w = 0.02 * torch.randn(N, K, generator=g, device=device, dtype=torch.float32)
    return w.to(torch.bfloat16)


@dataclasses.dataclass(frozen=True)
class Gemm:
    """One FP8 linear: Y[M, N] = X[M, K] . W[N, K]^T."""
    name: str
    M: int
    K: int
    N: int
    mode: int = CHANNEL_TOKEN
    x: str = ""          # which activation it reads; GEMMs naming the same one share it
    w: str = ""          # which weight it multiplies ("" = its own); the M values of one projection share one

    @property
    def flops(self) -> int:
        return 2 * self.M * self.N * self.K

    @property
    def weight(self) -> str:
        return self.w or self.name


def weight_seed(name: str) -> int:
    """Seed of a workload weight, from its name (stable across runs and processes)."""
    import zlib
    return zlib.crc32(name.encode()) % 1000


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    gemms: List[Gemm]
    tiny: bool = False


def workloads() -> dict:
    """The five workloads, keyed by name."""
    w = {}
    w["tiny_16x256x512"] = Workload("tiny_16x256x512", [Gemm("tiny", 16, 256, 512, x="x")], tiny=True)
    w["llama3.2-3b_mlp_m2048"] = Workload(
        "llama3.2-3b_mlp_m2048",
        [Gemm("gate_proj", 2048, 3072, 8192, x="mlp_in"), Gemm("up_proj", 2048, 3072, 8192, x="mlp_in")])
    w["llama3.1-8b_layer_m8192"] = Workload(
        "llama3.1-8b_layer_m8192",
        [Gemm("q_proj", 8192, 4096, 4096, x="attn_in"), Gemm("k_proj", 8192, 4096, 1024, x="attn_in"),
         Gemm("v_proj", 8192, 4096, 1024, x="attn_in"), Gemm("o_proj", 8192, 4096, 4096, x="attn_out"),
         Gemm("gate_proj", 8192, 4096, 14336, x="mlp_in"), Gemm("up_proj", 8192, 4096, 14336, x="mlp_in"),
         Gemm("down_proj", 8192, 14336, 4096, x="mlp_act")])
    w["llama3.2-3b_block128"] = Workload(
        "llama3.2-3b_block128",
        [Gemm(f"gate_proj_m{m}", m, 3072, 8192, BLOCK128, x=f"mlp_in_m{m}", w="gate_proj") for m in (1, 16, 4096)])
    g70 = []
    for m in (1, 8, 64, 512, 8192):
        g70 += [Gemm(f"gate_proj_m{m}", m, 8192, 28672, x=f"mlp_in_m{m}", w="gate_proj"),
                Gemm(f"up_proj_m{m}", m, 8192, 28672, x=f"mlp_in_m{m}", w="up_proj"),
                Gemm(f"down_proj_m{m}", m, 28672, 8192, x=f"mlp_act_m{m}", w="down_proj"),
                Gemm(f"qkv_proj_m{m}", m, 8192, 10240, x=f"attn_in_m{m}", w="qkv_proj")]
    w["llama3.1-70b_sweep"] = Workload("llama3.1-70b_sweep", g70)
    for m in (1, 8, 64, 512, 8192):   # one M of the sweep at a time
        w[f"llama3.1-70b_m{m}"] = Workload(f"llama3.1-70b_m{m}", [g for g in g70 if g.M == m])
    return w
