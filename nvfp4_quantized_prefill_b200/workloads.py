"""Seeded synthetic inputs for the prefill / decode linear layers.

This module is the one piece shared by the CUDA path's tests and benchmark and
by the CPU oracle: it only draws random numbers (on the CPU, with
``torch.Generator``) and rounds them to BF16.  It holds none of the method's
arithmetic.

Distributions (one generator per tensor, seeded from the workload seed and the
tensor's position in a fixed order, values drawn in FP32 then rounded to BF16
with round-to-nearest-even):

* ``outlier``: N(0, 1) with each entry multiplied by 20 with probability 0.01
  (independent Bernoulli per entry) -- the tiny-layer activation recipe.
* ``channel_gain``: N(0, 1) with round(0.02 * K) channels, chosen without
  replacement, multiplied by exp(N(0, 1)) (log-normal per-channel gain).
* ``student_t3``: Student-t with 3 degrees of freedom, Z / sqrt(chi2_3 / 3).
* weights: N(0, std) with std 0.02 (Llama-3-8B shapes) or 0.015 (70B shapes).
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Tuple

import torch

ACT_KINDS = ("outlier", "channel_gain", "student_t3")


def _gen(seed: int, stream: int, device: str = "cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) * 1_000_003 + int(stream) * 7919 + 17)
    return g


def activation(kind: str, M: int, K: int, seed: int, stream: int,
               device: str = "cpu") -> torch.Tensor:
    """BF16 [M, K] activation matrix drawn from the named distribution.

    device="cpu" is the reference stream used by the parity tests; another
    device draws the same recipe from that device's generator (different
    values, same distribution) -- used to build large benchmark inputs fast."""
    g = _gen(seed, stream, device)
    kw = dict(generator=g, dtype=torch.float32, device=device)
    if kind == "outlier":
        x = torch.randn(M, K, **kw)
        mask = torch.rand(M, K, **kw) < 0.01
        x = torch.where(mask, x * 20.0, x)
    elif kind == "channel_gain":
        x = torch.randn(M, K, **kw)
        n_ch = int(round(0.02 * K))
        ch = torch.randperm(K, generator=g, device=device)[:n_ch]
        gain = torch.exp(torch.randn(n_ch, **kw))
        x[:, ch] *= gain
    elif kind == "student_t3":
        z = torch.randn(M, K, **kw)
        c = torch.randn(M, K, **kw).pow_(2)
        c += torch.randn(M, K, **kw).pow_(2)
        c += torch.randn(M, K, **kw).pow_(2)
        x = z / torch.sqrt(c / 3.0)
    else:
        raise ValueError(f"unknown activation kind {kind!r}")
    return x.to(torch.bfloat16)


def weight(N: int, K: int, std: float, seed: int, stream: int,
           device: str = "cpu") -> torch.Tensor:
    """BF16 [N, K] weight matrix ~ N(0, std)."""
    g = _gen(seed, stream, device)
    w = torch.randn(N, K, generator=g, dtype=torch.float32, device=device)
    w.mul_(std)
    return w.to(torch.bfloat16)


def rmsnorm_gain(K: int, seed: int, stream: int, device: str = "cpu") -> torch.Tensor:
    """BF16 [K] RMSNorm gain ~ 1 + N(0, 0.1^2) (a trained gain stays near 1)."""
    g = _gen(seed, stream, device)
    v = torch.randn(K, generator=g, dtype=torch.float32, device=device)
    return (1.0 + 0.1 * v).to(torch.bfloat16)


@dataclasses.dataclass(frozen=True)
class Linear:
    name: str
    N: int
    K: int
    std: float


@dataclasses.dataclass(frozen=True)
class Workload:
    """A prefill workload: token count, activation recipe and the layer's
    linear projections (in execution order)."""
    name: str
    M: int
    act: str
    seed: int
    linears: Tuple[Linear, ...]
    decode_M: Tuple[int, ...]
    swiglu: bool = False        # gate+up -> SwiGLU -> down
    chunks: int = 1             # chunked prefill: M tokens per chunk
    rmsnorm: bool = False       # the first linear's input = RMSNorm(residual) * gain


# Workload table: shapes of the Mix-Quant evaluation's model families at
# prefill scale (Llama-3-8B / 70B shaped projections), synthetic data.
WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny linear 128x256x256", 128, "outlier", 0,
                     (Linear("w", 256, 256, 0.02),), (1,)),
    "llama3_8b_qkv_o": Workload(
        "llama3-8b qkv+o prefill, 8192 tokens", 8192, "channel_gain", 1,
        (Linear("qkv", 6144, 4096, 0.02), Linear("o", 4096, 4096, 0.02)), (1,)),
    "llama3_8b_mlp": Workload(
        "llama3-8b swiglu mlp prefill, 8192 tokens", 8192, "outlier", 2,
        (Linear("gate_up", 28672, 4096, 0.02), Linear("down", 4096, 14336, 0.02)), (1, 8),
        swiglu=True),
    "chunked_131k": Workload(
        "chunked prefill 131072 tokens in 16384-token chunks", 16384, "student_t3", 3,
        (Linear("o", 4096, 4096, 0.02), Linear("gate_up", 14336, 4096, 0.02)), (1,),
        chunks=8),
    "llama3_8b_qkv_rmsnorm": Workload(
        "llama3-8b rmsnorm -> qkv prefill, 8192 tokens", 8192, "channel_gain", 5,
        (Linear("qkv", 6144, 4096, 0.02),), (1,), rmsnorm=True),
    "llama3_70b_layer": Workload(
        "llama3-70b prefill layer linears, 16384 tokens", 16384, "outlier", 4,
        (Linear("qkv", 10240, 8192, 0.015), Linear("o", 8192, 8192, 0.015),
         Linear("gate_up", 57344, 8192, 0.015), Linear("down", 8192, 28672, 0.015)), (1,),
        swiglu=True),
}


def layer_weights(wl: Workload, device: str = "cpu") -> List[torch.Tensor]:
    """All weights of a workload, stream ids 100 + position."""
    return [weight(l.N, l.K, l.std, wl.seed, 100 + i, device) for i, l in enumerate(wl.linears)]


def layer_activation(wl: Workload, K: int, stream: int, M: int | None = None,
                     device: str = "cpu") -> torch.Tensor:
    return activation(wl.act, wl.M if M is None else M, K, wl.seed, stream, device)
