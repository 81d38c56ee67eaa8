"""Seeded synthetic inputs for the QLoRA NF4 layer (CPU tensors).

This module only draws random numbers; it holds none of the method's
arithmetic, so both the CUDA path and the CPU oracle can be fed the same
inputs.  Every tensor comes from its own torch CPU generator seeded with
``seed + index``, is drawn in fp32 and then cast, so it is identical on any
machine and independent of the device.

Distributions (the workloads the pages describe: Llama-7B..70B-shaped
frozen weights with normal-like values, bf16 activations, bf16 adapters):
  W0  ~ N(0, std^2), or Student-t(nu=5) rescaled to standard deviation std
  x   ~ N(0, 1)            (bf16)
  dh  ~ N(0, 1)            (bf16)
  A   ~ U(-1/sqrt(in), 1/sqrt(in))   (bf16)
  B   ~ N(0, 0.01^2)       (bf16, nonzero so the LoRA branch is exercised)
"""

from __future__ import annotations

import math

import torch

# tensor indices of the seed offsets
IDX_W, IDX_X, IDX_A, IDX_B, IDX_DH = 0, 1, 2, 3, 4


def _gen(seed: int, index: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed) + int(index))
    return g


def weight(out_f: int, in_f: int, std: float = 0.02, dist: str = "normal", seed: int = 0,
           index: int = IDX_W) -> torch.Tensor:
    """fp32 [out_f, in_f] frozen base weight."""
    g = _gen(seed, index)
    if dist == "normal":
        return torch.randn(out_f, in_f, generator=g, dtype=torch.float32) * std
    if dist == "student_t5":
        nu = 5
        z = torch.randn(out_f, in_f, generator=g, dtype=torch.float32)
        chi2 = torch.zeros(out_f, in_f, dtype=torch.float32)
        for _ in range(nu):
            chi2 += torch.randn(out_f, in_f, generator=g, dtype=torch.float32) ** 2
        t = z / torch.sqrt(chi2 / nu)
        return t * (std / math.sqrt(nu / (nu - 2)))
    raise ValueError(dist)


def activations(M: int, n: int, seed: int = 0, index: int = IDX_X) -> torch.Tensor:
    """bf16 [M, n] standard-normal activations (x) or output gradients (dh)."""
    return torch.randn(M, n, generator=_gen(seed, index), dtype=torch.float32).to(torch.bfloat16)


def lora_A(r: int, in_f: int, seed: int = 0, index: int = IDX_A) -> torch.Tensor:
    bound = 1.0 / math.sqrt(in_f)
    u = torch.rand(r, in_f, generator=_gen(seed, index), dtype=torch.float32)
    return ((u * 2.0 - 1.0) * bound).to(torch.bfloat16)


def lora_B(out_f: int, r: int, std: float = 0.01, seed: int = 0, index: int = IDX_B) -> torch.Tensor:
    return (torch.randn(out_f, r, generator=_gen(seed, index), dtype=torch.float32) * std).to(torch.bfloat16)


def problem(M: int, in_f: int, out_f: int, r: int, w_std: float = 0.02, w_dist: str = "normal",
            seed: int = 0) -> dict:
    """All inputs of one linear layer: W (fp32), x, A, B, dh (bf16), CPU tensors."""
    return dict(
        W=weight(out_f, in_f, w_std, w_dist, seed),
        x=activations(M, in_f, seed, IDX_X),
        A=lora_A(r, in_f, seed),
        B=lora_B(out_f, r, seed=seed),
        dh=activations(M, out_f, seed, IDX_DH),
    )
