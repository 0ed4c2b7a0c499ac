"""Seeded synthetic inputs shaped like the pages' LLaMA-family layers.

This module only draws random numbers (torch generators); it holds none of the
layer's arithmetic, so both the oracle-based tests and the CUDA path may use
it.  Every draw is reproducible from ``seed``.

Distributions:
* activations x: N(0, 1) rounded to fp16; optionally a seeded set of
  ``round(outlier_frac * K)`` input channels multiplied by ``outlier_mult``
  in every token (the prefill workload's outlier channels);
* ternary weights: iid uniform over {-1, 0, +1} (int8);
* sign weights: iid +-1 with p = 0.5, as fp16 (the dense matrix whose sign
  is packed);
* OneBit value vectors g, h: U(0.5, 1.5) * 0.02, rounded to fp16;
* SVID input: N(0, 0.02) fp32;
* RMSNorm weights: 1 + 0.1 N(0, 1), rounded to fp16.
"""
from __future__ import annotations

import torch


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def activations(M: int, K: int, seed: int, device="cpu", outlier_frac: float = 0.0,
                outlier_mult: float = 20.0) -> torch.Tensor:
    g = _gen(seed, device)
    x = torch.randn((M, K), generator=g, device=device, dtype=torch.float32)
    n_out = int(round(outlier_frac * K))
    if n_out > 0:
        cols = torch.randperm(K, generator=g, device=device)[:n_out]
        x[:, cols] *= outlier_mult
    return x.to(torch.float16)


def ternary_weights(N: int, K: int, seed: int, device="cpu") -> torch.Tensor:
    g = _gen(seed, device)
    return (torch.randint(0, 3, (N, K), generator=g, device=device, dtype=torch.int8) - 1).to(torch.int8)


def sign_weights(N: int, K: int, seed: int, device="cpu") -> torch.Tensor:
    g = _gen(seed, device)
    b = torch.randint(0, 2, (N, K), generator=g, device=device, dtype=torch.int8)
    return (b.to(torch.float16) * 2 - 1)


def value_vector(n: int, seed: int, device="cpu") -> torch.Tensor:
    g = _gen(seed, device)
    u = torch.rand((n,), generator=g, device=device, dtype=torch.float32)
    return ((u + 0.5) * 0.02).to(torch.float16)


def norm_weight(n: int, seed: int, device="cpu") -> torch.Tensor:
    g = _gen(seed, device)
    return (1.0 + 0.1 * torch.randn((n,), generator=g, device=device, dtype=torch.float32)).to(torch.float16)


def svid_weights(N: int, K: int, seed: int, device="cpu") -> torch.Tensor:
    g = _gen(seed, device)
    return torch.randn((N, K), generator=g, device=device, dtype=torch.float32) * 0.02
