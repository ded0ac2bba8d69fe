"""Seeded synthetic inputs for the blockwise-FP8 linear layer.

This module only draws random tensors; it holds none of the method's
arithmetic.  The tests, the benchmark and the oracle comparisons all take their
inputs from here, so both sides of every comparison see the same numbers.

Workloads restate the Qwen3-1.7B-like model of "Puro-2B: Poor Lab's
Qwen2-1.5B Trained on RTX 5090 within $5090" (section "方法": hidden 2048,
seq 4096, untied LM head) as synthetic tensors:

  * activations ~ N(0, 1) in bf16, with 1% of the K channels (round(0.01 K)
    indices from a seeded permutation) multiplied by 50 as outliers;
  * weights ~ N(0, 0.02);
  * output gradients ~ N(0, 1e-3).

Values are drawn in fp32 and rounded to bf16 (round-to-nearest-even).
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

# Qwen3-1.7B-like layer sizes (hidden 2048, 16 q heads + 2x8 kv heads of 128,
# MLP 6144, vocab 151936), 28 layers.
HIDDEN = 2048
QKV_OUT = 4096
MLP = 6144
VOCAB = 151936
LAYERS = 28


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def normal_bf16(shape, std: float, seed: int, device="cpu") -> torch.Tensor:
    """N(0, std^2) drawn in fp32 on `device`, rounded to bf16."""
    g = _gen(seed, device)
    x = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


def outlier_channels(K: int, seed: int, frac: float = 0.01) -> torch.Tensor:
    """round(frac*K) channel indices from a seeded permutation (CPU)."""
    n = int(round(frac * K))
    g = _gen(seed + 7919, "cpu")
    return torch.randperm(K, generator=g)[:n]


def activations_bf16(M: int, K: int, seed: int, device="cpu", outliers: bool = True,
                     outlier_gain: float = 50.0) -> torch.Tensor:
    """X [M,K] ~ N(0,1) bf16 with 1% of the channels scaled by 50."""
    g = _gen(seed, device)
    x = torch.randn(M, K, generator=g, device=device, dtype=torch.float32)
    if outliers:
        idx = outlier_channels(K, seed).to(x.device)
        x[:, idx] *= outlier_gain
    return x.to(torch.bfloat16)


def weights_bf16(N: int, K: int, seed: int, device="cpu") -> torch.Tensor:
    return normal_bf16((N, K), 0.02, seed, device)


def grads_bf16(M: int, N: int, seed: int, device="cpu") -> torch.Tensor:
    return normal_bf16((M, N), 1e-3, seed, device)


@dataclass(frozen=True)
class Linear:
    """One linear layer Y[M,N] = X[M,K] W[N,K]^T of the synthetic model."""
    name: str
    M: int
    K: int
    N: int

    def x(self, seed: int, device="cpu", outliers: bool = True) -> torch.Tensor:
        return activations_bf16(self.M, self.K, seed, device, outliers)

    def w(self, seed: int, device="cpu") -> torch.Tensor:
        return weights_bf16(self.N, self.K, seed + 1, device)

    def dy(self, seed: int, device="cpu") -> torch.Tensor:
        return grads_bf16(self.M, self.N, seed + 2, device)

    @property
    def flops(self) -> int:
        return 2 * self.M * self.N * self.K


# The configurations the tests and the benchmark use.
TINY = Linear("tiny", 256, 512, 512)
QKV = Linear("qkv", 4096, HIDDEN, QKV_OUT)
OPROJ = Linear("o_proj", 4096, HIDDEN, HIDDEN)
GATE_UP = Linear("gate_up", 16384, HIDDEN, 2 * MLP)
DOWN = Linear("down", 16384, MLP, HIDDEN)
LM_HEAD = Linear("lm_head", 16384, HIDDEN, VOCAB)


def layer_linears(M: int = 16384):
    """The four linears of one transformer layer at M tokens."""
    return [Linear("qkv", M, HIDDEN, QKV_OUT), Linear("o_proj", M, HIDDEN, HIDDEN),
            Linear("gate_up", M, HIDDEN, 2 * MLP), Linear("down", M, MLP, HIDDEN)]


def bf16_bits(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 bit patterns on the host (for the oracle)."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view("uint16")
