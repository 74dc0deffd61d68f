"""Seeded synthetic inputs shared by the oracle tests, the GPU tests and the
benchmark.

This module holds no NVFP4 arithmetic: it only draws random bf16 tensors with
the shapes and value distributions of FLUX-style transformer linear layers.
Every tensor is drawn on the CPU from a ``torch.Generator`` seeded per
workload, so the oracle and the CUDA path see identical bytes.

FLUX shapes: hidden size 3072, MLP ratio 4, 4096 image tokens (1024^2 latent)
plus 512 text tokens = 4608 tokens; 16896 tokens = 16384 image tokens (2048^2
latent) + 512 text.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def normal_bf16(shape, std: float, gen: torch.Generator) -> torch.Tensor:
    """N(0, std^2) samples rounded to bf16."""
    return (torch.randn(*shape, generator=gen, dtype=torch.float32) * std).to(torch.bfloat16)


def activations_with_outlier_channels(m: int, k: int, seed: int, frac: float = 0.01,
                                      factor: float = 20.0) -> torch.Tensor:
    """x ~ N(0,1) [m, k] with ``round(frac*k)`` input channels (columns, chosen
    by the seed) multiplied by ``factor``: the outlier-channel pattern of
    transformer activations.  bf16."""
    gen = _gen(seed)
    x = torch.randn(m, k, generator=gen, dtype=torch.float32)
    n_out = int(round(frac * k))
    if n_out:
        cols = torch.randperm(k, generator=gen)[:n_out]
        x[:, cols] *= factor
    return x.to(torch.bfloat16)


def laplace_activations(m: int, k: int, seed: int, spike_frac: float = 0.001,
                        spike_factor: float = 50.0, zero_block_frac: float = 0.01) -> torch.Tensor:
    """x ~ Laplace(0,1) [m, k]; a fraction ``spike_frac`` of entries times
    ``spike_factor``; a fraction ``zero_block_frac`` of the aligned 16-element
    runs along k set to exactly zero.  bf16."""
    gen = _gen(seed)
    u = torch.rand(m, k, generator=gen, dtype=torch.float64) - 0.5
    u = u.clamp(-0.5 + 1e-12, 0.5 - 1e-12)
    x = (-torch.sign(u) * torch.log1p(-2.0 * u.abs())).to(torch.float32)
    n_spike = int(round(spike_frac * m * k))
    if n_spike:
        idx = torch.randint(0, m * k, (n_spike,), generator=gen)
        x.view(-1)[idx] *= spike_factor
    if k % 16 == 0:
        runs = x.view(m, k // 16, 16)
        n_zero = int(round(zero_block_frac * m * (k // 16)))
        if n_zero:
            idx = torch.randint(0, m * (k // 16), (n_zero,), generator=gen)
            runs.view(-1, 16)[idx] = 0.0
    return x.to(torch.bfloat16)


@dataclass(frozen=True)
class LinearWorkload:
    """One NVFP4 linear layer y = x W^T + b with synthetic bf16 tensors."""
    name: str
    m: int
    k: int
    n: int
    seed: int
    outliers: bool = True
    bias: bool = True
    w_std: float = 0.02
    b_std: float = 0.01

    def activations(self) -> torch.Tensor:
        if self.outliers:
            return activations_with_outlier_channels(self.m, self.k, self.seed)
        return normal_bf16((self.m, self.k), 1.0, _gen(self.seed))

    def weight(self) -> torch.Tensor:
        return normal_bf16((self.n, self.k), self.w_std, _gen(self.seed + 1000))

    def bias_vec(self):
        if not self.bias:
            return None
        return normal_bf16((self.n,), self.b_std, _gen(self.seed + 2000))

    @property
    def flops(self) -> int:
        return 2 * self.m * self.n * self.k


#: Tiny W4A4 linear: x [128,256] ~ N(0,1), W [256,256] ~ N(0,0.02), no bias.
TINY = LinearWorkload("tiny_m128_k256_n256", 128, 256, 256, seed=0, outliers=False, bias=False)

#: FLUX double-stream MLP-up: x [4608,3072] with 1% outlier channels x20,
#: W [12288,3072] ~ N(0,0.02), bias [12288] ~ N(0,0.01).
MLP_UP = LinearWorkload("flux_mlp_up_m4608_k3072_n12288", 4608, 3072, 12288, seed=1)

#: Standalone activation quantize: Laplace(0,1) [4608,12288] with spikes and
#: zero blocks.
QUANT_M, QUANT_K, QUANT_SEED = 4608, 12288, 2


def quantize_input():
    return laplace_activations(QUANT_M, QUANT_K, QUANT_SEED)


#: FLUX single-stream block pair: fused QKV+MLP-in (N = 3*3072 + 4*3072) and
#: the output projection over [attention 3072 | MLP 12288] = K 15360.
SINGLE_IN = LinearWorkload("flux_single_in_m4608_k3072_n21504", 4608, 3072, 21504, seed=3,
                           outliers=False)
SINGLE_OUT = LinearWorkload("flux_single_out_m4608_k15360_n3072", 4608, 15360, 3072, seed=13,
                            outliers=False)
#: Column ranges of SINGLE_IN's output: Q (stands in for the attention output),
#: K and V (bf16 out), MLP (GELU-tanh, then quantized).
SINGLE_Q = (0, 3072)
SINGLE_KV = (3072, 9216)
SINGLE_MLP = (9216, 21504)

#: Token-count sweep of the attention-projection GEMM, K = N = 3072.
SWEEP = tuple(LinearWorkload(f"flux_proj_m{m}_k3072_n3072", m, 3072, 3072, seed=4 + i)
              for i, m in enumerate((512, 1024, 4608, 9216, 16896)))
