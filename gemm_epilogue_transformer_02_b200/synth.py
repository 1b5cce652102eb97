"""Seeded synthetic inputs for the CODA GEMM + epilogue hot path.

This module only draws random numbers and rounds them to bf16; it holds none
of the method's arithmetic.  The same tensors (as bf16 bit patterns) feed the
CUDA library and the fp64 oracle, so both sides see identical inputs.

Recipe (one CPU ``torch.Generator`` per workload, tensors drawn in the order
listed, ``randn`` in fp32, scaled by the stated std, rounded to bf16 with
round-to-nearest-even):

* ``tiny_block`` (256 tokens, hidden 512 -> 1536), seed 0:
  x[256,512] ~ N(0,1), res[256,512] ~ N(0,1), W1[512,512] and W2[512,1536]
  with std 1/sqrt(512), gamma[512] = 1 + 0.1 N(0,1), eps = 1e-6.
* ``llama1b_block_tail`` (8192 tokens, hidden 2048 -> fused gate/up 16384),
  seed 1: x, res [8192,2048] ~ N(0,1); W1[2048,2048], W2[2048,16384] std 0.02;
  gamma = 1 + 0.1 N(0,1).  The SwiGLU + down-projection continuation draws
  W_down[8192,2048] (std 0.02) next from the same generator and uses W2 as the
  fused gate/up weight.
* ``lmhead_ce`` (8192 tokens, hidden 2048, vocab 128256), seed 3:
  H[8192,2048] ~ N(0,1), W_vocab[2048,128256] std 0.02, labels uniform
  integers in [0, 128256).
* ``block_backward`` seed 4: dOut[8192,16384] std 0.01 (the forward state is
  the 1B block-tail workload).

All weights are stored ``[in, out]`` row-major; activations ``[tokens, features]``.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch

EPS = 1e-6


def normal_bf16(gen: torch.Generator, shape, std: float = 1.0, mean: float = 0.0) -> torch.Tensor:
    """Draw fp32 N(0,1), scale and shift, round to bf16 (RNE).  CPU tensor."""
    t = torch.randn(*shape, generator=gen, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    if mean != 0.0:
        t.add_(mean)
    return t.to(torch.bfloat16)


def gamma_bf16(gen: torch.Generator, n: int) -> torch.Tensor:
    """RMSNorm weight 1 + 0.1 N(0,1), rounded to bf16."""
    return normal_bf16(gen, (n,), std=0.1, mean=1.0)


def labels_uniform(gen: torch.Generator, m: int, vocab: int) -> torch.Tensor:
    """Uniform int64 labels in [0, vocab)."""
    return torch.randint(0, vocab, (m,), generator=gen, dtype=torch.int64)


def make_gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


@dataclass
class BlockInputs:
    x: torch.Tensor
    res: torch.Tensor
    W1: torch.Tensor
    W2: torch.Tensor
    gamma: torch.Tensor
    eps: float
    W_down: torch.Tensor | None = None


def block_inputs(M: int, K: int, N: int, N2: int, seed: int, w_std: float,
                 with_down: bool = False, F: int | None = None) -> BlockInputs:
    """Inputs of a GEMM-RMSNorm-GEMM block: h = x W1 + res, out = RMSNorm(h) W2.

    ``K`` is the width of x, ``N`` the hidden size (width of h), ``N2`` the
    width of the second GEMM.  With ``with_down`` the down-projection weight
    W_down[F, N] of the SwiGLU continuation is drawn next (F = N2 / 2).
    """
    g = make_gen(seed)
    x = normal_bf16(g, (M, K))
    res = normal_bf16(g, (M, N))
    W1 = normal_bf16(g, (K, N), std=w_std)
    W2 = normal_bf16(g, (N, N2), std=w_std)
    gamma = gamma_bf16(g, N)
    W_down = None
    if with_down:
        F = N2 // 2 if F is None else F
        W_down = normal_bf16(g, (F, N), std=w_std)
    return BlockInputs(x, res, W1, W2, gamma, EPS, W_down)


def tiny_block() -> BlockInputs:
    """256 tokens, hidden 512, second GEMM 1536; seed 0; W std 1/sqrt(512)."""
    return block_inputs(256, 512, 512, 1536, seed=0, w_std=1.0 / math.sqrt(512))


def llama1b_block_tail(with_down: bool = True) -> BlockInputs:
    """8192 tokens (batch 4 x seq 2048), hidden 2048, fused gate/up 16384; seed 1."""
    return block_inputs(8192, 2048, 2048, 16384, seed=1, w_std=0.02, with_down=with_down)


def lmhead_ce_inputs(M: int = 8192, K: int = 2048, V: int = 128256, seed: int = 3,
                     w_std: float = 0.02):
    """H[M,K] ~ N(0,1), W_vocab[K,V] std 0.02, labels uniform in [0,V)."""
    g = make_gen(seed)
    H = normal_bf16(g, (M, K))
    W = normal_bf16(g, (K, V), std=w_std)
    labels = labels_uniform(g, M, V)
    return H, W, labels


def block_backward_dout(M: int = 8192, N2: int = 16384, seed: int = 4, std: float = 0.01):
    """Upstream gradient of the block output, std 0.01."""
    g = make_gen(seed)
    return normal_bf16(g, (M, N2), std=std)


def bf16_bits(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 bit patterns (what the oracle widens itself)."""
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).numpy().view("uint16")
