"""Seeded synthetic inputs for the decode operators.

This module holds no arithmetic of the operators themselves: it only draws
random tensors and builds position-id layouts.  The GPU path (tests, bench,
smoke) and the CPU oracle both take their inputs from here, so they see the
same bits.

Recipe (one NumPy ``default_rng(seed)`` stream per tensor, seeds counted up in
the order the tensors are listed for a workload):
  * values are drawn in fp64 as ``mean + std * N(0, 1)``, cast to fp32 and then,
    for bf16 workloads, to bf16 by torch's round-to-nearest-even cast;
  * activations x ~ N(0, 1); residual ~ N(0, 2^2); gate ~ N(0, 2^2); up ~ N(0, 1);
    q, k ~ N(0, 1); norm weights gamma = 1 + 0.1 * N(0, 1);
  * M-RoPE position ids are int32 [3, tokens] (rows t, h, w).  The first
    ``text_tokens`` tokens are text: all three rows equal the token index.  The
    remaining tokens are an audio/vision-like grid: for the i-th of them,
    t = text_tokens + i // (gh * gw), h = (i // gw) % gh, w = i % gw.

Shapes follow a 1.7B-parameter speech decoder: hidden 2048, MLP width 6144,
16 query heads and 8 key heads of dimension 128, 28 layers.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

HIDDEN = 2048
INTER = 6144
N_Q_HEADS = 16
N_K_HEADS = 8
HEAD_DIM = 128
LAYERS = 28
SECTIONS = (24, 20, 20)
THETA = 1.0e6
EPS = 1.0e-6

_TORCH_DTYPE = {"bf16": torch.bfloat16, "f32": torch.float32}


def torch_dtype(dtype: str) -> torch.dtype:
    return _TORCH_DTYPE[dtype]


def normal(shape, seed: int, mean: float = 0.0, std: float = 1.0, dtype: str = "bf16") -> torch.Tensor:
    """CPU tensor of ``mean + std * N(0,1)`` drawn in fp64 from ``default_rng(seed)``."""
    rng = np.random.default_rng(seed)
    v = rng.standard_normal(size=shape)
    if std != 1.0:
        v *= std
    if mean != 0.0:
        v += mean
    t = torch.from_numpy(v).to(torch.float32)
    return t.to(_TORCH_DTYPE[dtype])


def rmsnorm_inputs(rows: int, hidden: int, dtype: str = "f32", seed: int = 0) -> dict:
    """x [rows, hidden] ~ N(0,1) (seed), gamma [hidden] = 1 + 0.1 N(0,1) (seed+1)."""
    return {
        "x": normal((rows, hidden), seed, dtype=dtype),
        "gamma": normal((hidden,), seed + 1, mean=1.0, std=0.1, dtype=dtype),
    }


def add_rmsnorm_inputs(rows: int, hidden: int, dtype: str = "bf16", seed: int = 0) -> dict:
    """x ~ N(0,1) (seed), residual ~ N(0,2^2) (seed+1), gamma (seed+2)."""
    return {
        "x": normal((rows, hidden), seed, dtype=dtype),
        "residual": normal((rows, hidden), seed + 1, std=2.0, dtype=dtype),
        "gamma": normal((hidden,), seed + 2, mean=1.0, std=0.1, dtype=dtype),
    }


def swiglu_inputs(rows: int, inter: int, dtype: str = "bf16", seed: int = 0) -> dict:
    """gate ~ N(0,2^2) (seed), up ~ N(0,1) (seed+1), separate [rows, inter] tensors."""
    return {
        "gate": normal((rows, inter), seed, std=2.0, dtype=dtype),
        "up": normal((rows, inter), seed + 1, dtype=dtype),
    }


def mrope_positions(tokens: int, text_tokens: int = 1024, grid=(8, 8)) -> torch.Tensor:
    """int32 [3, tokens] position ids: a text prefix, then a t/h/w grid."""
    gh, gw = grid
    pos = np.empty((3, tokens), dtype=np.int32)
    n_text = min(tokens, text_tokens)
    pos[:, :n_text] = np.arange(n_text, dtype=np.int32)
    i = np.arange(tokens - n_text, dtype=np.int64)
    pos[0, n_text:] = text_tokens + i // (gh * gw)
    pos[1, n_text:] = (i // gw) % gh
    pos[2, n_text:] = i % gw
    return torch.from_numpy(pos)


def mrope_inputs(tokens: int, n_q_heads: int = N_Q_HEADS, n_k_heads: int = N_K_HEADS,
                 head_dim: int = HEAD_DIM, dtype: str = "bf16", seed: int = 0,
                 text_tokens: int = 1024) -> dict:
    """q [T, Hq, D] (seed), k [T, Hk, D] (seed+1), both N(0,1); pos [3, T]."""
    return {
        "q": normal((tokens, n_q_heads, head_dim), seed, dtype=dtype),
        "k": normal((tokens, n_k_heads, head_dim), seed + 1, dtype=dtype),
        "pos": mrope_positions(tokens, text_tokens),
    }


def topk_inputs(rows: int, vocab: int, top_k: int, dtype: str = "bf16", seed: int = 0,
                std: float = 3.0) -> dict:
    """logits [rows, vocab] ~ N(0, std^2) (seed); gumbel [rows, top_k] float32
    Gumbel(0,1) draws from default_rng(seed + 1)."""
    rng = np.random.default_rng(seed + 1)
    return {
        "logits": normal((rows, vocab), seed, std=std, dtype=dtype),
        "gumbel": torch.from_numpy(rng.gumbel(size=(rows, top_k)).astype(np.float32)),
    }


@dataclass
class ChainShape:
    """Shape of the decode-step chain: per layer add+RMSNorm, M-RoPE on q/k,
    add+RMSNorm, SwiGLU, over ``batch`` candidates (one new token each)."""

    batch: int = 5
    layers: int = LAYERS
    hidden: int = HIDDEN
    inter: int = INTER
    n_q_heads: int = N_Q_HEADS
    n_k_heads: int = N_K_HEADS
    head_dim: int = HEAD_DIM


def decode_chain_inputs(shape: ChainShape, dtype: str = "bf16", seed: int = 0) -> dict:
    """Per-layer seeded buffers for the decode chain.

    Seeds: the starting residual [B, H] ~ N(0, 2^2) takes ``seed``; layer l takes
    seeds seed + 1 + 8 l ... seed + 8 + 8 l for, in order, x_attn, gamma_attn, q,
    k, x_mlp, gamma_mlp, gate, up.
    """
    B, H, I = shape.batch, shape.hidden, shape.inter
    out = {"residual": normal((B, H), seed, std=2.0, dtype=dtype)}
    keys = ("x_attn", "gamma_attn", "q", "k", "x_mlp", "gamma_mlp", "gate", "up")
    for key in keys:
        out[key] = []
    for layer in range(shape.layers):
        s = seed + 1 + 8 * layer
        out["x_attn"].append(normal((B, H), s, dtype=dtype))
        out["gamma_attn"].append(normal((H,), s + 1, mean=1.0, std=0.1, dtype=dtype))
        out["q"].append(normal((B, shape.n_q_heads, shape.head_dim), s + 2, dtype=dtype))
        out["k"].append(normal((B, shape.n_k_heads, shape.head_dim), s + 3, dtype=dtype))
        out["x_mlp"].append(normal((B, H), s + 4, dtype=dtype))
        out["gamma_mlp"].append(normal((H,), s + 5, mean=1.0, std=0.1, dtype=dtype))
        out["gate"].append(normal((B, I), s + 6, std=2.0, dtype=dtype))
        out["up"].append(normal((B, I), s + 7, dtype=dtype))
    return out


def decode_positions(step: int, batch: int) -> torch.Tensor:
    """Position ids of decode step ``step``: every row (t, h, w) equals the step."""
    return torch.full((3, batch), step, dtype=torch.int32)
