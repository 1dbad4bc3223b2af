"""Seeded synthetic inputs shared by the tests, ``bench.py`` and ``smoke()``.

This module only draws random numbers. It holds none of ClusterKV's arithmetic, so
both the CPU oracle and the CUDA path can take their inputs from it.

The workload follows the shapes on the ClusterKV pages: Llama-3.1-8B-like GQA heads
(head_dim 128, 8 KV heads, 32 query heads), a 32k context and a 1k-2k budget. The pages
name no dataset and print no tensors, so the keys are a clustered mixture:

* centers ``c_j = normalize(N(0, I_128))``, ``j < n_centers``, drawn per (layer, b, kv-head);
* each token draws a center uniformly and sets ``k = scale * (c_j + sigma * N(0, I))``,
  with ``sigma = 0.3`` and ``scale = 8``;
* values ``v ~ N(0, 1)`` and queries ``q ~ N(0, 1)``.

Every tensor is rounded to bf16 (round-to-nearest-even) and returned as its raw
``uint16`` bit pattern. Token order is i.i.d., so there is no positional locality.

Each (layer, b, kv-head) unit draws from its own counter-based Philox stream, keyed by
``(config_seed, tag << 40 | unit)``. A unit can therefore be regenerated on its own,
which lets the tests rebuild any sampled unit of a large workload on the CPU. The
``*_torch`` variants follow the same recipe with ``torch.Generator`` on any device.
They serve only as filler for units that no check reads.
"""
from __future__ import annotations

import numpy as np
import torch

D = 128
TAG_CENTERS, TAG_KEYS, TAG_VALUES, TAG_QUERIES, TAG_APPEND = 1, 2, 3, 4, 5


def unit_id(layer: int, b: int, h: int, batch: int, n_kv_heads: int) -> int:
    """Flat index of one (layer, sequence, KV head) unit."""
    return (layer * batch + b) * n_kv_heads + h


def _rng(config_seed: int, tag: int, idx: int) -> np.random.Generator:
    key = np.array([config_seed & (2**64 - 1), ((tag << 40) | idx) & (2**64 - 1)], dtype=np.uint64)
    return np.random.Generator(np.random.Philox(key=key))


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32/float64 array -> bf16 bit patterns (uint16), round-to-nearest-even."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32)


def centers(config_seed: int, unit: int, n_centers: int) -> np.ndarray:
    g = _rng(config_seed, TAG_CENTERS, unit)
    c = g.standard_normal((n_centers, D))
    return c / np.linalg.norm(c, axis=1, keepdims=True)


def _mixture(g: np.random.Generator, cen: np.ndarray, count: int, sigma: float, scale: float,
             labels: bool = False):
    j = g.integers(0, cen.shape[0], size=count)
    k = scale * (cen[j] + sigma * g.standard_normal((count, D)))
    return (k, j) if labels else k


def keys_values(config_seed: int, unit: int, n: int, n_centers: int,
                sigma: float = 0.3, scale: float = 8.0):
    """K, V of one unit: ``[n, 128]`` bf16 bit patterns each."""
    return keys_values_labeled(config_seed, unit, n, n_centers, sigma, scale)[:2]


def keys_values_labeled(config_seed: int, unit: int, n: int, n_centers: int,
                        sigma: float = 0.3, scale: float = 8.0):
    """K, V of one unit plus the mixture component each token was drawn from."""
    cen = centers(config_seed, unit, n_centers)
    k, j = _mixture(_rng(config_seed, TAG_KEYS, unit), cen, n, sigma, scale, labels=True)
    v = _rng(config_seed, TAG_VALUES, unit).standard_normal((n, D))
    return to_bf16_bits(k), to_bf16_bits(v), j.astype(np.int32)


def appended_tokens(config_seed: int, unit: int, count: int, n_centers: int,
                    sigma: float = 0.3, scale: float = 8.0):
    """K, V of ``count`` generated tokens of one unit, drawn from the same mixture."""
    cen = centers(config_seed, unit, n_centers)
    g = _rng(config_seed, TAG_APPEND, unit)
    k = _mixture(g, cen, count, sigma, scale)
    v = g.standard_normal((count, D))
    return to_bf16_bits(k), to_bf16_bits(v)


def queries(config_seed: int, layer: int, b: int, steps: int, n_q_heads: int) -> np.ndarray:
    """Decode queries of one (layer, sequence): ``[steps, n_q_heads, 128]`` bf16 bits."""
    g = _rng(config_seed, TAG_QUERIES, (layer << 20) | b)
    return to_bf16_bits(g.standard_normal((steps, n_q_heads, D)))


def layer_kv(config_seed: int, layer: int, batch: int, n_kv_heads: int, n: int, n_centers: int):
    """K, V of one layer: ``[batch, n_kv_heads, n, 128]`` bf16 bits each."""
    K = np.empty((batch, n_kv_heads, n, D), np.uint16)
    V = np.empty_like(K)
    for b in range(batch):
        for h in range(n_kv_heads):
            u = unit_id(layer, b, h, batch, n_kv_heads)
            K[b, h], V[b, h] = keys_values(config_seed, u, n, n_centers)
    return K, V


def _torch_gen(config_seed: int, tag: int, idx: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(((config_seed * 1000003) ^ (tag << 40) ^ idx) & (2**63 - 1))
    return g


def keys_values_torch(config_seed: int, unit: int, n: int, n_centers: int, device,
                      sigma: float = 0.3, scale: float = 8.0):
    """Same recipe as :func:`keys_values` drawn with ``torch.Generator`` on ``device``.

    Returns bf16 tensors ``[n, 128]``. The stream differs from the numpy one. It fills
    units that no parity check reads, such as the bench's extra layer stores.
    """
    g = _torch_gen(config_seed, TAG_CENTERS, unit, device)
    cen = torch.randn(n_centers, D, generator=g, device=device)
    cen = cen / cen.norm(dim=1, keepdim=True)
    g = _torch_gen(config_seed, TAG_KEYS, unit, device)
    j = torch.randint(0, n_centers, (n,), generator=g, device=device)
    k = scale * (cen[j] + sigma * torch.randn(n, D, generator=g, device=device))
    g = _torch_gen(config_seed, TAG_VALUES, unit, device)
    v = torch.randn(n, D, generator=g, device=device)
    return k.to(torch.bfloat16), v.to(torch.bfloat16)


def queries_torch(config_seed: int, layer: int, b: int, steps: int, n_q_heads: int, device):
    g = _torch_gen(config_seed, TAG_QUERIES, (layer << 20) | b, device)
    return torch.randn(steps, n_q_heads, D, generator=g, device=device).to(torch.bfloat16)


def appended_tokens_torch(config_seed: int, unit: int, count: int, n_centers: int, device,
                          sigma: float = 0.3, scale: float = 8.0):
    """Same recipe as :func:`appended_tokens` drawn with ``torch.Generator`` on ``device``."""
    g = _torch_gen(config_seed, TAG_CENTERS, unit, device)
    cen = torch.randn(n_centers, D, generator=g, device=device)
    cen = cen / cen.norm(dim=1, keepdim=True)
    g = _torch_gen(config_seed, TAG_APPEND, unit, device)
    j = torch.randint(0, n_centers, (count,), generator=g, device=device)
    k = scale * (cen[j] + sigma * torch.randn(count, D, generator=g, device=device))
    v = torch.randn(count, D, generator=g, device=device)
    return k.to(torch.bfloat16), v.to(torch.bfloat16)
