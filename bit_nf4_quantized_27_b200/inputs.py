"""Seeded synthetic inputs for the NF4 linear-layer workloads.

This module holds none of the method's arithmetic: it draws normal numbers from
fixed seeds, scales them, and rounds them to the storage dtype.  The CPU oracle
(tests only) and the CUDA path both read the bytes it returns.

Recipe (one ``torch.Generator('cpu')`` per tensor):

  seed = 20260000 + 100 * workload_id + tensor_id + 10 * layer
  tensor ids: W = 1, X = 2, A = 3, B = 4, dY = 5
  values = randn(shape) * std, then round-to-nearest-even to the storage dtype

Standard deviations: W 0.02 (the glossary snippet's randn * 0.02), X and dY 1,
LoRA A with variance 1/K (so X A^T has unit variance), LoRA B 0.01.  The normal
weights stand in for pretrained weights, as the QLoRA glossary page assumes.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

W_ID, X_ID, A_ID, B_ID, DY_ID = 1, 2, 3, 4, 5


def seed_for(workload_id: int, tensor_id: int, layer: int = 0) -> int:
    return 20260000 + 100 * workload_id + tensor_id + 10 * layer


def normal(shape, std: float, seed: int, dtype=torch.bfloat16) -> torch.Tensor:
    """randn(shape) * std from a fresh CPU generator, rounded to ``dtype``."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return (torch.randn(*shape, generator=g, dtype=torch.float32) * std).to(dtype)


@dataclass(frozen=True)
class Layer:
    name: str
    n: int          # out_features (rows of W)
    k: int          # in_features (cols of W)


@dataclass(frozen=True)
class Workload:
    wid: int
    name: str
    m: int                      # tokens
    r: int
    alpha: float
    layers: tuple = field(default_factory=tuple)
    w_dtype: torch.dtype = torch.bfloat16


def _block(hidden: int, inter: int):
    return (Layer("q", hidden, hidden), Layer("k", hidden, hidden), Layer("v", hidden, hidden),
            Layer("o", hidden, hidden), Layer("gate", inter, hidden), Layer("up", inter, hidden),
            Layer("down", hidden, inter))


# The five workloads: sizes as the QLoRA pages and the model shapes they name.
TINY = Workload(1, "tiny_256x256_m16_r8", 16, 8, 16.0, (Layer("w", 256, 256),), torch.float32)
QUANT_4096 = Workload(2, "quant_4096x4096", 0, 0, 0.0, (Layer("w", 4096, 4096),))
QUANT_11008 = Workload(2, "quant_11008x4096", 0, 0, 0.0, (Layer("w", 11008, 4096),))
GEMV = Workload(3, "gemv_11008x4096_r64", 16, 64, 16.0, (Layer("up", 11008, 4096),))
LLAMA7B_BLOCK = Workload(4, "llama7b_block_m2048_r64", 2048, 64, 16.0, _block(4096, 11008))
L65B_BLOCK = Workload(5, "65b_block_m4096_r64", 4096, 64, 16.0, _block(8192, 22016))

WORKLOADS = {w.name: w for w in (TINY, QUANT_4096, QUANT_11008, GEMV, LLAMA7B_BLOCK, L65B_BLOCK)}


def weight(wl: Workload, layer: int = 0, std: float = 0.02) -> torch.Tensor:
    ly = wl.layers[layer]
    return normal((ly.n, ly.k), std, seed_for(wl.wid, W_ID, layer), wl.w_dtype)


def activations(wl: Workload, layer: int = 0, m: int | None = None) -> torch.Tensor:
    ly = wl.layers[layer]
    return normal((wl.m if m is None else m, ly.k), 1.0, seed_for(wl.wid, X_ID, layer))


def lora_a(wl: Workload, layer: int = 0) -> torch.Tensor:
    ly = wl.layers[layer]
    return normal((wl.r, ly.k), 1.0 / math.sqrt(ly.k), seed_for(wl.wid, A_ID, layer))


def lora_b(wl: Workload, layer: int = 0, std: float = 0.01) -> torch.Tensor:
    ly = wl.layers[layer]
    return normal((ly.n, wl.r), std, seed_for(wl.wid, B_ID, layer))


def grad_output(wl: Workload, layer: int = 0, m: int | None = None) -> torch.Tensor:
    ly = wl.layers[layer]
    return normal((wl.m if m is None else m, ly.n), 1.0, seed_for(wl.wid, DY_ID, layer))


def custom(n: int, k: int, m: int, r: int, seed: int, w_std: float = 0.02,
           w_dtype=torch.bfloat16, b_std: float = 0.01):
    """Inputs of arbitrary shape for parity sweeps (ragged tails, odd sizes).
    Returns (W, X, A, B, dY) with the same distributions as the workloads."""
    w = normal((n, k), w_std, seed + W_ID, w_dtype)
    x = normal((m, k), 1.0, seed + X_ID)
    a = normal((r, k), 1.0 / math.sqrt(k), seed + A_ID)
    b = normal((n, r), b_std, seed + B_ID)
    dy = normal((m, n), 1.0, seed + DY_ID)
    return w, x, a, b, dy


def keep_mask(m: int, k: int, p: float, seed: int) -> torch.Tensor:
    """Drawn dropout keep mask for [m, k] (each element kept with probability
    1 - p), packed one bit per element: bit (j % 8) of byte j // 8 of row i.
    Returns uint8 [m, k // 8] (k % 8 == 0)."""
    g = torch.Generator().manual_seed(seed)
    keep = torch.rand((m, k), generator=g, dtype=torch.float64) >= p
    weights = (1 << torch.arange(8, dtype=torch.int32))
    return (keep.view(m, k // 8, 8).to(torch.int32) * weights).sum(-1).to(torch.uint8)
