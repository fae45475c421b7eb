"""Data parallelism for the NF4 linear layers with LoRA.

Every rank holds the same frozen NF4 weights and LoRA adapters and runs its own
tokens.  The layer's outputs and input gradients are per-token, so they need no
exchange; the adapter gradients dA = s U^T X and dB = s dY^T T are sums over
tokens, so summing each rank's dA, dB over the ranks gives exactly the gradient
of the whole batch.  That sum is the only collective: one all-reduce per step
over a single flat fp32 buffer holding every layer's dA and dB.
"""

from __future__ import annotations

import torch


def flat_size(layer_shapes, r: int) -> int:
    """Elements of the flat gradient buffer for layers [(N, K), ...] at rank r."""
    return sum(r * k + n * r for n, k in layer_shapes)


def grad_views(flat: torch.Tensor, layer_shapes, r: int):
    """Views (dA [r, K], dB [N, r]) into `flat`, one pair per layer, in order."""
    if flat.numel() != flat_size(layer_shapes, r):
        raise ValueError("flat buffer size does not match the layer shapes")
    views, off = [], 0
    for n, k in layer_shapes:
        da = flat[off:off + r * k].view(r, k)
        off += r * k
        db = flat[off:off + n * r].view(n, r)
        off += n * r
        views.append((da, db))
    return views


def token_shard(m_total: int, world: int, rank: int) -> slice:
    """Contiguous token rows of `rank` when m_total tokens are split over `world`."""
    per = (m_total + world - 1) // world
    lo = min(m_total, rank * per)
    return slice(lo, min(m_total, lo + per))


def allreduce_grads(flat: torch.Tensor, group=None) -> None:
    """Sum the adapter gradients over the ranks (in place)."""
    import torch.distributed as dist

    if dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)
