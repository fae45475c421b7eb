"""The seeded input generators shared by the oracle and the CUDA path (CPU only)."""

import itertools
import math

import numpy as np
import torch

from bit_nf4_quantized_27_b200 import inputs as I


def test_seeds_are_distinct_within_and_across_workloads():
    seen = {}
    for wl in (I.TINY, I.QUANT_4096, I.GEMV, I.LLAMA7B_BLOCK, I.L65B_BLOCK):
        for layer, tid in itertools.product(range(len(wl.layers)), (I.W_ID, I.X_ID, I.A_ID, I.B_ID, I.DY_ID)):
            s = I.seed_for(wl.wid, tid, layer)
            assert s not in seen, (wl.name, layer, tid, seen.get(s))
            seen[s] = (wl.name, layer, tid)


def test_same_seed_same_bytes_and_dtype():
    a = I.weight(I.LLAMA7B_BLOCK, 2)
    b = I.weight(I.LLAMA7B_BLOCK, 2)
    assert a.dtype == torch.bfloat16 and torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert not torch.equal(a, I.weight(I.LLAMA7B_BLOCK, 3))
    assert I.weight(I.TINY).dtype == torch.float32


def test_values_are_the_storage_rounding_of_scaled_normals():
    g = torch.Generator("cpu")
    g.manual_seed(I.seed_for(I.GEMV.wid, I.X_ID, 0))
    ref = (torch.randn(I.GEMV.m, 4096, generator=g) * 1.0).to(torch.bfloat16)
    assert torch.equal(I.activations(I.GEMV).view(torch.int16), ref.view(torch.int16))


def test_shapes_and_standard_deviations():
    wl = I.LLAMA7B_BLOCK
    ly = wl.layers[4]  # gate: 4096 -> 11008
    w, x, a, b, dy = (I.weight(wl, 4), I.activations(wl, 4), I.lora_a(wl, 4), I.lora_b(wl, 4),
                      I.grad_output(wl, 4))
    assert tuple(w.shape) == (ly.n, ly.k) == (11008, 4096)
    assert tuple(x.shape) == (wl.m, ly.k) and tuple(dy.shape) == (wl.m, ly.n)
    assert tuple(a.shape) == (wl.r, ly.k) and tuple(b.shape) == (ly.n, wl.r)
    for t, std in ((w, 0.02), (x, 1.0), (a, 1 / math.sqrt(ly.k)), (b, 0.01), (dy, 1.0)):
        v = t.float().numpy().astype(np.float64)
        assert abs(v.mean()) < 0.02 * std
        assert abs(v.std() / std - 1) < 0.02


def test_block_layer_shapes():
    for wl, h, f in ((I.LLAMA7B_BLOCK, 4096, 11008), (I.L65B_BLOCK, 8192, 22016)):
        assert [ly.name for ly in wl.layers] == ["q", "k", "v", "o", "gate", "up", "down"]
        assert [(ly.n, ly.k) for ly in wl.layers] == [(h, h)] * 4 + [(f, h)] * 2 + [(h, f)]
    assert (I.LLAMA7B_BLOCK.m, I.L65B_BLOCK.m, I.GEMV.m, I.TINY.m) == (2048, 4096, 16, 16)
    assert (I.GEMV.r, I.LLAMA7B_BLOCK.r, I.TINY.r) == (64, 64, 8)
