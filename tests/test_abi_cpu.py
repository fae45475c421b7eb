"""The C-ABI library loads, exports every declared symbol, and its host-side
logic (sizes, table, argument checks) behaves without a GPU."""

import ctypes

import numpy as np
import pytest

import oracle as O
from bit_nf4_quantized_27_b200 import binding as bd
from bit_nf4_quantized_27_b200.build import build


@pytest.fixture(scope="module")
def L():
    build()
    return bd.lib()


def test_exports_every_declared_symbol(L):
    names = bd.header_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(L, n), n


def test_abi_version(L):
    assert L.qlora_abi_version() == 2


def test_codebook_equals_oracle_bit_for_bit(L):
    got = np.array(bd.codebook(), dtype=np.float32)
    assert np.array_equal(got.view(np.uint32), O.nf4_levels().view(np.uint32))


@pytest.mark.parametrize("rows,cols", [(256, 256), (4096, 4096), (11008, 4096), (3, 64), (1, 64 * 300)])
def test_storage_bytes_match_oracle(L, rows, cols):
    total, c, s, g = bd.storage_bytes(rows, cols)
    oc, os_, og = O.storage_bytes(rows, cols)
    assert (c, s, g) == (oc, os_, og) and total == c + s + g


def test_storage_bytes_rejects_bad_cols(L):
    assert bd.storage_bytes(4, 65)[0] == 0
    assert bd.storage_bytes(0, 64)[0] == 0


def test_workspace_bytes(L):
    assert bd.workspace_bytes(16, 11008, 4096, 64, False) >= 256 + 16 * 64 * 2
    assert bd.workspace_bytes(2048, 4096, 4096, 64, True) >= 256 + 2 * 2048 * 64 * 2
    assert bd.workspace_bytes(0, 1, 64, 8, False) == 0
    assert bd.workspace_bytes(1, 1, 64, 512, False) == 0


def _t(rows, cols, codes=0x1000, sc=0x2000, c2=0x3000):
    return bd.NF4TensorC(rows, cols, codes, sc, c2)


def test_argument_checks_without_gpu(L):
    # Every check runs before any device work; fake (never dereferenced) pointers.
    W, ws = ctypes.c_void_p(0x10000), ctypes.c_void_p(0x20000)
    good = _t(64, 64)
    assert L.qlora_nf4_quantize(W, 1, ctypes.byref(_t(64, 65)), ws, None) == 2
    assert L.qlora_nf4_quantize(W, 1, ctypes.byref(_t(64, 64, codes=0)), ws, None) == 1
    assert L.qlora_nf4_quantize(None, 1, ctypes.byref(good), ws, None) == 1
    assert L.qlora_nf4_quantize(W, 7, ctypes.byref(good), ws, None) == 1
    assert L.qlora_nf4_quantize(ctypes.c_void_p(0x10008), 1, ctypes.byref(good), ws, None) == 3
    assert L.qlora_nf4_quantize(W, 1, ctypes.byref(_t(64, 64, codes=0x1004)), ws, None) == 3
    bad_fmt = _t(64, 64)
    bad_fmt.scale_format = 3
    assert L.qlora_nf4_quantize(W, 1, ctypes.byref(bad_fmt), ws, None) == 1
    bad_fmt.scale_format = -1
    assert L.qlora_nf4_dequantize(ctypes.byref(bad_fmt), ws, 1, None) == 1
    ad = bd.LoraC(64, 16.0, 0x4000, 0x5000)
    X, Y = ctypes.c_void_p(0x6000), ctypes.c_void_p(0x7000)
    assert L.qlora_linear_fwd(ctypes.byref(good), ctypes.byref(bd.LoraC(12, 16.0, 0x4000, 0x5000)), X, 4, Y, 1,
                              None, ws, 1 << 20, None) == 1
    assert L.qlora_linear_fwd(ctypes.byref(good), ctypes.byref(ad), X, 0, Y, 1, None, ws, 1 << 20, None) == 1
    assert L.qlora_linear_fwd(ctypes.byref(good), ctypes.byref(ad), X, 4, Y, 1, None, ws, 16, None) == 4
    assert L.qlora_linear_fwd(ctypes.byref(_t(60, 64)), ctypes.byref(ad), X, 4, Y, 1, None, ws, 1 << 20, None) == 2
    assert L.qlora_linear_bwd(ctypes.byref(good), ctypes.byref(ad), X, None, 4, None, X, 1, X, X, 1, ws, 1 << 20,
                              None) == 1


def test_valid_call_without_gpu_reports_no_device(L):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    W, ws = ctypes.c_void_p(0x10000), ctypes.c_void_p(0x20000)
    assert L.qlora_nf4_quantize(W, 1, ctypes.byref(_t(64, 64)), ws, None) == 8


def test_selftest_argument_checks_without_gpu(L):
    ws = ctypes.c_void_p(0x20000)
    assert L.qlora_selftest_bounded_wait(None, 1000, None) == 1
    assert L.qlora_selftest_bounded_wait(ws, 0, None) == 1
    assert L.qlora_selftest_bounded_wait(ws, 2000001, None) == 1
    assert L.qlora_selftest_bounded_wait(ctypes.c_void_p(0x20010), 1000, None) == 3
    import torch
    if not torch.cuda.is_available():
        assert L.qlora_selftest_bounded_wait(ws, 1000, None) == 8


def test_status_strings(L):
    for code in range(9):
        assert L.qlora_status_string(code)
    assert L.qlora_status_string(0) == b"ok"


def test_device_level_literals_match_bit_patterns():
    # the kernels use the 16 levels both as float32 bit patterns and as hex-float
    # immediates; both lists, and the oracle's table, must be identical
    import os
    import re
    import struct

    src = open(os.path.join(os.path.dirname(bd.LIB_PATH), "csrc", "nf4_device.cuh")).read()
    bits_block = src[src.index("kNf4LevelBits[16] = {"):]
    bits = [int(b, 16) for b in re.findall(r"0x([0-9a-f]{8})u", bits_block[:bits_block.index("};")])]
    fn = src[src.index("constexpr float nf4_level(int j)"):]
    fn = fn[:fn.index("}")]
    lits = re.findall(r"(-?0x[0-9a-f.]+p[+-]\d+)f", fn)
    vals = [struct.unpack("<I", struct.pack("<f", float.fromhex(v)))[0] for v in lits]
    assert len(bits) == 16 and len(vals) == 16
    assert bits == vals
    assert bits == [int(x) for x in O.nf4_levels().view(np.uint32)]


def test_merge_and_adamw_argument_checks_without_gpu(L):
    good = _t(64, 64)
    ad = bd.LoraC(64, 16.0, 0x4000, 0x5000)
    out = ctypes.c_void_p(0x6000)
    assert L.qlora_lora_merge(ctypes.byref(good), ctypes.byref(ad), None, None) == 1
    assert L.qlora_lora_merge(ctypes.byref(good), ctypes.byref(ad), ctypes.c_void_p(0x6008), None) == 3
    assert L.qlora_lora_merge(ctypes.byref(good), ctypes.byref(bd.LoraC(12, 16.0, 0x4000, 0x5000)), out, None) == 1
    assert L.qlora_lora_merge(ctypes.byref(_t(64, 65)), ctypes.byref(ad), out, None) == 2
    p, g, m, v, h = (ctypes.c_void_p(a) for a in (0x10000, 0x20000, 0x30000, 0x40000, 0x50000))
    hp = bd.AdamWC(1e-3, 0.9, 0.999, 1e-8, 0.01)
    assert L.qlora_adamw_step(p, h, g, m, v, 0, ctypes.byref(hp), 1, None) == 1
    assert L.qlora_adamw_step(p, h, g, m, v, 10, ctypes.byref(hp), 0, None) == 1
    assert L.qlora_adamw_step(p, h, g, m, v, 10, ctypes.byref(bd.AdamWC(1e-3, 1.0, 0.999, 1e-8, 0.0)), 1, None) == 1
    assert L.qlora_adamw_step(p, h, g, m, v, 10, ctypes.byref(bd.AdamWC(1e-3, 0.9, 0.999, 0.0, 0.0)), 1, None) == 1
    assert L.qlora_adamw_step(p, h, None, m, v, 10, ctypes.byref(hp), 1, None) == 1
    assert L.qlora_adamw_step(ctypes.c_void_p(0x10004), h, g, m, v, 10, ctypes.byref(hp), 1, None) == 3
    assert L.qlora_adamw_step(p, ctypes.c_void_p(0x50002), g, m, v, 10, ctypes.byref(hp), 1, None) == 3
    import torch
    if not torch.cuda.is_available():
        assert L.qlora_adamw_step(p, None, g, m, v, 10, ctypes.byref(hp), 1, None) == 8
        assert L.qlora_lora_merge(ctypes.byref(good), ctypes.byref(ad), out, None) == 8


def test_multi_adapter_argument_checks_without_gpu(L):
    good = _t(1024, 1024)
    ads = (bd.LoraC * 2)(bd.LoraC(16, 16.0, 0x4000, 0x5000), bd.LoraC(16, 8.0, 0x6000, 0x7000))
    idx = (ctypes.c_int32 * 3)(0, 1, 1)
    X, Y, ws = ctypes.c_void_p(0x10000), ctypes.c_void_p(0x20000), ctypes.c_void_p(0x30000)
    f = L.qlora_linear_fwd_multi
    assert f(ctypes.byref(good), ads, 2, idx, X, 3, Y, 1, ws, 1 << 20, None) in (0, 8)  # valid (no GPU: 8)
    bad_idx = (ctypes.c_int32 * 3)(0, 2, 1)
    assert f(ctypes.byref(good), ads, 2, bad_idx, X, 3, Y, 1, ws, 1 << 20, None) == 1
    assert f(ctypes.byref(good), ads, 2, idx, X, 17, Y, 1, ws, 1 << 20, None) == 1
    assert f(ctypes.byref(good), ads, 0, idx, X, 3, Y, 1, ws, 1 << 20, None) == 1
    mixed = (bd.LoraC * 2)(bd.LoraC(16, 16.0, 0x4000, 0x5000), bd.LoraC(32, 8.0, 0x6000, 0x7000))
    assert f(ctypes.byref(good), mixed, 2, idx, X, 3, Y, 1, ws, 1 << 20, None) == 1
    assert f(ctypes.byref(_t(1024, 576)), ads, 2, idx, X, 3, Y, 1, ws, 1 << 20, None) == 2
    assert f(ctypes.byref(good), ads, 2, idx, X, 3, Y, 1, ws, 64, None) == 4


def test_dropout_argument_checks_without_gpu(L):
    good = _t(64, 64)
    ad = bd.LoraC(64, 16.0, 0x4000, 0x5000)
    X, keep, Y, ws = (ctypes.c_void_p(a) for a in (0x10000, 0x20000, 0x30000, 0x40000))
    f = L.qlora_linear_fwd_dropout
    big = 1 << 24
    assert f(ctypes.byref(good), ctypes.byref(ad), X, keep, 1.0, 32, Y, 1, None, ws, big, None) == 1
    assert f(ctypes.byref(good), ctypes.byref(ad), X, keep, -0.1, 32, Y, 1, None, ws, big, None) == 1
    assert f(ctypes.byref(good), ctypes.byref(ad), X, None, 0.1, 32, Y, 1, None, ws, big, None) == 1
    assert f(ctypes.byref(good), ctypes.byref(ad), X, ctypes.c_void_p(0x20008), 0.1, 32, Y, 1, None, ws, big,
             None) == 3
    assert f(ctypes.byref(good), ctypes.byref(ad), X, keep, 0.1, 32, Y, 1, None, ws, 64, None) == 4
    b = L.qlora_linear_bwd_dropout
    dX, dA, dB = (ctypes.c_void_p(a) for a in (0x50000, 0x60000, 0x70000))
    assert b(ctypes.byref(good), ctypes.byref(ad), X, X, keep, 1.5, 32, None, dX, 1, dA, dB, 1, ws, big, None) == 1
    assert b(ctypes.byref(good), ctypes.byref(ad), X, X, None, 0.1, 32, None, dX, 1, dA, dB, 1, ws, big, None) == 1
    # the dropout workspace holds the masked copy of X on top of the plain one
    for bwd in (0, 1):
        assert L.qlora_workspace_bytes_dropout(300, 512, 1024, 64, bwd) >= \
            L.qlora_workspace_bytes(300, 512, 1024, 64, bwd) + 300 * 1024 * 2


def test_keep_mask_generator_packs_like_the_oracle():
    import numpy as np
    import torch

    from bit_nf4_quantized_27_b200 import inputs as I

    packed = I.keep_mask(5, 48, 0.3, 11)
    assert packed.dtype == torch.uint8 and tuple(packed.shape) == (5, 6)
    g = torch.Generator().manual_seed(11)
    want = (torch.rand((5, 48), generator=g, dtype=torch.float64) >= 0.3).numpy()
    assert np.array_equal(O.unpack_keep(packed.numpy(), 5, 48), want)


def test_multi_workspace_size(L):
    for m, n, k, r in ((1, 11008, 4096, 64), (16, 11008, 4096, 64), (7, 1000, 512, 24)):
        lo = L.qlora_workspace_bytes(m, n, k, r, 0)
        assert L.qlora_workspace_bytes_multi(m, n, k, r) == lo + ((m * n * 4 + 255) // 256) * 256
    assert L.qlora_workspace_bytes_multi(17, 1024, 1024, 16) == 0
    assert L.qlora_workspace_bytes_multi(4, 1024, 1024, 300) == 0
