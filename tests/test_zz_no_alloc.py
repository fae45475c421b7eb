"""The forward entry point for callers that cannot allocate device memory when
they call in (for example a plugin run from another runtime's launch callback,
where cudaMalloc is not allowed).  It takes no workspace: its scratch is a static
device array inside the library.  Its results must match qlora_linear_fwd's
within the tolerance the parity tests use, on consecutive calls that reuse the
shared scratch."""

import ctypes

import numpy as np
import pytest
import torch

from bit_nf4_quantized_27_b200 import binding as bd
from bit_nf4_quantized_27_b200 import inputs as I
from bit_nf4_quantized_27_b200.build import build

SCRATCH_BYTES = 256 + 2 * 1024 * 1024
TOL = 1e-2


def _fn():
    build()
    f = bd.lib().qlora_linear_fwd_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.POINTER(bd.NF4TensorC), ctypes.POINTER(bd.LoraC), ctypes.c_void_p, ctypes.c_int64,
                  ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]
    return f


def test_rejects_sizes_beyond_its_scratch():
    # host-side check, before any device work: M * r * 2 bytes over the limit
    f = _fn()
    t = bd.NF4TensorC(64, 64, 0x1000, 0x2000, 0x3000)
    ad = bd.LoraC(64, 16.0, 0x4000, 0x5000)
    too_many = SCRATCH_BYTES // (64 * 2) + 1
    assert f(ctypes.byref(t), ctypes.byref(ad), ctypes.c_void_p(0x6000), too_many, ctypes.c_void_p(0x7000), 1,
             None, None) == 2


@pytest.mark.parametrize("m,expect_size_error", [(16384, False), (16385, True)])
def test_size_limit_boundary(m, expect_size_error):
    # 256 status bytes + M * 64 * 2 bytes of s*T: 16384 tokens at rank 64 fill the
    # scratch exactly, one token more does not.  X is NULL, so a call that gets
    # past the size check stops at a later host check (no device here, or the
    # NULL X) and launches nothing.
    f = _fn()
    t = bd.NF4TensorC(64, 64, 0x1000, 0x2000, 0x3000)
    ad = bd.LoraC(64, 16.0, 0x4000, 0x5000)
    rc = f(ctypes.byref(t), ctypes.byref(ad), None, m, ctypes.c_void_p(0x7000), 1, None, None)
    if expect_size_error:
        assert rc == 2
    else:
        assert rc in (1, 8), rc  # QLORA_ERR_INVALID_ARGUMENT (NULL X) or QLORA_ERR_NO_DEVICE


def _close(got: torch.Tensor, want: torch.Tensor):
    g = got.float().cpu().numpy().astype(np.float64)
    w = want.float().cpu().numpy().astype(np.float64)
    rms = float(np.sqrt(np.mean(w ** 2)))
    assert np.all(np.isfinite(g))
    assert float(np.max(np.abs(g - w))) <= TOL * rms


@pytest.mark.gpu
def test_matches_workspace_entry_point_on_consecutive_calls():
    f = _fn()
    stream = torch.cuda.current_stream()
    # two different layers in a row: a tensor-core-path shape, then a decode shape
    for n, k, m, r, seed in ((1024, 512, 300, 64, 11), (328, 576, 4, 16, 12)):
        w, x, a, b, _ = I.custom(n, k, m, r, seed)
        w, x, a, b = w.cuda(), x.cuda(), a.cuda(), b.cuda()
        q = bd.quantize(w)
        y_ref, t_ref = bd.linear_fwd(q, a, b, 16.0, x, y_dtype=torch.float32)
        y = torch.empty(m, n, dtype=torch.float32, device="cuda")
        t = torch.empty(2, m, r, dtype=torch.bfloat16, device="cuda")
        tq, ad = q.c_struct(), bd.LoraC(r, 16.0, a.data_ptr(), b.data_ptr())
        rc = f(ctypes.byref(tq), ctypes.byref(ad), ctypes.c_void_p(x.data_ptr()), m, ctypes.c_void_p(y.data_ptr()),
               bd.QLORA_F32, ctypes.c_void_p(t.data_ptr()), ctypes.c_void_p(stream.cuda_stream))
        assert rc == 0
        torch.cuda.synchronize()
        _close(y, y_ref)
        _close(t[0].float() + t[1].float(), t_ref[0].float() + t_ref[1].float())
