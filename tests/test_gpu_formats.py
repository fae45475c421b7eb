"""The alternative 8-bit scale formats (E5M2, linear byte) on the GPU against
the oracle: quantise and dequantise bit for bit, and every kernel that decodes
block scales (decode forward, two-launch GEMV, single-CTA and CTA-pair fused
GEMMs forward and backward, merged export) within the linear layer's bar."""

import numpy as np
import pytest
import torch

import oracle as O
from bit_nf4_quantized_27_b200 import binding as bd
from bit_nf4_quantized_27_b200 import inputs as I

pytestmark = pytest.mark.gpu

FORMATS = ["e5m2", "u8"]
TOL = 1e-2


def _check(name, got, ref):
    g = got.float().cpu().numpy().astype(np.float64)
    ref = np.asarray(ref, np.float64)
    rms = float(np.sqrt(np.mean(ref ** 2)))
    err = float(np.abs(g - ref).max())
    assert np.all(np.isfinite(g)), name
    assert err <= TOL * rms, f"{name}: max err {err:.3e} vs {TOL * rms:.3e}"


def _quant_both(w: torch.Tensor, fmt: str):
    rows, cols = w.shape
    ws = bd.new_workspace(bd.STATUS_BYTES)
    q = bd.quantize(w.cuda().contiguous(), ws=ws, scale_format=fmt)
    assert bd.read_status(ws) == 0
    ref = O.quantize(w.float().numpy(), rows, cols, scale_format=fmt)
    return q, ref


@pytest.mark.parametrize("fmt", FORMATS)
def test_quantise_dequantise_bit_exact(fmt):
    rows, cols = 6, 64 * 600
    g = torch.Generator().manual_seed(5)
    w = (torch.randn(rows, cols, generator=g) * 0.02).to(torch.bfloat16)
    w[0, :64 * 300] = 0                                          # a whole zero group
    w[1, 64:128] = 1e-30                                         # tiny constant block
    w[2, 64:128] *= 1e4                                          # block far above its group
    w[3, :64] = torch.tensor([1.0] + [0.5] * 63).to(torch.bfloat16)
    q, ref = _quant_both(w, fmt)
    assert np.array_equal(q.codes.cpu().numpy(), ref["codes"])
    assert np.array_equal(q.scale_codes.cpu().numpy(), ref["scale_codes"])
    assert np.array_equal(q.c2.cpu().numpy().view(np.uint32), ref["c2"].view(np.uint32))
    wd = O.dequantize(ref["codes"], ref["scale_codes"], ref["c2"], rows, cols, scale_format=fmt)
    got16 = bd.dequantize(q, torch.bfloat16).cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got16.reshape(-1), O.bf16_bits(wd.reshape(-1)))
    got32 = bd.dequantize(q, torch.float32).cpu().numpy()
    assert np.array_equal(got32.reshape(-1).view(np.uint32), wd.reshape(-1).view(np.uint32))


@pytest.mark.parametrize("fmt", FORMATS)
def test_full_size_quantise_bit_exact(fmt):
    w = I.weight(I.QUANT_4096)
    q, ref = _quant_both(w, fmt)
    assert np.array_equal(q.codes.cpu().numpy(), ref["codes"])
    assert np.array_equal(q.scale_codes.cpu().numpy(), ref["scale_codes"])
    assert np.array_equal(q.c2.cpu().numpy().view(np.uint32), ref["c2"].view(np.uint32))


@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("n,k,m,r", [(1040, 4096, 4, 64),      # one-kernel decode forward
                                     (1024, 8192, 3, 64),      # two-launch GEMV (K > 4096)
                                     (520, 1024, 100, 16),     # single-CTA fused GEMM
                                     (1024, 512, 300, 64)])    # CTA-pair fused GEMM
def test_linear_fwd_bwd(fmt, n, k, m, r):
    w, x, a, b, dy = I.custom(n, k, m, r, 7 * n + k + m)
    q, ref = _quant_both(w, fmt)
    wd = O.dequantize(ref["codes"], ref["scale_codes"], ref["c2"], n, k, scale_format=fmt)
    xf, af, bf, dyf = (t.float().numpy() for t in (x, a, b, dy))
    y, t = bd.linear_fwd(q, a.cuda(), b.cuda(), 16.0, x.cuda(), y_dtype=torch.float32)
    yr, tr = O.linear_fwd(wd, af, bf, xf, 16.0, r)
    _check(f"y {fmt}", y, yr)
    _check(f"T {fmt}", t[0].float() + t[1].float(), tr)
    dx, da, db = bd.linear_bwd(q, a.cuda(), b.cuda(), 16.0, x.cuda(), dy.cuda(), t, dx_dtype=torch.float32,
                               grad_dtype=torch.float32)
    dxr, dar, dbr = O.linear_bwd(wd, af, bf, xf, dyf, 16.0, r)
    _check(f"dX {fmt}", dx, dxr)
    _check(f"dA {fmt}", da, dar)
    _check(f"dB {fmt}", db, dbr)


@pytest.mark.parametrize("fmt", FORMATS)
def test_multi_adapter_decode(fmt):
    n, k, m, r = 1024, 4096, 4, 16
    w, x, _, _, _ = I.custom(n, k, m, r, 61)
    q, ref = _quant_both(w, fmt)
    wd = O.dequantize(ref["codes"], ref["scale_codes"], ref["c2"], n, k, scale_format=fmt)
    ads, adr = [], []
    for i in range(2):
        _, _, a, b, _ = I.custom(n, k, 1, r, 70 + i)
        ads.append((a.cuda(), b.cuda(), 16.0))
        adr.append((a.float().numpy(), b.float().numpy(), 16.0, r))
    which = [0, 1, 1, 0]
    y = bd.linear_fwd_multi(q, ads, which, x.cuda(), y_dtype=torch.float32)
    yr = O.linear_fwd_multi(wd, adr, which, x.float().numpy())
    _check(f"y multi {fmt}", y, yr)


@pytest.mark.parametrize("fmt", FORMATS)
def test_merged_export(fmt):
    n, k, r = 384, 512, 16
    w, _, a, b, _ = I.custom(n, k, 1, r, 83, b_std=0.05)
    q, ref = _quant_both(w, fmt)
    got = bd.merge(q, a.cuda(), b.cuda(), 16.0).float().cpu().numpy().astype(np.float64)
    want = O.merge_export(ref["codes"], ref["scale_codes"], ref["c2"], n, k, a.float().numpy(), b.float().numpy(),
                          16.0, r, scale_format=fmt).astype(np.float64)
    # one bf16 rounding of the exact sum, plus the float32 rank-r product's own error
    terms = O.lora_scale(16.0, r) * (np.abs(b.double().numpy()) @ np.abs(a.double().numpy()))
    aw = np.abs(want)
    ulp = np.where(aw > 0, 2.0 ** (np.floor(np.log2(np.where(aw > 0, aw, 1.0))) - 7), 2.0 ** -133)
    assert np.all(np.abs(got - want) <= ulp + r * 2.0 ** -24 * terms)
    assert np.mean(got == want) > 0.999
