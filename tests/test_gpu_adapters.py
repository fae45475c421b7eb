"""GPU merged export and AdamW step of the adapters against the CPU oracle.

Merged export: the oracle rounds the exact W' + s B A to bf16 once; the kernel
accumulates s B A over the r terms in float32 first.  Float32 accumulation of r
products is off by at most about r * 2^-24 times the sum of their magnitudes, so
each element is held to one bf16 ulp of the oracle value plus that bound (which
matters only where the terms cancel), and almost all must be bit-identical.
AdamW: float32 arithmetic against float64 over six steps.  The momentum is a
sum of terms of either sign, so it is held to 2e-6 of the running sum of their
magnitudes; the variance (all terms positive) and the parameters to 2e-6
relative; the bf16 copy must be exactly bf16 of the float32 parameters."""

import numpy as np
import pytest
import torch

import oracle as O
from bit_nf4_quantized_27_b200 import binding as bd
from bit_nf4_quantized_27_b200 import inputs as I

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n,k,r", [(256, 256, 8), (1000, 320, 16), (328, 576, 128), (520, 1088, 72),
                                   (4096, 4096, 64), (1, 512, 8), (136, 64, 256), (300, 1344, 200)])
def test_merge_matches_oracle(n, k, r):
    w, _, a, b, _ = I.custom(n, k, 1, r, 40 * n + k + r)
    q = O.quantize(w.float().numpy(), n, k)
    ref = O.merge_export(q["codes"], q["scale_codes"], q["c2"], n, k, a.float().numpy(), b.float().numpy(), 16.0, r)
    terms = O.lora_scale(16.0, r) * (np.abs(b.double().numpy()) @ np.abs(a.double().numpy()))
    qg = bd.quantize(w.cuda())
    got = bd.merge(qg, a.cuda(), b.cuda(), 16.0)
    torch.cuda.synchronize()
    gv = got.float().cpu().numpy().astype(np.float64)
    rv = ref.astype(np.float64)
    a_ = np.abs(rv)
    ulp = np.where(a_ > 0, 2.0 ** (np.floor(np.log2(np.where(a_ > 0, a_, 1.0))) - 7), 2.0 ** -133)
    err = np.abs(gv - rv)
    bound = ulp + r * 2.0 ** -24 * terms
    assert np.all(err <= bound), f"{n}x{k} r={r}: max {np.max(err / bound):.2f} of the bound"
    assert np.mean(gv == rv) > 0.999
    assert bd.read_library_status() == 0


def test_merge_with_b_zero_is_the_dequantised_weight():
    n, k, r = 640, 512, 32
    w, _, a, _, _ = I.custom(n, k, 1, r, 77)
    qg = bd.quantize(w.cuda())
    got = bd.merge(qg, a.cuda(), torch.zeros(n, r, dtype=torch.bfloat16, device="cuda"), 16.0)
    deq = bd.dequantize(qg)
    torch.cuda.synchronize()
    assert torch.equal(got.view(torch.int16), deq.view(torch.int16))


@pytest.mark.parametrize("minimum_ws", [False, True])
def test_multi_adapter_bf16_output_is_the_rounded_float32_output(minimum_ws):
    """bf16 Y must be bf16(the float32 Y of the same call): one rounding of the sum."""
    n, k, m, r = 2048, 1024, 6, 32
    w, x, _, _, _ = I.custom(n, k, m, r, 4242)
    ads = [(a.cuda(), b.cuda(), al) for a, b, al in _adapters(n, k, r, 3, 4343)]
    idx = [t % 3 for t in range(m)]
    qg = bd.quantize(w.cuda())
    size = bd.workspace_bytes(m, n, k, r, False) if minimum_ws else bd.workspace_bytes_multi(m, n, k, r)
    ws = bd.new_workspace(size, torch.device("cuda"))
    y32 = bd.linear_fwd_multi(qg, ads, idx, x.cuda(), y_dtype=torch.float32, ws=ws)
    y16 = bd.linear_fwd_multi(qg, ads, idx, x.cuda(), y_dtype=torch.bfloat16, ws=ws)
    torch.cuda.synchronize()
    assert bd.read_status(ws) == 0
    assert torch.equal(y16.view(torch.int16), y32.to(torch.bfloat16).view(torch.int16))


@pytest.mark.parametrize("n", [1, 7, 1000003])
def test_adamw_matches_oracle_over_six_steps(n):
    g = torch.Generator().manual_seed(n)
    p0 = torch.randn(n, generator=g, dtype=torch.float64).float()
    grads = [torch.randn(n, generator=g, dtype=torch.float64).float() * (0.05 * (i + 1)) for i in range(6)]
    hp = dict(lr=2e-3, beta1=0.9, beta2=0.995, eps=1e-8, weight_decay=0.01)
    p, m, v = p0.cuda(), torch.zeros(n, device="cuda"), torch.zeros(n, device="cuda")
    p16 = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    rp, rm, rv = p0.double().numpy(), np.zeros(n), np.zeros(n)
    mag_m = np.zeros(n)  # running sum of the momentum's term magnitudes
    for t, gr in enumerate(grads, start=1):
        bd.adamw_step(p, gr.cuda(), m, v, t, p_bf16=p16, **hp)
        rp, rm, rv = O.adamw_step(rp, gr.double().numpy(), rm, rv, t, **hp)
        mag_m = hp["beta1"] * mag_m + (1 - hp["beta1"]) * np.abs(gr.double().numpy())
    torch.cuda.synchronize()
    gp, gm, gv = (x.cpu().double().numpy() for x in (p, m, v))
    assert np.all(np.abs(gp - rp) <= 2e-6 * (np.abs(rp) + hp["lr"]))
    assert np.all(np.abs(gm - rm) <= 2e-6 * mag_m)
    assert np.all(np.abs(gv - rv) <= 2e-6 * (np.abs(rv) + 1e-12))
    assert torch.equal(p16, p.to(torch.bfloat16))


def _adapters(n, k, r, count, seed):
    out = []
    for i in range(count):
        _, _, a, b, _ = I.custom(n, k, 1, r, seed + 7 * i)
        out.append((a, b * (1 + i), 16.0 / (1 + i)))  # distinct B scale and alpha per adapter
    return out


def _check(name, got, ref):
    g = got.float().cpu().numpy().astype(np.float64)
    rms = float(np.sqrt(np.mean(ref ** 2)))
    err = float(np.max(np.abs(g - ref)))
    assert np.all(np.isfinite(g)) and err <= 1e-2 * rms, f"{name}: {err:.3e} vs {1e-2 * rms:.3e}"


@pytest.mark.parametrize("n,k,m,r,count", [(11008, 4096, 1, 64, 2), (11008, 4096, 5, 64, 3), (11008, 4096, 16, 64, 16),
                                           (1024, 1024, 9, 16, 4), (2048, 8192, 4, 128, 2), (512, 256, 3, 8, 3),
                                           (1024, 1024, 6, 24, 3), (512, 512, 16, 72, 5), (768, 2048, 7, 256, 2)])
def test_multi_adapter_gemv_matches_oracle(n, k, m, r, count):
    w, x, _, _, _ = I.custom(n, k, m, r, 9000 + n + m)
    ads = _adapters(n, k, r, count, 9100 + k)
    idx = [(3 * t + 1) % count for t in range(m)]
    q = O.quantize(w.float().numpy(), n, k)
    wd = O.dequantize(q["codes"], q["scale_codes"], q["c2"], n, k)
    ref = O.linear_fwd_multi(wd, [(a.float().numpy(), b.float().numpy(), al, r) for a, b, al in ads], idx,
                             x.float().numpy())
    qg = bd.quantize(w.cuda())
    y = bd.linear_fwd_multi(qg, [(a.cuda(), b.cuda(), al) for a, b, al in ads], idx, x.cuda(), y_dtype=torch.float32)
    torch.cuda.synchronize()
    _check(f"y {n}x{k} m={m}", y, ref)
    # the minimum workspace: the adapters' term inside the GEMV instead of its own pass
    ws = bd.new_workspace(bd.workspace_bytes(m, n, k, r, False), torch.device("cuda"))
    y_min = bd.linear_fwd_multi(qg, [(a.cuda(), b.cuda(), al) for a, b, al in ads], idx, x.cuda(),
                                y_dtype=torch.float32, ws=ws)
    torch.cuda.synchronize()
    _check(f"y {n}x{k} m={m}, minimum workspace", y_min, ref)
    assert bd.read_status(ws) == 0
    # the adapters' own contribution, alone
    y0 = bd.linear_fwd_multi(qg, [(a.cuda(), torch.zeros_like(b).cuda(), al) for a, b, al in ads], idx, x.cuda(),
                             y_dtype=torch.float32)
    torch.cuda.synchronize()
    _check("lora part", y - y0, ref - x.float().numpy().astype(np.float64) @ wd.astype(np.float64).T)
