"""GPU forward/backward of the NF4 linear layer with LoRA against the CPU oracle.

Tolerance (the stated bar for outputs and gradients): max |gpu - oracle| <=
1e-2 * RMS(oracle).  Float32 outputs are held to exactly that; bf16 outputs may in
addition carry their own rounding, one bf16 ulp of the oracle value.  The oracle
quantises the raw weights itself; nothing it uses comes from the GPU."""

import math

import numpy as np
import pytest
import torch

import oracle as O
from bit_nf4_quantized_27_b200 import binding as bd
from bit_nf4_quantized_27_b200 import inputs as I

pytestmark = pytest.mark.gpu

TOL = 1e-2


def _ulp_bf16(v):
    a = np.abs(v)
    e = np.floor(np.log2(np.where(a > 0, a, 1e-38)))
    return np.where(a > 0, 2.0 ** (e - 7), 2.0 ** -133)


def check(name, got: torch.Tensor, ref: np.ndarray, rms: float | None = None):
    g = got.float().cpu().numpy().astype(np.float64)
    ref = np.asarray(ref, np.float64)
    assert g.shape == ref.shape, (name, g.shape, ref.shape)
    rms = float(np.sqrt(np.mean(ref ** 2))) if rms is None else rms
    err = np.abs(g - ref)
    bound = TOL * rms + (_ulp_bf16(ref) if got.dtype == torch.bfloat16 else 0.0)
    worst = float(np.max(err - bound))
    assert np.all(np.isfinite(g)), name
    assert worst <= 0, f"{name}: max err {err.max():.3e} vs bound {TOL * rms:.3e} (rms {rms:.3e})"
    return float(err.max() / rms) if rms > 0 else 0.0


class Case:
    """Inputs + oracle for one layer."""

    def __init__(self, w, x, a, b, dy, alpha):
        self.w, self.x, self.a, self.b, self.dy, self.alpha = w, x, a, b, dy, alpha
        self.n, self.k = w.shape
        self.m, self.r = x.shape[0], a.shape[0]
        q = O.quantize(w.float().numpy(), self.n, self.k)
        self.wd = O.dequantize(q["codes"], q["scale_codes"], q["c2"], self.n, self.k)
        self.xf, self.af, self.bf, self.dyf = (t.float().numpy() for t in (x, a, b, dy))

    def gpu(self):
        qg = bd.quantize(self.w.cuda())
        return qg, self.a.cuda(), self.b.cuda(), self.x.cuda(), self.dy.cuda()

    def ref_fwd(self, rows=None):
        x = self.xf if rows is None else self.xf[rows]
        return O.linear_fwd(self.wd, self.af, self.bf, x, self.alpha, self.r)

    def ref_bwd(self):
        return O.linear_bwd(self.wd, self.af, self.bf, self.xf, self.dyf, self.alpha, self.r)


def _custom(n, k, m, r, seed, alpha=16.0, w_dtype=torch.bfloat16, b_std=0.01):
    return Case(*I.custom(n, k, m, r, seed, w_dtype=w_dtype, b_std=b_std), alpha)


def _run_fwd_bwd(c: Case, y_dtype, g_dtype, save_t=True):
    qg, a, b, x, dy = c.gpu()
    y, t = bd.linear_fwd(qg, a, b, c.alpha, x, y_dtype=y_dtype, save_t=save_t)
    dx, da, db = bd.linear_bwd(qg, a, b, c.alpha, x, dy, t, dx_dtype=g_dtype, grad_dtype=g_dtype)
    torch.cuda.synchronize()
    return y, t, dx, da, db


def _check_all(c: Case, y, t, dx, da, db):
    yr, tr = c.ref_fwd()
    check("y", y, yr)
    if t is not None:
        check("T", t[0].float() + t[1].float(), tr)
    dxr, dar, dbr = c.ref_bwd()
    check("dX", dx, dxr)
    check("dA", da, dar)
    check("dB", db, dbr)


def test_tiny_workload():
    wl = I.TINY
    c = Case(I.weight(wl), I.activations(wl), I.lora_a(wl), I.lora_b(wl), I.grad_output(wl), wl.alpha)
    for dt in (torch.float32, torch.bfloat16):
        _check_all(c, *_run_fwd_bwd(c, dt, dt))


@pytest.mark.parametrize("m", [1, 3, 4, 9, 16])
def test_gemv_path_small_shapes(m):
    c = _custom(328, 576, m, 64, 1000 + m)
    for dt in (torch.float32, torch.bfloat16):
        qg, a, b, x, _ = c.gpu()
        y, t = bd.linear_fwd(qg, a, b, c.alpha, x, y_dtype=dt)
        yr, tr = c.ref_fwd()
        check(f"y m={m}", y, yr)
        check(f"T m={m}", t[0].float() + t[1].float(), tr)


@pytest.mark.parametrize("n,k,m,r", [(1024, 256, 1, 8), (2048, 1024, 3, 16), (4096, 8192, 5, 64),
                                     (1040, 4096, 8, 128), (2064, 12288, 12, 64), (3072, 4096, 16, 64),
                                     (4816, 1024, 2, 64), (1536, 4096, 9, 48)])
def test_gemv_staged_shapes(n, k, m, r):
    # staged decode kernel: fewer active warps (K < 4096), 4096-column chunks
    # (K > 4096), ranks beyond 64, both partial-sum widths (M <= 8 and M > 8), and
    # a last CTA with fewer row groups than the others
    c = _custom(n, k, m, r, 31 * n + k + m)
    qg, a, b, x, _ = c.gpu()
    y, t = bd.linear_fwd(qg, a, b, c.alpha, x, y_dtype=torch.float32)
    yr, tr = c.ref_fwd()
    check(f"y {n}x{k} m={m} r={r}", y, yr)
    check(f"T {n}x{k} m={m} r={r}", t[0].float() + t[1].float(), tr)


@pytest.mark.parametrize("m", [1, 4, 16])
def test_gemv_workload_11008x4096(m):
    wl = I.GEMV
    c = Case(I.weight(wl), I.activations(wl, m=m), I.lora_a(wl), I.lora_b(wl), I.grad_output(wl, m=m), wl.alpha)
    qg, a, b, x, _ = c.gpu()
    y, _ = bd.linear_fwd(qg, a, b, c.alpha, x, y_dtype=torch.float32)
    yr, _ = c.ref_fwd()
    check("y", y, yr)
    # LoRA contribution alone must be right too (it is ~1.5% of y's RMS)
    y0, _ = bd.linear_fwd(qg, a, torch.zeros_like(b), c.alpha, x, y_dtype=torch.float32)
    lora_ref = yr - (c.xf.astype(np.float64) @ c.wd.astype(np.float64).T)
    check("lora part", y - y0, lora_ref)


@pytest.mark.parametrize("n,k,m,r", [(256, 256, 17, 8), (328, 320, 200, 16), (1024, 1024, 512, 64),
                                     (264, 640, 129, 128), (512, 192, 300, 256), (4104, 128, 64, 64)])
def test_tensor_core_path_ragged(n, k, m, r):
    c = _custom(n, k, m, r, 7 * n + k + m + r)
    for dt in (torch.float32, torch.bfloat16):
        _check_all(c, *_run_fwd_bwd(c, dt, dt))


def test_backward_recomputes_t():
    c = _custom(512, 512, 96, 64, 55)
    qg, a, b, x, dy = c.gpu()
    dx, da, db = bd.linear_bwd(qg, a, b, c.alpha, x, dy, None, dx_dtype=torch.float32, grad_dtype=torch.float32)
    dxr, dar, dbr = c.ref_bwd()
    check("dX", dx, dxr)
    check("dA", da, dar)
    check("dB", db, dbr)


@pytest.mark.parametrize("n,k,m,r", [(1000, 320, 600, 16), (264, 640, 513, 128), (4104, 128, 1030, 8),
                                     (512, 1024, 257, 64)])
def test_cta_pair_path_ragged(n, k, m, r):
    # from 257 tokens the fused forward / dX GEMMs run on CTA pairs (512-token
    # tiles, 256 columns split between the two CTAs): ragged N, K and M
    c = _custom(n, k, m, r, 11 * n + k + m + r)
    for dt in (torch.float32, torch.bfloat16):
        _check_all(c, *_run_fwd_bwd(c, dt, dt))


@pytest.mark.parametrize("n,k,m", [(20480, 256, 512), (256, 20480, 512), (10240, 320, 600)])
def test_cta_pair_last_round_split(n, k, m):
    # more 512-token tiles than resident CTA pairs, with a short last round: its
    # tiles run as 256-token halves (forward: N = 20480 or 10240; dX: K = 20480)
    c = _custom(n, k, m, 16, 3 * n + k + m)
    _check_all(c, *_run_fwd_bwd(c, torch.float32, torch.float32))


@pytest.mark.parametrize("n,k,m,r", [(1024, 1024, 512, 64), (512, 2048, 300, 16), (640, 4096, 2048, 128)])
def test_minimum_workspace_without_k_split(n, k, m, r):
    # the least workspace the entry points accept runs the rank-r GEMMs (X A^T,
    # dY B) without splitting K; the reported size splits K over more CTAs
    c = _custom(n, k, m, r, 5 * n + m)
    qg, a, b, x, dy = c.gpu()
    mr = (m * r * 2 + 255) // 256 * 256
    assert bd.workspace_bytes(m, n, k, r, False) > 256 + mr
    for fw, bw in ((256 + mr, 256 + 4 * mr), (None, None)):
        wsf = bd.new_workspace(fw) if fw else None
        wsb = bd.new_workspace(bw) if bw else None
        y, t = bd.linear_fwd(qg, a, b, c.alpha, x, y_dtype=torch.float32, ws=wsf)
        dx, da, db = bd.linear_bwd(qg, a, b, c.alpha, x, dy, t, dx_dtype=torch.float32, grad_dtype=torch.float32,
                                   ws=wsb)
        torch.cuda.synchronize()
        _check_all(c, y, t, dx, da, db)


@pytest.mark.parametrize("m", [4, 300])
def test_b_zero_is_base_layer(m):
    c = _custom(512, 512, m, 64, 77, b_std=0.0)
    y, t, dx, da, db = _run_fwd_bwd(c, torch.float32, torch.float32)
    base = c.xf.astype(np.float64) @ c.wd.astype(np.float64).T
    check("y", y, base)
    assert torch.count_nonzero(da) == 0


@pytest.mark.parametrize("m", [4, 300])
def test_w_zero_isolates_lora(m):
    w, x, a, b, dy = I.custom(512, 512, m, 64, 88)
    c = Case(torch.zeros_like(w), x, a, b, dy, 16.0)
    y, t, dx, da, db = _run_fwd_bwd(c, torch.float32, torch.float32)
    yr, _ = c.ref_fwd()
    check("y", y, yr)
    dxr, dar, dbr = c.ref_bwd()
    check("dX", dx, dxr)


def test_merged_form():
    c = _custom(512, 512, 64, 64, 99)
    qg, a, b, x, _ = c.gpu()
    y, _ = bd.linear_fwd(qg, a, b, c.alpha, x, y_dtype=torch.float32)
    wm = O.merged_weight(c.wd, c.af, c.bf, c.alpha, c.r)
    check("y", y, c.xf.astype(np.float64) @ wm.T)


def test_autograd_wrapper():
    c = _custom(256, 256, 32, 16, 5)
    qg, a, b, x, dy = c.gpu()
    x = x.clone().requires_grad_(True)
    a = a.clone().requires_grad_(True)
    b = b.clone().requires_grad_(True)
    y = bd.QLoRALinearFunction.apply(x, a, b, qg, c.alpha)
    y.backward(dy)
    dxr, dar, dbr = c.ref_bwd()
    check("dX", x.grad, dxr)
    check("dA", a.grad, dar)
    check("dB", b.grad, dbr)


@pytest.mark.parametrize("m", [256, 300])
def test_deterministic(m):
    c = _custom(1024, 1024, m, 64, 3)
    r1 = _run_fwd_bwd(c, torch.float32, torch.float32)
    r2 = _run_fwd_bwd(c, torch.float32, torch.float32)
    for u, v in zip(r1, r2):
        assert torch.equal(u, v)


def _lora_parts(c: Case, rows=None):
    """The LoRA terms of y and dX alone: from the GPU as the call with B minus the
    call with B = 0 (float32 outputs; the base product is the same in both), and
    from the oracle, on all rows or on `rows`.  Returns, per term, (got, want,
    bound): the fused kernels take the LoRA product as extra K steps with the
    bf16 rounding of s T (or s U) as one operand, so each element is within
    2^-8 (|s T| |B^T|) of the exact term, plus one float32 rounding of the
    running sum per step."""
    qg, a, b, x, dy = c.gpu()
    y, t = bd.linear_fwd(qg, a, b, c.alpha, x, y_dtype=torch.float32)
    y0, _ = bd.linear_fwd(qg, a, torch.zeros_like(b), c.alpha, x, y_dtype=torch.float32)
    dx, _, _ = bd.linear_bwd(qg, a, b, c.alpha, x, dy, t, dx_dtype=torch.float32, grad_dtype=torch.float32)
    dx0, _, _ = bd.linear_bwd(qg, a, torch.zeros_like(b), c.alpha, x, dy, t, dx_dtype=torch.float32,
                              grad_dtype=torch.float32)
    torch.cuda.synchronize()
    s = O.lora_scale(c.alpha, c.r)
    x64, dy64, a64, b64 = (np.asarray(v, np.float64) for v in (c.xf, c.dyf, c.af, c.bf))
    wd = c.wd.astype(np.float64)
    sel = slice(None) if rows is None else rows
    idx = slice(None) if rows is None else torch.from_numpy(rows)
    st = s * (x64[sel] @ a64.T)
    su = s * (dy64[sel] @ b64)
    y0v, dx0v = y0[idx].double().cpu().numpy(), dx0[idx].double().cpu().numpy()
    y_term = y[idx].double().cpu().numpy() - y0v
    dx_term = dx[idx].double().cpu().numpy() - dx0v
    # the LoRA K steps come after the base steps in the same float32 accumulator:
    # each 16-deep step rounds once, relative to the running sum
    steps = c.r // 16 + 1
    y_bound = 2.0 ** -8 * (np.abs(st) @ np.abs(b64.T)) + steps * 2.0 ** -24 * (np.abs(y0v) + np.abs(y_term))
    dx_bound = 2.0 ** -8 * (np.abs(su) @ np.abs(a64)) + steps * 2.0 ** -24 * (np.abs(dx0v) + np.abs(dx_term))
    return (y_term, st @ b64.T, y_bound), (dx_term, su @ a64, dx_bound)


def _check_term(name, got, want, bound):
    rms = float(np.sqrt(np.mean(want ** 2)))
    assert np.all(np.isfinite(got)), name
    worst = float(np.max(np.abs(got - want) - bound))
    assert worst <= 1e-6 * rms, f"{name}: exceeds its bound by {worst:.3e} (term rms {rms:.3e})"
    # and the bound itself is a small fraction of the term (2^-8 of |s U| |A|,
    # a few percent of |s U A| for r = 64 terms of mixed signs)
    assert float(np.sqrt(np.mean(bound ** 2))) <= 0.05 * rms, name


@pytest.mark.parametrize("m", [17, 128, 256])
def test_lora_term_alone_single_cta(m):
    # 17..256 tokens run the single-CTA fused kernel; its LoRA K steps are held to
    # their own error bound (the term is about 1.5% of y's RMS)
    c = _custom(1024, 1024, m, 64, 4000 + m)
    yt, dxt = _lora_parts(c)
    _check_term(f"y lora m={m}", *yt)
    _check_term(f"dX lora m={m}", *dxt)


def test_lora_term_alone_65b_layer():
    # the CTA-pair kernel at a full block shape: 8192x8192, 4096 tokens, r = 64
    wl = I.L65B_BLOCK
    c = Case(I.weight(wl, 0), I.activations(wl, 0), I.lora_a(wl, 0), I.lora_b(wl, 0), I.grad_output(wl, 0),
             wl.alpha)
    rng = np.random.default_rng(65)
    rows = np.sort(rng.choice(c.m, 32, replace=False))
    yt, dxt = _lora_parts(c, rows)
    _check_term("y lora rows", *yt)
    _check_term("dX lora rows", *dxt)


def _sampled(wl, layer, nrows=48):
    c = Case(I.weight(wl, layer), I.activations(wl, layer), I.lora_a(wl, layer), I.lora_b(wl, layer),
             I.grad_output(wl, layer), wl.alpha)
    qg, a, b, x, dy = c.gpu()
    y, t = bd.linear_fwd(qg, a, b, c.alpha, x, y_dtype=torch.bfloat16)
    dx, da, db = bd.linear_bwd(qg, a, b, c.alpha, x, dy, t, dx_dtype=torch.bfloat16, grad_dtype=torch.float32)
    torch.cuda.synchronize()
    rng = np.random.default_rng(layer)
    rows = np.sort(rng.choice(c.m, nrows, replace=False))
    rows[-1] = c.m - 1
    yr, tr = c.ref_fwd(rows)
    check("y rows", y[torch.from_numpy(rows)], yr)
    s = O.lora_scale(c.alpha, c.r)
    x64, dy64, a64, b64 = (np.asarray(v, np.float64) for v in (c.xf, c.dyf, c.af, c.bf))
    u = dy64 @ b64
    dxr = dy64[rows] @ c.wd.astype(np.float64) + s * (u[rows] @ a64)
    check("dX rows", dx[torch.from_numpy(rows)], dxr)
    t64 = x64 @ a64.T
    check("dA", da, s * (u.T @ x64))
    check("dB", db, s * (dy64.T @ t64))


@pytest.mark.parametrize("layer", [0, 4, 6], ids=["q", "gate", "down"])
def test_llama7b_block_layers_full_size(layer):
    _sampled(I.LLAMA7B_BLOCK, layer)


@pytest.mark.parametrize("layer", [0, 4, 6], ids=["q", "gate", "down"])
def test_65b_block_layers_full_size(layer):
    _sampled(I.L65B_BLOCK, layer, nrows=24)


@pytest.mark.parametrize("n,k,m,r,p", [(328, 576, 4, 64, 0.1), (1024, 1024, 300, 16, 0.25), (512, 512, 200, 64, 0.5),
                                       (4104, 128, 1030, 8, 0.05), (640, 4096, 2048, 128, 0.1)])
def test_lora_dropout_matches_oracle(n, k, m, r, p):
    c = _custom(n, k, m, r, 13 * n + k + m)
    keep = I.keep_mask(m, k, p, 99 + m)
    kb = O.unpack_keep(keep.numpy(), m, k)
    qg, a, b, x, dy = c.gpu()
    for dt in (torch.float32, torch.bfloat16):
        y, t = bd.linear_fwd_dropout(qg, a, b, c.alpha, x, keep.cuda(), p, y_dtype=dt)
        dx, da, db = bd.linear_bwd_dropout(qg, a, b, c.alpha, x, dy, keep.cuda(), p, t, dx_dtype=dt, grad_dtype=dt)
        torch.cuda.synchronize()
        yr, tr = O.linear_fwd_dropout(c.wd, c.af, c.bf, c.xf, kb, p, c.alpha, c.r)
        check("y", y, yr)
        check("T", t[0].float() + t[1].float(), tr)
        dxr, dar, dbr = O.linear_bwd_dropout(c.wd, c.af, c.bf, c.xf, c.dyf, kb, p, c.alpha, c.r)
        check("dX", dx, dxr)
        if dt == torch.float32:
            # the adapter's share of dX alone (about 1% of it), the masked term: it
            # multiplies A by the bf16 rounding of s U, so each element is within
            # 2^-8 of (|s U| |A|) * keep / (1 - p) of the exact term, plus the float32
            # accumulation error of the base product dY W' it is separated from
            base = c.dyf.astype(np.float64) @ c.wd.astype(np.float64)
            su = O.lora_scale(c.alpha, c.r) * (c.dyf.astype(np.float64) @ c.bf.astype(np.float64))
            bound = 2.0 ** -8 * (np.abs(su) @ np.abs(c.af.astype(np.float64))) * kb / (1 - p) + \
                n * 2.0 ** -24 * (np.abs(c.dyf.astype(np.float64)) @ np.abs(c.wd.astype(np.float64)))
            term = dx.double().cpu().numpy() - base
            term_ref = dxr - base
            assert np.all(np.abs(term - term_ref) <= bound + 1e-6 * np.sqrt(np.mean(term_ref ** 2)))
        check("dA", da, dar)
        check("dB", db, dbr)
    # backward recomputing T from the masked input
    dx2, da2, db2 = bd.linear_bwd_dropout(qg, a, b, c.alpha, x, dy, keep.cuda(), p, None, dx_dtype=torch.float32,
                                          grad_dtype=torch.float32)
    torch.cuda.synchronize()
    check("dB (T recomputed)", db2, dbr)
    check("dA (T recomputed)", da2, dar)


@pytest.mark.parametrize("n,k,m,r", [(1000, 256, 1, 8), (1000, 768, 7, 24), (2040, 1280, 16, 64),
                                     (3080, 3840, 11, 40), (11008, 4096, 2, 16), (256, 4096, 16, 256)])
def test_one_kernel_decode_shapes(n, k, m, r):
    # the one-kernel decode path: rows not a multiple of 16, K giving 1, 3, 5, 15
    # and 16 warps per row group, ranks below a k-step (r % 16 != 0) and two
    # 64-rank chunks
    c = _custom(n, k, m, r, 13 * n + k + m + r)
    qg, a, b, x, _ = c.gpu()
    ws = bd.new_workspace(bd.workspace_bytes(m, n, k, r, False))
    for dt in (torch.float32, torch.bfloat16):
        y, t = bd.linear_fwd(qg, a, b, c.alpha, x, y_dtype=dt, ws=ws)
        yr, tr = c.ref_fwd()
        check(f"y {n}x{k} m={m} r={r}", y, yr)
        check(f"T {n}x{k} m={m} r={r}", t[0].float() + t[1].float(), tr)
    assert bd.read_status(ws) == 0


def test_decode_lora_term_alone():
    # W = 0 (every code 7): y = s (X A^T) B^T, the LoRA path alone, on the decode
    # kernel at 1, 9 and 16 tokens
    for m in (1, 9, 16):
        c = _custom(2048, 1024, m, 64, 71 + m, b_std=0.5)
        c.w = torch.zeros_like(c.w)
        c.wd = np.zeros_like(c.wd)
        qg, a, b, x, _ = c.gpu()
        y, _ = bd.linear_fwd(qg, a, b, c.alpha, x, y_dtype=torch.float32)
        yr, _ = c.ref_fwd()
        check(f"lora alone m={m}", y, yr)


def test_decode_consecutive_calls_share_a_workspace():
    # Calls on one workspace, alternating two weights (different grids), with new
    # tokens each time: the grid barrier's generation moves on every call and its
    # count returns to zero; the results stay bit-identical for repeated inputs.
    c1 = _custom(4096, 2048, 4, 64, 501)
    c2 = _custom(1536, 4096, 16, 32, 502)
    g1, g2 = c1.gpu(), c2.gpu()
    ws = bd.new_workspace(max(bd.workspace_bytes(16, 4096, 4096, 64, False), 4096))
    first = {}
    for it in range(6):
        for name, c, gp in (("a", c1, g1), ("b", c2, g2)):
            qg, a, b, x, _ = gp
            xi = x if it % 2 == 0 else x.flip(0).contiguous()
            y, _ = bd.linear_fwd(qg, a, b, c.alpha, xi, y_dtype=torch.float32, ws=ws)
            key = (name, it % 2)
            if key in first:
                assert torch.equal(y, first[key]), key
            else:
                first[key] = y.clone()
                xr = c.xf if it % 2 == 0 else c.xf[::-1]
                yr, _ = O.linear_fwd(c.wd, c.af, c.bf, xr, c.alpha, c.r)
                check(f"y {name} {it}", y, yr)
    assert bd.read_status(ws) == 0
    hdr = ws[:16].view(torch.int32).cpu()
    assert int(hdr[1]) == 0  # barrier count back to zero


def test_decode_graph_replay():
    # 24 calls captured in one CUDA graph (consecutive kernels overlap through
    # programmatic dependent launch), replayed twice, against eager results
    c = _custom(11008, 4096, 1, 64, 777)
    qg, a, b, x, _ = c.gpu()
    ws = bd.new_workspace(bd.workspace_bytes(16, 11008, 4096, 64, False))
    xs = [torch.randn(1, 4096, device="cuda").to(torch.bfloat16) for _ in range(3)]
    ys = [torch.empty(1, 11008, dtype=torch.float32, device="cuda") for _ in range(24)]
    want = [bd.linear_fwd(qg, a, b, c.alpha, xs[i % 3], y_dtype=torch.float32, ws=ws)[0].clone() for i in range(3)]
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            for i in range(24):
                bd.linear_fwd(qg, a, b, c.alpha, xs[i % 3], ws=ws, out=ys[i], save_t=False)
    for _ in range(2):
        for y in ys:
            y.zero_()
        g.replay()
        torch.cuda.synchronize()
        for i, y in enumerate(ys):
            assert torch.equal(y, want[i % 3]), (i, float((y - want[i % 3]).abs().max()))
    del g
    assert bd.read_status(ws) == 0
