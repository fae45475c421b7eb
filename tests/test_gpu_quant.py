"""GPU quantise / dequantise against the CPU oracle: bit-exact codes, E4M3 scale
codes, second-level constants and dequantised bf16 weights."""

import numpy as np
import pytest
import torch

import oracle as O
from bit_nf4_quantized_27_b200 import binding as bd
from bit_nf4_quantized_27_b200 import inputs as I

pytestmark = pytest.mark.gpu


def _gpu_quant(w_cpu: torch.Tensor):
    ws = bd.new_workspace(bd.STATUS_BYTES)
    q = bd.quantize(w_cpu.cuda().contiguous(), ws=ws)
    st = bd.read_status(ws)
    return q, st


def _compare_quant(w_cpu: torch.Tensor):
    rows, cols = w_cpu.shape
    q, st = _gpu_quant(w_cpu)
    assert st == 0
    ref = O.quantize(w_cpu.float().numpy(), rows, cols)
    codes = q.codes.cpu().numpy()
    if not np.array_equal(codes, ref["codes"]):
        bad = np.flatnonzero(codes != ref["codes"])
        raise AssertionError(f"{bad.size} code bytes differ, first at {bad[:5]}")
    assert np.array_equal(q.scale_codes.cpu().numpy(), ref["scale_codes"])
    assert np.array_equal(q.c2.cpu().numpy().view(np.uint32), ref["c2"].view(np.uint32))
    return q, ref


def _compare_dequant(q, ref, rows, cols):
    wd = O.dequantize(ref["codes"], ref["scale_codes"], ref["c2"], rows, cols)
    got16 = bd.dequantize(q, torch.bfloat16).cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got16.reshape(-1), O.bf16_bits(wd.reshape(-1)))
    got32 = bd.dequantize(q, torch.float32).cpu().numpy()
    assert np.array_equal(got32.view(np.uint32), wd.view(np.uint32))


def test_dequantize_into_a_16_byte_aligned_view():
    """W_out only 16-byte aligned (not 32): the 16-byte-store kernel writes it."""
    rows, cols = 96, 320
    w = I.custom(rows, cols, 1, 8, 515)[0]
    q, ref = _compare_quant(w)
    wd = O.dequantize(ref["codes"], ref["scale_codes"], ref["c2"], rows, cols)
    buf = torch.full((rows * cols + 8,), -1, dtype=torch.int16, device="cuda")
    view = buf[8:].view(torch.bfloat16).view(rows, cols)  # 16 bytes past a 256-byte aligned start
    assert view.data_ptr() % 32 == 16
    bd.dequantize(q, torch.bfloat16, out=view)
    got = buf.cpu().numpy().view(np.uint16)
    assert np.all(got[:8] == 0xFFFF)  # nothing before the view is touched
    assert np.array_equal(got[8:], O.bf16_bits(wd.reshape(-1)))


def test_tiny_workload_fp32():
    w = I.weight(I.TINY)
    assert w.dtype == torch.float32 and w.shape == (256, 256)
    q, ref = _compare_quant(w)
    _compare_dequant(q, ref, 256, 256)


@pytest.mark.parametrize("rows,cols,seed", [(8, 192, 1), (64, 64 * 300, 2), (3, 64, 3), (130, 640, 4),
                                            (1, 64 * 513, 5)])
def test_ragged_shapes_bf16(rows, cols, seed):
    w = I.normal((rows, cols), 0.02, 777 + seed)
    q, ref = _compare_quant(w)
    _compare_dequant(q, ref, rows, cols)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_special_blocks(dtype):
    rows, cols = 4, 64 * 600
    g = torch.Generator().manual_seed(99)
    w = (torch.randn(rows, cols, generator=g) * 0.02).to(dtype)
    w[0, :64 * 300] = 0                        # zero blocks and a whole zero group
    w[1, 64:128] = 1e-30                       # tiny constant block
    w[1, 128:192] = torch.randn(64, generator=g).to(dtype) * 1e-39  # subnormal scale
    w[2, :64] = torch.tensor([1.0] + [0.5] * 63).to(dtype)
    w[3, 64:128] *= 1e4                        # block far above its group
    q, ref = _compare_quant(w)
    _compare_dequant(q, ref, rows, cols)


def test_near_switch_points_many_scales():
    # Weights at and around every switch point of the code search, under many
    # non-power-of-two scales, so the fast reciprocal path must fall back to the
    # exact quotient.
    lv = O.nf4_levels().astype(np.float64)
    mids = (lv[1:] + lv[:-1]) / 2
    rng = np.random.default_rng(4)
    blocks = []
    for _ in range(512):
        S = np.float32(rng.uniform(1e-3, 3.0))
        blk = np.empty(64, np.float32)
        blk[0] = S
        x = rng.choice(mids, 63) * S
        xs = x.astype(np.float32)
        xs = np.nextafter(xs, np.float32(np.inf) * np.sign(rng.standard_normal(63)).astype(np.float32))
        blk[1:] = np.clip(xs, -S, S)
        blocks.append(blk)
    w = torch.from_numpy(np.stack(blocks).reshape(64, 512))
    _compare_quant(w)
    # the same values rounded to bf16 (a different set of quotients)
    _compare_quant(w.to(torch.bfloat16))


@pytest.mark.parametrize("wl", [I.QUANT_4096, I.QUANT_11008], ids=lambda w: w.name)
def test_full_size_bit_exact(wl):
    w = I.weight(wl)
    q, ref = _compare_quant(w)
    _compare_dequant(q, ref, *w.shape)


def test_nonfinite_sets_status():
    w = torch.randn(4, 256).to(torch.bfloat16) * 0.02
    w[2, 70] = float("inf")
    _, st = _gpu_quant(w)
    assert st == 5
    w[2, 70] = float("nan")
    _, st = _gpu_quant(w)
    assert st == 5


def test_requantise_idempotent_on_gpu():
    w = I.normal((256, 1024), 0.02, 31)
    q, _ = _gpu_quant(w)
    wd = bd.dequantize(q, torch.bfloat16)
    ws = bd.new_workspace(bd.STATUS_BYTES)
    q2 = bd.quantize(wd, ws=ws)
    assert torch.equal(q.codes, q2.codes)


def test_every_float32_in_the_unit_interval():
    # Every float32 x in [-1, 1] (both zeros included, 2 130 706 434 values) goes
    # through the kernel with S = 1, so x = w / S exactly: 63 values per block of
    # 64 next to a 1.0 that fixes the block's absmax.  The expected code is the
    # number of the oracle's switch points below x (the switch points come from
    # bisecting the oracle's own code assignment).
    from tests.test_host_layout import _oracle_switch_points

    thr = torch.tensor(_oracle_switch_points(), dtype=torch.int64).to(torch.int32).view(torch.float32).cuda()
    ws = bd.new_workspace(bd.STATUS_BYTES)
    per = 63
    nblk = 1 << 22                                  # blocks per chunk: 264 M values, 1 GiB of input
    top = 0x3F800000                                # bits of 1.0
    checked = 0
    for sign in (0, 0x80000000):
        for start in range(0, top + 1, per * nblk):
            n = min(per * nblk, top + 1 - start)
            nb = (n + per - 1) // per
            bits = torch.arange(start, start + nb * per, dtype=torch.int64, device="cuda")
            bits = torch.minimum(bits, torch.tensor(top, device="cuda")) | sign
            x = bits.to(torch.int64).view(-1)
            x = torch.where(x >= 1 << 31, x - (1 << 32), x).to(torch.int32).view(torch.float32).view(nb, per)
            w = torch.cat([torch.ones(nb, 1, device="cuda"), x], dim=1).contiguous()
            q = bd.quantize(w, ws=ws)
            p = q.codes.view(nb, 32)
            codes = torch.stack([p & 15, p >> 4], dim=2).view(nb, 64)[:, 1:]
            want = torch.searchsorted(thr, x.contiguous(), side="left", out_int32=True)
            bad = (codes.to(torch.int32) != want).sum().item()
            assert bad == 0, (hex(sign), start, bad)
            checked += n
            del bits, x, w, q, p, codes, want
    assert bd.read_status(ws) == 0
    assert checked == 2 * (top + 1)
