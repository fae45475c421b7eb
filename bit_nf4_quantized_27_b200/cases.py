"""Single named cases of the hot path, for profiling one kernel at a time.

Usage: python -m bit_nf4_quantized_27_b200.cases CASE [--reps R]

CASE is one of:
  fwd_8192      forward of one 8192x8192 layer, 4096 tokens, r=64 (65B-shaped q)
  bwd_8192      backward of the same layer
  fwd_11008     forward of 11008x4096 (gate/up of the Llama-7B block), 2048 tokens
  fwd_65b_up / bwd_65b_up       22016x8192 (gate/up of the 65B-shaped block), 4096 tokens
  fwd_65b_down / bwd_65b_down   8192x22016 (down of the 65B-shaped block), 4096 tokens
  gemv_m1 / gemv_m4 / gemv_m16   decode forward, W 11008x4096, r=64
  gemv_multi16  decode forward of 16 tokens, each with its own r=64 adapter
  quant_11008   quantise an 11008x4096 bf16 weight
  dequant_11008 dequantise it
  quant_4096 / dequant_4096     the same for a 4096x4096 weight
  merge_8192    merged export of an 8192x8192 NF4 weight with an r = 64 adapter
  adamw_65b     AdamW step over the adapters of the 65B-shaped block (flat fp32)
Inputs are drawn on the device from fixed seeds; every run exits 0 on success.
"""

import argparse
import sys

import torch

from . import binding as bd


def _layer(n, k, m, r=64, seed=1):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    w = (torch.randn(n, k, generator=g, device="cuda") * 0.02).to(torch.bfloat16)
    x = torch.randn(m, k, generator=g, device="cuda").to(torch.bfloat16)
    a = (torch.randn(r, k, generator=g, device="cuda") / k ** 0.5).to(torch.bfloat16)
    b = (torch.randn(n, r, generator=g, device="cuda") * 0.01).to(torch.bfloat16)
    dy = torch.randn(m, n, generator=g, device="cuda").to(torch.bfloat16)
    return w, x, a, b, dy


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("case")
    ap.add_argument("--reps", type=int, default=3)
    args = ap.parse_args(argv)
    c = args.case
    torch.cuda.set_device(0)
    if c.startswith(("fwd", "bwd")):
        n, k, m = {"8192": (8192, 8192, 4096), "11008": (11008, 4096, 2048), "65b_up": (22016, 8192, 4096),
                   "65b_down": (8192, 22016, 4096)}[c.split("_", 1)[1]]
        w, x, a, b, dy = _layer(n, k, m)
        q = bd.quantize(w)
        y, t = bd.linear_fwd(q, a, b, 16.0, x)
        ws_f = bd.new_workspace(bd.workspace_bytes(m, n, k, 64, False))
        ws_b = bd.new_workspace(bd.workspace_bytes(m, n, k, 64, True))
        for _ in range(args.reps):
            if c.startswith("fwd"):
                bd.linear_fwd(q, a, b, 16.0, x, ws=ws_f, out=y, t_out=t)
            else:
                bd.linear_bwd(q, a, b, 16.0, x, dy, t, ws=ws_b)
        st = bd.read_status(ws_f) or bd.read_status(ws_b)
    elif c == "gemv_multi16":
        w, x, _, _, _ = _layer(11008, 4096, 16)
        q = bd.quantize(w)
        ads = []
        for i in range(16):
            _, _, a, b, _ = _layer(11008, 4096, 1, seed=100 + i)
            ads.append((a, b, 16.0))
        ws = bd.new_workspace(bd.workspace_bytes_multi(16, 11008, 4096, 64))
        for _ in range(args.reps):
            bd.linear_fwd_multi(q, ads, list(range(16)), x, ws=ws)
        st = bd.read_status(ws)
    elif c.startswith("gemv"):
        m = int(c.split("_m")[1])
        w, x, a, b, _ = _layer(11008, 4096, m)
        q = bd.quantize(w)
        ws = bd.new_workspace(bd.workspace_bytes(m, 11008, 4096, 64, False))
        for _ in range(args.reps):
            bd.linear_fwd(q, a, b, 16.0, x, ws=ws)
        st = bd.read_status(ws)
    elif c in ("quant_11008", "dequant_11008", "quant_4096", "dequant_4096"):
        w, *_ = _layer(11008 if c.endswith("11008") else 4096, 4096, 1)
        ws = bd.new_workspace(bd.STATUS_BYTES)
        q = bd.quantize(w, ws=ws)
        out = torch.empty_like(w)
        for _ in range(args.reps):
            if c.startswith("quant"):
                bd.quantize(w, out=q, ws=ws)
            else:
                bd.dequantize(q, out=out)
        st = bd.read_status(ws)
    elif c == "merge_8192":
        w, _, a, b, _ = _layer(8192, 8192, 1)
        q = bd.quantize(w)
        del w
        out = torch.empty(8192, 8192, dtype=torch.bfloat16, device="cuda")
        for _ in range(args.reps):
            bd.merge(q, a, b, 16.0, out=out)
        st = 0
    elif c == "adamw_65b":
        n = sum(64 * k + nn * 64 for nn, k in ((8192, 8192),) * 4 + ((22016, 8192),) * 2 + ((8192, 22016),))
        p, g, m, v = (torch.randn(n, device="cuda") * 0.01 for _ in range(4))
        v.abs_()
        p16 = torch.empty(n, dtype=torch.bfloat16, device="cuda")
        for i in range(args.reps):
            bd.adamw_step(p, g, m, v, i + 1, 1e-4, weight_decay=0.01, p_bf16=p16)
        st = 0
    else:
        raise SystemExit(f"unknown case {c}")
    torch.cuda.synchronize()
    if st:
        raise SystemExit(f"device status {bd.STATUS_NAMES[st]}")
    print(f"{c}: ok")


if __name__ == "__main__":
    sys.exit(main())
