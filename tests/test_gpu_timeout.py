"""The device-side give-up path of the bounded waits, on the GPU, without a fault:
a one-CTA kernel waits on a barrier that nothing completes, gives up after the
limit it is given, records QLORA_ERR_TIMEOUT in the status word, waits for the
copy it has in flight and frees its tensor memory.  The context stays usable: a
normal forward call afterwards runs clean and matches the oracle."""

import time

import numpy as np
import pytest
import torch

import oracle as O
from bit_nf4_quantized_27_b200 import binding as bd
from bit_nf4_quantized_27_b200 import inputs as I

pytestmark = pytest.mark.gpu

TIMEOUT = 6  # QLORA_ERR_TIMEOUT


@pytest.mark.parametrize("limit_us", [1000, 20000])
def test_wait_gives_up_and_reports_timeout(limit_us):
    ws = bd.new_workspace(bd.STATUS_BYTES)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    bd.selftest_bounded_wait(ws, limit_us)
    st = bd.read_status(ws)  # synchronises the stream
    elapsed = time.perf_counter() - t0
    assert st == TIMEOUT
    assert elapsed >= limit_us * 1e-6  # it waited at least the limit
    assert elapsed < limit_us * 1e-6 + 2.0  # and then left
    # the status word holds exactly that flag
    assert int(ws[:4].view(torch.int32).item()) == 1 << TIMEOUT


def test_context_usable_after_timeout():
    ws = bd.new_workspace(bd.STATUS_BYTES)
    bd.selftest_bounded_wait(ws, 1000)
    assert bd.read_status(ws) == TIMEOUT
    bd.clear_status(ws)
    assert bd.read_status(ws) == 0
    # a decode-shaped and a tensor-core-shaped forward on the same context
    for m in (4, 40):
        w, x, a, b, _ = I.custom(512, 512, m, 16, 900 + m)
        ref = O.quantize(w.float().numpy(), 512, 512)
        wd = O.dequantize(ref["codes"], ref["scale_codes"], ref["c2"], 512, 512)
        q = bd.quantize(w.cuda())
        wsf = bd.new_workspace(bd.workspace_bytes(m, 512, 512, 16, False))
        y, _ = bd.linear_fwd(q, a.cuda(), b.cuda(), 16.0, x.cuda(), ws=wsf, y_dtype=torch.float32)
        assert bd.read_status(wsf) == 0
        yr, _ = O.linear_fwd(wd, a.float().numpy(), b.float().numpy(), x.float().numpy(), 16.0, 16)
        err = np.abs(y.cpu().numpy().astype(np.float64) - yr).max()
        assert err <= 1e-2 * np.sqrt(np.mean(yr ** 2)), (m, err)
