"""The data-parallel path on CPU: two gloo ranks, each with its own token shard.

The adapter gradients each rank computes (here with the oracle), packed into the
flat buffer and summed by all-reduce, must equal the gradients of the whole
batch; a rank that leaves before the collective must make the other rank's
all-reduce fail within the process-group timeout instead of hanging."""

import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle as O
from bit_nf4_quantized_27_b200 import dp
from bit_nf4_quantized_27_b200 import inputs as I

SHAPES = [(96, 128), (64, 192)]  # (N, K) per layer
R, ALPHA, M = 8, 16.0, 40


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _layer_inputs(li):
    n, k = SHAPES[li]
    w, x, a, b, dy = I.custom(n, k, M, R, 5000 + 100 * li)
    q = O.quantize(w.float().numpy(), n, k)
    wd = O.dequantize(q["codes"], q["scale_codes"], q["c2"], n, k)
    return wd, a.float().numpy(), b.float().numpy(), x.float().numpy(), dy.float().numpy()


def _worker(rank, world, port, mode, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=5))
    try:
        flat = torch.zeros(dp.flat_size(SHAPES, R), dtype=torch.float64)
        views = dp.grad_views(flat, SHAPES, R)
        sl = dp.token_shard(M, world, rank)
        for li, (da_v, db_v) in enumerate(views):
            wd, a, b, x, dy = _layer_inputs(li)
            _, da, db = O.linear_bwd(wd, a, b, x[sl], dy[sl], ALPHA, R)
            da_v.copy_(torch.from_numpy(da))
            db_v.copy_(torch.from_numpy(db))
        if mode == "leave" and rank == 1:
            return  # leaves between steps, before the collective
        try:
            dp.allreduce_grads(flat)
            out[rank] = flat.numpy().copy()
        except Exception as e:  # the survivor must see an error, not hang
            out[rank] = repr(e)
    finally:
        if not (mode == "leave" and rank == 1):
            try:
                dist.destroy_process_group()
            except Exception:
                pass


def _run(mode):
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        port = _free_port()
        procs = [ctx.Process(target=_worker, args=(r, 2, port, mode, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
            if p.is_alive():
                p.kill()
                raise AssertionError("rank did not finish")
        return dict(out)


def test_shards_cover_all_tokens():
    for m in (1, 7, 40, 4096):
        for world in (1, 2, 3, 8):
            rows = []
            for r in range(world):
                s = dp.token_shard(m, world, r)
                rows.extend(range(s.start, s.stop))
            assert rows == list(range(m))


def test_grad_views_layout():
    flat = torch.arange(dp.flat_size(SHAPES, R), dtype=torch.float32)
    views = dp.grad_views(flat, SHAPES, R)
    assert [tuple(v.shape) for pair in views for v in pair] == [(R, 128), (96, R), (R, 192), (64, R)]
    assert views[0][1].data_ptr() == views[0][0].data_ptr() + 4 * R * 128
    with pytest.raises(ValueError):
        dp.grad_views(torch.zeros(3), SHAPES, R)


def test_allreduced_shards_equal_full_batch_gradient():
    out = _run("ok")
    assert set(out) == {0, 1}
    for rank in (0, 1):
        got = dp.grad_views(torch.from_numpy(out[rank]), SHAPES, R)
        for li, (da, db) in enumerate(got):
            wd, a, b, x, dy = _layer_inputs(li)
            _, da_ref, db_ref = O.linear_bwd(wd, a, b, x, dy, ALPHA, R)
            assert np.allclose(da.numpy(), da_ref, rtol=1e-12, atol=1e-12)
            assert np.allclose(db.numpy(), db_ref, rtol=1e-12, atol=1e-12)


def test_rank_leaving_fails_collective_instead_of_hanging():
    out = _run("leave")
    assert 1 not in out
    assert isinstance(out.get(0), str) and out[0]
