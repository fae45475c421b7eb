"""The benchmark's reference arm and FLOP accounting, on the CPU.

`bench.py --impl reference` times the oracle on the host cores and prints one
JSON line; under torchrun only rank 0 works and prints.
"""

import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from bit_nf4_quantized_27_b200 import inputs as I  # noqa: E402


def _run(extra_env=None):
    env = dict(os.environ)
    env.update(extra_env or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                           "--warmup", "3", "--ref-seconds", "0.5"], capture_output=True, text=True, timeout=300,
                          env=env, cwd=ROOT)


def test_reference_arm_prints_the_contract_line():
    p = _run()
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [ln for ln in p.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["metric"] == bench.METRIC and d["unit"] == bench.UNIT
    assert d["steps"] == 1 and d["warmup"] == 3 and d["higher_is_better"] is True
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["config"]["workload"] == "65b_block_m4096_r64"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    # ms_per_step is one full step of the workload at the measured rate
    wl = I.L65B_BLOCK
    flops = sum(sum(bench.layer_flops(wl.m, ly.n, ly.k, wl.r)) for ly in wl.layers)
    assert d["ms_per_step"] == pytest.approx(flops / (d["value"] * 1e12) * 1e3, rel=1e-9)


def test_reference_arm_other_ranks_exit_without_work():
    p = _run({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert p.returncode == 0, p.stderr[-2000:]
    assert not [ln for ln in p.stdout.splitlines() if ln.startswith("{")]


def test_layer_flops_definition():
    # forward 2MNK + 2Mr(N + K); backward 2MNK (dX) + 4Mr(N + K) (U, s U A, dA, dB)
    m, n, k, r = 4096, 22016, 8192, 64
    f, b = bench.layer_flops(m, n, k, r)
    assert f == 2 * m * n * k + 2 * m * r * (n + k)
    assert b == 2 * m * n * k + 4 * m * r * (n + k)


def test_block_step_flops():
    wl = I.L65B_BLOCK
    assert [(ly.n, ly.k) for ly in wl.layers] == [(8192, 8192)] * 4 + [(22016, 8192)] * 2 + [(8192, 22016)]
    fwd = sum(bench.layer_flops(wl.m, ly.n, ly.k, wl.r)[0] for ly in wl.layers)
    bwd = sum(bench.layer_flops(wl.m, ly.n, ly.k, wl.r)[1] for ly in wl.layers)
    assert fwd == pytest.approx(6.713e12, rel=1e-3)
    assert bwd == pytest.approx(6.795e12, rel=1e-3)


def test_launch_count_per_step():
    # per layer: quantise, T + its split-K finish, fused GEMM, U + finish, dX, dA and dB in one launch
    assert bench.launches_per_step(7) == 56
