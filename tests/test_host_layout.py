"""Host logic of the decode GEMV's shared-memory placement (no GPU needed).

Builds tests/host/gemv_layout_check.cu (host code including the kernel header)
and runs it: every layout the launcher can choose must fit the opt-in limit,
keep its alignments and have no overlapping buffers.
"""

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("nvcc") is None and not os.path.exists("/usr/local/cuda/bin/nvcc"),
                    reason="nvcc not available")
def test_gemv_shared_memory_layouts(tmp_path):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    exe = tmp_path / "gemv_layout_check"
    src = os.path.join(ROOT, "tests", "host", "gemv_layout_check.cu")
    b = subprocess.run([nvcc, "-std=c++17", "-O1", "-gencode", "arch=compute_100a,code=sm_100a", "-I",
                        os.path.join(ROOT, "include"), "-o", str(exe), src], capture_output=True, text=True,
                       timeout=600)
    assert b.returncode == 0, b.stderr[-3000:]
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout[-3000:]
    assert "0 failures" in r.stdout


def _oracle_switch_points():
    """Largest float32 x in [L_j, L_j+1] whose oracle code (S = 1, so x = w / S
    exactly) is <= j, by bisection on the float32 line."""
    import numpy as np

    import oracle as O

    lv = O.nf4_levels()

    def code(x):
        blk = np.zeros(64, np.float32)
        blk[0], blk[1] = 1.0, x
        return int(O.assign_codes(blk, O.block_absmax(blk), lv)[1])

    def key(f):
        u = int(np.float32(f).view(np.uint32))
        return (~u & 0xFFFFFFFF) if u & 0x80000000 else (u | 0x80000000)

    def unkey(k):
        u = (k & 0x7FFFFFFF) if k & 0x80000000 else (~k & 0xFFFFFFFF)
        return np.array([u], np.uint32).view(np.float32)[0]

    out = []
    for j in range(15):
        lo, hi = key(lv[j]), key(lv[j + 1])
        while hi - lo > 1:
            mid = (lo + hi) // 2
            if code(unkey(mid)) <= j:
                lo = mid
            else:
                hi = mid
        out.append(int(unkey(lo).view(np.uint32)))
    return out


@pytest.mark.skipif(shutil.which("nvcc") is None and not os.path.exists("/usr/local/cuda/bin/nvcc"),
                    reason="nvcc not available")
def test_quantiser_cell_table(tmp_path):
    # The kernel's cell table keeps every switch point more than 8 float32 steps
    # from every cell edge, and its switch points are the oracle's.
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    exe = tmp_path / "cell_table_check"
    src = os.path.join(ROOT, "tests", "host", "cell_table_check.cu")
    b = subprocess.run([nvcc, "-std=c++17", "-O1", "-Xcompiler", "-ffp-contract=off", "-I",
                        os.path.join(ROOT, "include"), "-o", str(exe), src], capture_output=True, text=True,
                       timeout=600)
    assert b.returncode == 0, b.stderr[-3000:]
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout[-3000:]
    lines = dict(ln.split(" ", 1) for ln in r.stdout.splitlines() if not ln.startswith("switch"))
    assert lines["ok"] == "1" and int(lines["min_edge_ulps"]) > 8
    got = [int(ln.split()[2], 16) for ln in r.stdout.splitlines() if ln.startswith("switch")]
    assert got == _oracle_switch_points()


@pytest.mark.skipif(shutil.which("nvcc") is None and not os.path.exists("/usr/local/cuda/bin/nvcc"),
                    reason="nvcc not available")
def test_decode_plans(tmp_path):
    # the one-kernel decode path: every plan fits, is aligned, has no overlapping
    # buffers, and its CTAs cover every row exactly once
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    exe = tmp_path / "decode_plan_check"
    src = os.path.join(ROOT, "tests", "host", "decode_plan_check.cu")
    b = subprocess.run([nvcc, "-std=c++17", "-O1", "-gencode", "arch=compute_100a,code=sm_100a", "-I",
                        os.path.join(ROOT, "include"), "-o", str(exe), src], capture_output=True, text=True,
                       timeout=600)
    assert b.returncode == 0, b.stderr[-3000:]
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout[-3000:]
    assert " 0 failures" in r.stdout
