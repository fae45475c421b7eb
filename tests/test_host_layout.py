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
