"""The trailing update's schedule with super-blocks (far_range in
csrc/kernels.cuh, compiled host-side): every block's errors reach every later
column block exactly once, from the next sweep's prologue or from one far
application, and only from blocks already finished.  Covers the workloads'
column counts (576 .. 8192, partial last blocks included), 64- and 128-column
blocks, and no super-blocks (S = 1)."""
import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def sim(tmp_path_factory):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    exe = str(tmp_path_factory.mktemp("far") / "far_sim")
    r = subprocess.run([nvcc, "-std=c++17", "-O2", "-gencode", "arch=compute_100a,code=sm_100a",
                        os.path.join(HERE, "far_sim.cu"), "-o", exe],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return exe


@pytest.mark.parametrize("n", [1, 128, 129, 576, 640, 896, 1000, 1536, 2048, 4864, 5632, 8192])
@pytest.mark.parametrize("block,S", [(128, 4), (128, 1), (128, 2), (64, 1)])
def test_far_schedule(sim, n, block, S):
    out = subprocess.run([sim, str(n), str(block), str(S)], capture_output=True, text=True)
    assert out.returncode == 0, out.stdout + out.stderr
    assert out.stdout.strip() == "ok"
