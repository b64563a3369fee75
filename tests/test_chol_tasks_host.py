"""The dataflow factorisation's task numbering (csrc/chol_tasks.cuh, compiled
host-side): every tile task decoded exactly once, and every dependency, on a
worker task or on a step of the chain, ordered before the task that waits for
it, so that tasks claimed in order by running CTAs cannot deadlock.  Block
counts cover the smallest cases, the workloads' sizes (576, 896, 1536, 2048,
4864, 5632 and 8192 columns are 9, 14, 24, 32, 76, 88 and 128 blocks) and a
few in between."""
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
    exe = str(tmp_path_factory.mktemp("chol") / "chol_tasks_sim")
    r = subprocess.run([nvcc, "-std=c++17", "-O2", "-gencode", "arch=compute_100a,code=sm_100a",
                        os.path.join(HERE, "chol_tasks_sim.cu"), "-o", exe],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return exe


@pytest.mark.parametrize("N", list(range(1, 41)) + [57, 76, 88, 128])
def test_task_numbering(sim, N):
    out = subprocess.run([sim, str(N)], capture_output=True, text=True)
    assert out.returncode == 0, out.stdout + out.stderr
    assert out.stdout.startswith(f"ok {N} ")
