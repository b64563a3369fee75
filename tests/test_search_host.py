"""The library's binary search on the scale factor (SSQR and HPTQ), run on the
host from the same source (csrc/search.cuh, compiled host-side), against the
oracle's bisection.

For a deliberately non-monotone measure of α (SplitMix64 of α's float bits),
one pass a step and the lookahead rounds (three candidates, two steps a round)
must both reproduce the oracle's trace (α, measure) entry for entry, and its
final α, over many seeds, budgets, step counts and brackets, including
degenerate ones (an empty bracket, adjacent floats, a budget nothing meets).
"""
import os
import shutil
import subprocess

import numpy as np
import pytest

from oracle import ssqr as osq

HERE = os.path.dirname(os.path.abspath(__file__))
M64 = (1 << 64) - 1


def _measure(a, seed, span):
    x = int(np.float32(a).view(np.uint32)) ^ seed
    x = (x + 0x9E3779B97F4A7C15) & M64
    x = ((x ^ (x >> 30)) * 0xBF58476D1CE4E5B9) & M64
    x = ((x ^ (x >> 27)) * 0x94D049BB133111EB) & M64
    x ^= x >> 31
    return x % span


@pytest.fixture(scope="module")
def sim(tmp_path_factory):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    exe = str(tmp_path_factory.mktemp("search") / "search_sim")
    src = os.path.join(HERE, "search_sim.cu")
    r = subprocess.run([nvcc, "-std=c++17", "-O2", "-gencode", "arch=compute_100a,code=sm_100a",
                        src, "-o", exe], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return exe


def _run(exe, seed, span, limit, iters, lo, hi):
    out = subprocess.run([exe, str(seed), str(span), str(limit), str(iters), repr(lo), repr(hi)],
                         capture_output=True, text=True, check=True).stdout.split("\n")
    res = {}
    for line in out:
        if not line:
            continue
        f = line.split()
        vals = f[2:]
        res[f[0]] = (np.float32(float(f[1])),
                     [(np.float32(float(vals[2 * k])), int(vals[2 * k + 1]))
                      for k in range(len(vals) // 2)])
    return res


def _cases():
    rng = np.random.default_rng(0)
    cases = []
    for i in range(120):
        span = int(rng.integers(2, 1000))
        limit = int(rng.integers(-1, span + 1))
        iters = int(rng.integers(0, 24))
        lo = float(np.float32(rng.uniform(0.01, 1.0)))
        hi = float(np.float32(lo + rng.uniform(0.0, 4.0)))
        cases.append((i + 1, span, limit, iters, lo, hi))
    # degenerate brackets: empty, adjacent floats, three floats wide
    a = np.float32(0.75)
    cases += [(900, 50, 25, 6, float(a), float(a)),
              (901, 50, 25, 6, float(a), float(np.nextafter(a, np.float32(2)))),
              (902, 50, 25, 9, float(a), float(np.nextafter(np.nextafter(np.nextafter(
                  a, np.float32(2)), np.float32(2)), np.float32(2))))]
    return cases


@pytest.mark.parametrize("seed,span,limit,iters,lo,hi", _cases())
def test_library_search_equals_the_oracle_bisection(sim, seed, span, limit, iters, lo, hi):
    res = _run(sim, seed, span, limit, iters, lo, hi)
    run = lambda a: {"mask": np.ones(_measure(a, seed, span), bool)}
    alpha, _, trace = osq.bisect_alpha(run, limit, iters, lo, hi)
    for mode in ("seq", "rnd"):
        final, tr = res[mode]
        assert final == alpha, (mode, final, alpha)
        for k, (a_o, c_o) in enumerate(trace):
            assert tr[k] == (np.float32(a_o), c_o), (mode, k, tr[k], (a_o, c_o))
        assert all(c == -1 for _, c in tr[len(trace):]), (mode, tr)
    assert res["seq"] == res["rnd"]
