"""GPU parity at the workloads' full sizes, through the same calls bench.py makes.

The single 576×576 layer and the SmolLM-135M layer are checked in full (every
row).  For the Qwen2.5-0.5B and TinyLlama-1.1B layers and the 8192² stress
layer the GPU runs the whole problem and the oracle checks the Hessian and U
in full (float64 on the GPU's own H) and the sweep on sampled rows — a row's
result depends only on that row and U, so sampled rows are exact checks.
"""
import numpy as np
import pytest
import torch

from oracle import gptq as og
from workloads import problems_for

from . import parity as P

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
SAMPLE_ROWS = 96


def _rows(m, seed):
    rng = np.random.default_rng(seed)
    k = min(m, SAMPLE_ROWS)
    return np.sort(rng.choice(m, size=k, replace=False))


def _check_problem(p, full_rows: bool, order=None, seed=0, hessian_full=True):
    order = order or p.order
    out = P.run_gpu(p.X, p.W, p.bits, p.group, p.block, p.damp, order, None, DEV,
                    qdq=full_rows)
    stats = {}
    if hessian_full:
        stats.update(P.check_hessian(p.X, out["H"]))
    _, s2 = P.check_prepare(out["H"], out, p.damp, order)
    stats.update(s2)
    rows = None if full_rows else _rows(p.m, seed)
    stats.update(P.check_quantize(p.W, out, None, p.bits, p.group, p.block, rows=rows))
    if full_rows:
        stats.update(P.check_layer_loss(p.X, p.W, out, p.bits, p.group, p.block, p.damp, order))
    # round-to-nearest dominance on the whole problem (every row), with the
    # float64 Hessian on the fully checked sizes and the GPU's checked H else
    if full_rows:
        H = og.hessian(p.X.to(torch.float64).numpy())
    else:
        H = out["H"].astype(np.float64)
    stats.update(P.check_rtn_dominance(p.W, out, H, p.bits, p.group))
    return stats, out


def _check_hessian_tiles(X, H, tiles=24, seed=5):
    """A float32 H of a large problem against float64 2·XᵀX on seeded 128×128
    tiles spread over the whole matrix: diagonal tiles, tiles far from the
    diagonal, and their mirrors in the lower triangle; H exactly symmetric."""
    assert np.array_equal(H, H.T), "Hessian not symmetric"
    n, T = H.shape[0], X.shape[0]
    nt = -(-n // 128)
    rng = np.random.default_rng(seed)
    picks = {(0, 0), (nt - 1, nt - 1), (0, nt - 1), (nt - 1, 0)}
    while len(picks) < tiles:
        i, j = (int(v) for v in rng.integers(0, nt, size=2))
        picks.add((i, j))
        picks.add((j, i))
    Xs = X.to(torch.float64)
    worst = 0.0
    for i, j in sorted(picks):
        r0, r1, c0, c1 = 128 * i, min(128 * i + 128, n), 128 * j, min(128 * j + 128, n)
        A, B = Xs[:, r0:r1].numpy(), Xs[:, c0:c1].numpy()
        ref = og.hessian_block(A, B)
        S = 2.0 * (np.abs(A).T @ np.abs(B))
        tol = 2.0 * T * 2.0 ** -24 * S + 1e-30
        ratio = float(np.max(np.abs(H[r0:r1, c0:c1] - ref) / tol))
        assert ratio <= 1.0, ((i, j), ratio)
        worst = max(worst, ratio)
    return {"tiles": len(picks), "hessian_err_over_bound": worst}


def test_single_layer_full():
    p = problems_for(0)[0]
    st, _ = _check_problem(p, full_rows=True)
    assert st["code_diff"] <= 1e-3 * st["codes"]


@pytest.mark.parametrize("which", [0, 1])
def test_smollm_layer_full(which):
    p = problems_for(1)[which]
    st, _ = _check_problem(p, full_rows=True)
    assert st["code_diff"] <= 1e-3 * st["codes"]


@pytest.mark.parametrize("which", [0, 1])
def test_qwen_layer_sampled(which):
    p = problems_for(2, layer=3)[which]
    _check_problem(p, full_rows=False, seed=which)


@pytest.mark.parametrize("bits,which", [(4, 0), (4, 1), (3, 1)])
def test_tinyllama_layer_sampled(bits, which):
    p = problems_for(3, layer=5, bits=bits)[which]
    _check_problem(p, full_rows=False, seed=bits * 10 + which)


@pytest.mark.parametrize("order", ["act", "reverse"])
def test_stress_layer_sampled(order):
    p = problems_for(4, order=order)[0]
    # the float64 Hessian of 16384×8192 is checked on sampled tiles
    _, out = _check_problem(p, full_rows=False, order=order, seed=7, hessian_full=False)
    st = _check_hessian_tiles(p.X, out["H"], seed=3 if order == "act" else 4)
    assert st["tiles"] >= 24


def test_smollm_down_min_pivot():
    """The SmolLM down projection (576×1536) under the min-pivot order, every row."""
    p = problems_for(1, order="minpivot")[1]
    st, _ = _check_problem(p, full_rows=True)
    assert st["code_diff"] <= 1e-3 * st["codes"]
