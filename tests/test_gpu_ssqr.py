"""GPU parity of SSQR against the float64 oracle.

Page: "The Geometry of LLM Quantization: GPTQ as Babai's Nearest Plane
Algorithm", §3 (SSQR) and §2.3 (Satz 5).  The GPU receives the oracle's own
preparation (U rounded to float32, perm, dead), so no value the oracle sees
comes from the CUDA path.

Tolerances (the hot path's criterion, with the float32 bound stated below):
  * a (code, outlier flag) pair may differ only where the oracle's
    pre-rounding value lies within 1e-4 code units of a rounding boundary, at
    most 0.1 % of the weights; zeros equal except at such a near-tie; layer
    loss to 1e-3 relative;
  * scales agree to 1e-5 relative in every group of at least 32 columns.  A
    trailing group of a few columns (n mod group small) is held to the
    forward-error bound of the float32 propagation that built its values
    instead: its range spans only a few values, after the most updates;
  * a kept value agrees with the oracle's current value to 1e-5 of
    |w| + s₀·(2^b − 1) (float32 against float64 current values), with the
    same float32 forward-error allowance in a narrow trailing group;
  * the binary search: both sides evaluate the same float32 midpoints as long
    as their decisions agree; a decision may differ only where the oracle's
    outlier count lies within the code-flip allowance of the budget.
"""
import numpy as np
import pytest
import torch

from oracle import gptq as og
from oracle import ssqr as osq
from workloads import cone_activations, student_t_weights

from . import parity as P

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
VAL_RTOL = 1e-5


def _g():
    import post_weight_quantization_08_b200 as g
    return g


def _setup(m, n, order, seed, T=2048, wdtype=torch.float32):
    X = cone_activations(T, n, seed).to(torch.bfloat16)
    W = student_t_weights(m, n, seed + 1).to(wdtype)
    H = og.hessian(X.to(torch.float64).numpy())
    prep = og.prepare(H, 0.01, order)
    U32 = prep["U"].astype(np.float32)
    gp = {"U": torch.from_numpy(U32).to(DEV),
          "perm": torch.from_numpy(prep["perm"].astype(np.int32)).to(DEV),
          "dead": torch.from_numpy(prep["dead"].astype(np.uint8)).to(DEV)}
    Wz = W.to(torch.float64).numpy().copy()
    Wz[:, prep["dead"]] = 0.0
    return W, H, prep, U32, gp, Wz


def _dense_outliers(q, m, n):
    rp = q["row_ptr"].cpu().numpy()
    ci = q["col_idx"].cpu().numpy()
    vv = q["val"].cpu().numpy()
    mask = np.zeros((m, n), bool)
    vals = np.zeros((m, n), np.float64)
    rows = np.repeat(np.arange(m), np.diff(rp))
    mask[rows, ci] = True
    vals[rows, ci] = vv
    # CSR: columns ascending within each row, no duplicates
    for r in range(m):
        c = ci[rp[r]:rp[r + 1]]
        assert np.all(np.diff(c) > 0)
    return mask, vals


def _check_outputs(q, W, Wz, prep, U32, bits, group, block, alpha):
    m, n = W.shape
    codes = P.unpack_rows(q["qweight"].cpu().numpy(), bits, n)
    scale = q["scale"].cpu().numpy()
    zero = q["zero"].cpu().numpy().astype(np.float32)
    mask, vals = _dense_outliers(q, m, n)
    perm = prep["perm"]
    f = osq.follow_ssqr(Wz[:, perm], U32.astype(np.float64), bits, group, block, alpha,
                        codes[:, perm], mask[:, perm], vals[:, perm], scale, zero)
    assert f["n_bad"] == 0 and f["z_bad"] == 0, f
    assert f["n_diff"] <= P.CODE_FRAC * m * n, f
    assert f["z_diff"] <= P.ZERO_FRAC * zero.size, f
    assert f["scale_bad"] == 0 and f["scale_wide_over"] == 0 and f["val_bad"] == 0, f
    if n % group == 0 or n % group >= 32:
        assert f["max_scale_rel"] <= P.SCALE_RTOL, f
        assert f["max_val_rel"] <= VAL_RTOL, f
    loss_or = float(np.sum(f["err"] ** 2))
    loss_gpu = float(q["loss_row"].cpu().to(torch.float64).sum())
    assert abs(loss_gpu - loss_or) <= P.LOSS_RTOL * loss_or + 1e-10 * float(np.sum(Wz ** 2))
    if q.get("Qdq") is not None:
        g_idx = q["g_idx"].cpu().numpy()
        deq = scale[:, g_idx] * (codes.astype(np.float32) - zero[:, g_idx])
        want = np.where(mask, vals, deq)
        got = q["Qdq"].cpu().numpy()
        assert np.allclose(got, want, rtol=0, atol=1e-7 * np.abs(want).max())
    return f, mask


@pytest.mark.parametrize("m,n,bits,group,block,alpha,order", [
    (300, 320, 3, 64, 128, 0.5, "act"),       # ragged rows, 2½ blocks
    (128, 576, 4, 128, 128, 0.8, "act"),      # 4½ blocks, one row tile
    (257, 96, 2, 32, 32, 0.7, "natural"),     # a tile of one row, many blocks
    (64, 200, 3, 32, 64, 1.0, "reverse"),     # α = 1: only propagated overflow
    (50, 130, 3, 32, 64, 0.6, "act"),         # n % 4 ≠ 0: the SIMT trailing path
])
def test_fixed_alpha_matches_oracle(m, n, bits, group, block, alpha, order):
    g = _g()
    W, H, prep, U32, gp, Wz = _setup(m, n, order, 101)
    q = g.ssqr_quantize(W.to(DEV), gp, bits, group, block, target=1.0, iters=0,
                        alpha_lo=alpha, alpha_hi=alpha, nnz_cap=m * n, want_qdq=True,
                        want_trace=True)
    torch.cuda.synchronize()
    assert float(q["alpha"].cpu()[0]) == np.float32(alpha)
    f, mask = _check_outputs(q, W, Wz, prep, U32, bits, group, block, np.float32(alpha))
    assert int(q["trace_count"].cpu()[0]) == int(mask.sum())
    if alpha < 1:
        assert mask.sum() > 0


def _oracle_search(Wp, U, bits, group, block, n_max, iters, lo, hi):
    return osq.bisect_alpha(lambda a: osq.ssqr_blocked(Wp, U, bits, group, block, a),
                            n_max, iters, lo, hi)


@pytest.mark.parametrize("m,n,bits,group,target,wdtype,iters,lookahead", [
    (576, 576, 3, 128, 0.01, torch.bfloat16, 10, True),   # a SmolLM-135M attention projection
    (576, 576, 3, 128, 0.01, torch.bfloat16, 10, False),  # one pass a step: the same trace
    (192, 576, 2, 64, 0.005, torch.float32, 9, True),     # an odd step count
    (300, 260, 4, 32, 0.02, torch.float32, 10, True),     # a trailing group of 4 columns
])
def test_binary_search_matches_oracle(m, n, bits, group, target, wdtype, iters, lookahead):
    g = _g()
    W, H, prep, U32, gp, Wz = _setup(m, n, "act", 202, wdtype=wdtype)
    q = g.ssqr_quantize(W.to(DEV), gp, bits, group, 128, target=target, iters=iters,
                        want_qdq=True, want_trace=True, lookahead=lookahead)
    torch.cuda.synchronize()
    ta = q["trace_alpha"].cpu().numpy()
    tc = q["trace_count"].cpu().numpy()
    n_max = osq.max_outliers(target, m, n)
    a_or, _, trace_or = _oracle_search(Wz[:, prep["perm"]], U32.astype(np.float64), bits,
                                       group, 128, n_max, iters, 1.0 / 16, 1.0)
    allow = int(P.CODE_FRAC * m * n)
    diverged = False
    for k, (a_o, c_o) in enumerate(trace_or):
        assert ta[k] == np.float32(a_o), (k, ta[k], a_o)
        assert abs(int(tc[k]) - c_o) <= allow, (k, tc[k], c_o)
        if (tc[k] <= n_max) != (c_o <= n_max):
            assert abs(c_o - n_max) <= allow     # an ambiguous decision
            diverged = True
            break
    alpha = float(q["alpha"].cpu()[0])
    if not diverged:
        assert alpha == np.float32(a_or)
    # the last pass reproduces the accepted pass's count (deterministic kernels)
    nnz = int(q["row_ptr"][-1])
    acc = [int(c) for a, c in zip(ta, tc) if c >= 0 and a == np.float32(alpha)]
    assert acc and acc[-1] == nnz and nnz <= n_max
    _check_outputs(q, W, Wz, prep, U32, bits, group, 128, np.float32(alpha))


def test_over_budget_at_the_upper_end_stops_there():
    g = _g()
    m, n = 128, 256
    W, H, prep, U32, gp, Wz = _setup(m, n, "act", 303)
    q = g.ssqr_quantize(W.to(DEV), gp, 3, 128, 128, target=0.0, iters=6, alpha_lo=0.25,
                        alpha_hi=0.5, nnz_cap=m * n, want_trace=True)
    torch.cuda.synchronize()
    tc = q["trace_count"].cpu().numpy()
    assert float(q["alpha"].cpu()[0]) == 0.5
    assert tc[0] > 0 and np.all(tc[1:] == -1)
    assert int(q["row_ptr"][-1]) == tc[0] == q["col_idx"].numel()
    _check_outputs(q, W, Wz, prep, U32, 3, 128, 128, np.float32(0.5))


def test_capacity_is_reported_and_row_pointers_stay_complete():
    g = _g()
    m, n = 64, 128
    W, H, prep, U32, gp, Wz = _setup(m, n, "natural", 404)
    q = g.ssqr_quantize(W.to(DEV), gp, 2, 32, 64, target=1.0, iters=0, alpha_lo=0.3,
                        alpha_hi=0.3, nnz_cap=3, check=False)
    st, _ = g.gptq_check(q["info"])
    assert st == 7                                   # GPTQ_ERR_CAPACITY
    rp = q["row_ptr"].cpu().numpy()
    assert rp[0] == 0 and rp[-1] > 3 and np.all(np.diff(rp) >= 0)
    with pytest.raises(g.GptqError):
        g.ssqr_quantize(W.to(DEV), gp, 2, 32, 64, target=1.0, iters=0, alpha_lo=0.3,
                        alpha_hi=0.3, nnz_cap=3)


def test_the_whole_search_replays_from_a_cuda_graph():
    """No host round trip inside the call: captured once, replayed, the same
    outputs as the eager call."""
    g = _g()
    m, n = 256, 384
    W, H, prep, U32, gp, Wz = _setup(m, n, "act", 505)
    Wd = W.to(DEV)
    ref = g.ssqr_quantize(Wd, gp, 3, 128, 128, target=0.01, iters=8, want_trace=True)
    torch.cuda.synchronize()
    ws = g.workspace(g.gptq_ssqr_workspace_bytes(m, n, 128), DEV)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        warm = g.ssqr_quantize(Wd, gp, 3, 128, 128, target=0.01, iters=8, want_trace=True,
                               nnz_cap=m * n, ws=ws, stream=s, check=False)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        out = g.ssqr_quantize(Wd, gp, 3, 128, 128, target=0.01, iters=8, want_trace=True,
                              nnz_cap=m * n, ws=ws, stream=s, check=False)
    for k in ("qweight", "scale", "row_ptr"):
        out[k].zero_()
    graph.replay()
    torch.cuda.synchronize()
    del warm
    nnz = int(ref["row_ptr"][-1])
    for k in ("qweight", "scale", "zero", "row_ptr", "alpha", "trace_alpha", "trace_count"):
        assert torch.equal(out[k], ref[k]), k
    assert torch.equal(out["col_idx"][:nnz], ref["col_idx"])
    assert torch.equal(out["val"][:nnz], ref["val"])


def test_argument_errors():
    g = _g()
    W = student_t_weights(64, 64, 7).to(DEV)
    prep = g.prepare(torch.eye(64, device=DEV) * 2.0)
    with pytest.raises(g.GptqError):
        g.ssqr_quantize(W, prep, 8, 32, 64)          # bits
    with pytest.raises(g.GptqError):
        g.ssqr_quantize(W, prep, 3, 32, 64, target=1.5)
    with pytest.raises(g.GptqError):
        g.ssqr_quantize(W, prep, 3, 32, 64, alpha_lo=0.5, alpha_hi=0.25)


@pytest.mark.parametrize("m,n,alpha", [(130, 200, 0.6), (1, 96, 0.5)])
def test_dead_columns_zero_rows_and_one_row(m, n, alpha):
    """Dead columns (inputs that never fire: W zeroed there, never an outlier),
    an all-zero weight row (its groups take [−1, 1]), and a single row."""
    g = _g()
    X = cone_activations(2048, n, 505).to(torch.bfloat16)
    X[:, [0, 7, n - 1]] = 0
    W = student_t_weights(m, n, 506)
    if m > 1:
        W[3] = 0
    H = og.hessian(X.to(torch.float64).numpy())
    prep = og.prepare(H, 0.01, "act")
    assert prep["dead"].sum() == 3
    U32 = prep["U"].astype(np.float32)
    gp = {"U": torch.from_numpy(U32).to(DEV),
          "perm": torch.from_numpy(prep["perm"].astype(np.int32)).to(DEV),
          "dead": torch.from_numpy(prep["dead"].astype(np.uint8)).to(DEV)}
    Wz = W.to(torch.float64).numpy().copy()
    Wz[:, prep["dead"]] = 0.0
    q = g.ssqr_quantize(W.to(DEV), gp, 3, 32, 64, target=1.0, iters=0, alpha_lo=alpha,
                        alpha_hi=alpha, nnz_cap=m * n, want_qdq=True)
    torch.cuda.synchronize()
    f, mask = _check_outputs(q, W, Wz, prep, U32, 3, 32, 64, np.float32(alpha))
    assert not mask[:, prep["dead"]].any()
    if m > 1:
        assert not mask[3].any()
        assert np.all(q["Qdq"].cpu().numpy()[3] == 0)
