"""GPU parity of HPTQ against the float64 oracle.

Page: "The Geometry of LLM Quantization: GPTQ as Babai's Nearest Plane
Algorithm", §3 (HPTQ), §4 (3.125 bits) and §2.3 (Satz 5).  The GPU receives
the oracle's own preparation (U rounded to float32, perm, dead).

What is compared:
  * codes, scales and the layer loss in follow mode, with the hot
    path's tolerances (a code may differ only within 1e-4 code units of a
    rounding boundary, at most 0.1 %; scales 1e-5 relative, a narrow trailing
    group held to the float32 forward-error bound; loss 1e-3);
  * the Huffman code, where several are optimal: the GPU's lengths must form
    a complete prefix code (Kraft sum 1) whose cost on the GPU's histogram
    equals the optimum the oracle computes for that histogram; the code words
    are the canonical ones of those lengths, bit for bit;
  * the bit stream: bit for bit the oracle's encoding of the GPU's codes with
    the GPU's lengths, and it decodes back to the codes;
  * the search: the same float32 midpoints while decisions agree; coded sizes
    within the allowance of the code flips; a differing decision only where
    the oracle's size lies within that allowance of the budget.
"""
import numpy as np
import pytest
import torch

from oracle import gptq as og
from oracle import hptq as oh
from workloads import cone_activations, student_t_weights

from . import parity as P

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
SYM0 = 2048


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
    return W, prep, U32, gp, Wz


def _table(q):
    lens = q["code_len"].cpu().numpy().astype(np.int64)
    words = q["code_word"].cpu().numpy().view(np.uint64)
    return ({s - SYM0: int(lens[s]) for s in np.nonzero(lens)[0]},
            {s - SYM0: (int(words[s]), int(lens[s])) for s in np.nonzero(lens)[0]})


def _check_outputs(q, W, Wz, prep, U32, bits, group, block, alpha):
    m, n = W.shape
    codes = q["codes"].cpu().numpy().astype(np.int64)
    scale = q["scale"].cpu().numpy()
    perm = prep["perm"]
    f = oh.follow_hptq(Wz[:, perm], U32.astype(np.float64), bits, group, block, alpha,
                       codes[:, perm], scale)
    assert f["n_bad"] == 0, f
    assert f["n_diff"] <= P.CODE_FRAC * m * n, f
    assert f["scale_bad"] == 0 and f["scale_wide_over"] == 0, f
    if n % group == 0 or n % group >= 32:
        assert f["max_scale_rel"] <= P.SCALE_RTOL, f
    loss_or = float(np.sum(f["err"] ** 2))
    loss_gpu = float(q["loss_row"].cpu().to(torch.float64).sum())
    assert abs(loss_gpu - loss_or) <= P.LOSS_RTOL * loss_or + 1e-10 * float(np.sum(Wz ** 2))
    # the code: complete, optimal for the GPU's own histogram, canonical words
    lens, words = _table(q)
    hist = oh.histogram(codes)
    assert set(hist) == set(lens)
    if len(lens) > 1:
        assert oh.kraft(lens) == 1.0
    assert oh.cost(hist, lens) == oh.cost(hist, oh.huffman_lengths(hist))
    assert words == oh.canonical_codes(lens)
    # the stream: the oracle's encoding of the same codes and lengths
    ro_or, st_or = oh.encode(codes, lens)
    ro = q["row_off"].cpu().numpy()
    st = q["stream"].cpu().numpy().view(np.uint32)
    assert np.array_equal(ro, ro_or)
    assert np.array_equal(st[:st_or.size], st_or)
    if m * n <= 40_000:
        assert np.array_equal(oh.decode(st, ro, lens, m, n), codes)
    if q.get("Qdq") is not None:
        g_idx = q["g_idx"].cpu().numpy()
        want = scale[:, g_idx] * codes.astype(np.float32)
        assert np.allclose(q["Qdq"].cpu().numpy(), want, rtol=0, atol=1e-7 * np.abs(want).max())
    return f, codes


@pytest.mark.parametrize("m,n,bits,group,block,alpha,order", [
    (300, 320, 4, 64, 128, 1.0, "act"),       # ragged rows, 2½ blocks
    (128, 576, 3, 128, 128, 0.7, "act"),      # 4½ blocks
    (257, 96, 2, 32, 32, 2.0, "natural"),     # a coarse grid, many blocks
    (50, 130, 4, 32, 64, 1.3, "act"),         # n % 4 ≠ 0: the SIMT trailing path
    (1, 40, 8, 32, 32, 1.0, "reverse"),       # one row, 8 nominal bits
])
def test_fixed_alpha_matches_oracle(m, n, bits, group, block, alpha, order):
    g = _g()
    W, prep, U32, gp, Wz = _setup(m, n, order, 111)
    q = g.hptq_quantize(W.to(DEV), gp, bits, group, block, budget=64.0, iters=0,
                        alpha_lo=alpha, alpha_hi=alpha, stream_cap=2 * n * m + 64,
                        want_qdq=True, want_trace=True)
    torch.cuda.synchronize()
    assert float(q["alpha"].cpu()[0]) == np.float32(alpha)
    _, codes = _check_outputs(q, W, Wz, prep, U32, bits, group, block, np.float32(alpha))
    assert int(q["trace_bits"].cpu()[0]) == int(q["row_off"][-1])
    if alpha < 1:
        half = 2 ** (bits - 1)
        assert codes.min() < -half or codes.max() >= half   # the grid is unbounded


@pytest.mark.parametrize("m,n,bits,group,budget,wdtype,iters,lookahead", [
    (576, 576, 4, 128, 3.125, torch.bfloat16, 10, True),  # SmolLM-135M, the page's budget
    (576, 576, 4, 128, 3.125, torch.bfloat16, 10, False), # one pass a step: the same trace
    (192, 576, 3, 64, 2.5, torch.float32, 9, True),       # an odd step count
    (300, 260, 4, 32, 3.125, torch.float32, 10, True),    # a trailing group of 4 columns
])
def test_binary_search_matches_oracle(m, n, bits, group, budget, wdtype, iters, lookahead):
    g = _g()
    W, prep, U32, gp, Wz = _setup(m, n, "act", 222, wdtype=wdtype)
    q = g.hptq_quantize(W.to(DEV), gp, bits, group, 128, budget=budget, iters=iters,
                        want_qdq=True, want_trace=True, lookahead=lookahead)
    torch.cuda.synchronize()
    ta = q["trace_alpha"].cpu().numpy()
    tb = q["trace_bits"].cpu().numpy()
    b_max = oh.max_bits(budget, m, n)
    a_or, _, trace_or = oh.bisect_alpha(
        lambda a: oh.hptq_blocked(Wz[:, prep["perm"]], U32.astype(np.float64), bits, group,
                                  128, a), b_max, iters, 1.0 / 16, 16.0)
    allow = 2 * 64 * int(P.CODE_FRAC * m * n)
    diverged = False
    for k, (a_o, b_o) in enumerate(trace_or):
        assert ta[k] == np.float32(a_o), (k, ta[k], a_o)
        assert abs(int(tb[k]) - b_o) <= allow, (k, tb[k], b_o)
        if (tb[k] <= b_max) != (b_o <= b_max):
            assert abs(b_o - b_max) <= allow
            diverged = True
            break
    alpha = float(q["alpha"].cpu()[0])
    if not diverged:
        assert alpha == np.float32(a_or)
    nbits = int(q["row_off"][-1])
    acc = [int(b) for a, b in zip(ta, tb) if b >= 0 and a == np.float32(alpha)]
    assert acc and acc[-1] == nbits
    # within budget, unless already the coarsest grid was over it
    assert nbits <= b_max or (alpha == np.float32(16.0) and np.all(tb[1:] == -1))
    _check_outputs(q, W, Wz, prep, U32, bits, group, 128, np.float32(alpha))


def test_capacity_is_reported_and_row_offsets_stay_complete():
    g = _g()
    m, n = 64, 128
    W, prep, U32, gp, Wz = _setup(m, n, "natural", 333)
    q = g.hptq_quantize(W.to(DEV), gp, 4, 32, 64, budget=64.0, iters=0, alpha_lo=1.0,
                        alpha_hi=1.0, stream_cap=5, check=False)
    st, _ = g.gptq_check(q["info"])
    assert st == 7                                   # GPTQ_ERR_CAPACITY
    ro = q["row_off"].cpu().numpy()
    assert ro[0] == 0 and ro[-1] > 5 * 32 and np.all(np.diff(ro) > 0)


def test_the_whole_search_replays_from_a_cuda_graph():
    g = _g()
    m, n = 256, 384
    W, prep, U32, gp, Wz = _setup(m, n, "act", 444)
    Wd = W.to(DEV)
    ref = g.hptq_quantize(Wd, gp, 4, 128, 128, budget=3.125, iters=8, want_trace=True)
    torch.cuda.synchronize()
    ws = g.workspace(g.gptq_hptq_workspace_bytes(m, n, 128), DEV)
    cap = ref["stream"].numel() + 16
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        g.hptq_quantize(Wd, gp, 4, 128, 128, budget=3.125, iters=8, want_trace=True,
                        stream_cap=cap, ws=ws, stream=s, check=False)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        out = g.hptq_quantize(Wd, gp, 4, 128, 128, budget=3.125, iters=8, want_trace=True,
                              stream_cap=cap, ws=ws, stream=s, check=False)
    for k in ("codes", "row_off", "stream"):
        out[k].zero_()
    graph.replay()
    torch.cuda.synchronize()
    for k in ("codes", "scale", "code_len", "code_word", "row_off", "alpha",
              "trace_alpha", "trace_bits"):
        assert torch.equal(out[k], ref[k]), k
    assert torch.equal(out["stream"][:ref["stream"].numel()], ref["stream"])


def test_argument_errors():
    g = _g()
    W = student_t_weights(64, 64, 7).to(DEV)
    prep = g.prepare(torch.eye(64, device=DEV) * 2.0)
    with pytest.raises(g.GptqError):
        g.hptq_quantize(W, prep, 5, 32, 64)           # bits
    with pytest.raises(g.GptqError):
        g.hptq_quantize(W, prep, 4, 32, 64, budget=0.0)
    with pytest.raises(g.GptqError):
        g.hptq_quantize(W, prep, 4, 32, 64, alpha_lo=2.0, alpha_hi=1.0)


@pytest.mark.parametrize("m,n,alpha", [(130, 200, 0.6), (1, 96, 2.0)])
def test_dead_columns_zero_rows_and_one_row(m, n, alpha):
    """Dead columns and an all-zero row code as the lattice point 0; a single
    row, on a coarse grid, may leave one symbol (coded in 1 bit)."""
    g = _g()
    X = cone_activations(2048, n, 515).to(torch.bfloat16)
    X[:, [0, 7, n - 1]] = 0
    W = student_t_weights(m, n, 516)
    if m > 1:
        W[3] = 0
    H = og.hessian(X.to(torch.float64).numpy())
    prep = og.prepare(H, 0.01, "act")
    U32 = prep["U"].astype(np.float32)
    gp = {"U": torch.from_numpy(U32).to(DEV),
          "perm": torch.from_numpy(prep["perm"].astype(np.int32)).to(DEV),
          "dead": torch.from_numpy(prep["dead"].astype(np.uint8)).to(DEV)}
    Wz = W.to(torch.float64).numpy().copy()
    Wz[:, prep["dead"]] = 0.0
    q = g.hptq_quantize(W.to(DEV), gp, 4, 32, 64, budget=64.0, iters=0, alpha_lo=alpha,
                        alpha_hi=alpha, stream_cap=2 * m * n + 64, want_qdq=True)
    torch.cuda.synchronize()
    _, codes = _check_outputs(q, W, Wz, prep, U32, 4, 32, 64, np.float32(alpha))
    assert np.all(codes[:, prep["dead"]] == 0)
    if m > 1:
        assert np.all(codes[3] == 0)


def test_a_single_symbol_codes_in_one_bit():
    """An all-zero matrix: every coordinate is 0, one symbol, 1 bit a weight."""
    g = _g()
    m, n = 40, 64
    X = cone_activations(256, n, 525).to(torch.bfloat16)
    prep = og.prepare(og.hessian(X.to(torch.float64).numpy()), 0.01, "act")
    gp = {"U": torch.from_numpy(prep["U"].astype(np.float32)).to(DEV),
          "perm": torch.from_numpy(prep["perm"].astype(np.int32)).to(DEV),
          "dead": torch.from_numpy(prep["dead"].astype(np.uint8)).to(DEV)}
    q = g.hptq_quantize(torch.zeros(m, n, device=DEV), gp, 4, 32, 64, budget=1.0, iters=4)
    torch.cuda.synchronize()
    lens = q["code_len"].cpu().numpy()
    assert lens[2048] == 1 and lens.sum() == 1
    assert int(q["row_off"][-1]) == m * n
    assert np.all(q["codes"].cpu().numpy() == 0)
    assert np.all(q["stream"].cpu().numpy() == 0)
