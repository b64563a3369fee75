"""Pins of the HPTQ oracle against what the page and the mathematics fix.

Page: "The Geometry of LLM Quantization: GPTQ as Babai's Nearest Plane
Algorithm", §3 (HPTQ: one unbounded integer grid for inliers and outliers,
Huffman-coded to a compression budget), §4 (3.125 bits) and §2.3 (Satz 5).
The Huffman code is pinned against an exhaustive search over Kraft-feasible
code lengths, a textbook example and the entropy bounds; the sweep against
scalar loops, the GPTQ oracle and the Satz 5 half step; the codec by a round
trip.  The last test plants plausible mistakes and checks each is caught.
"""
import itertools

import numpy as np
import pytest

from oracle import gptq as G
from oracle import hptq as Hq


def _spd(n, rng):
    A = rng.standard_normal((n + 3, n))
    return A.T @ A + 0.05 * np.eye(n)


def _heavy(m, n, rng, scale=0.02):
    return rng.standard_t(3, size=(m, n)) * scale


# ---------------------------------------------------------------- Huffman

def _optimal_cost_by_search(counts):
    """The least Σ c_i·l_i over integer lengths with Σ 2^−l_i ≤ 1 (Kraft:
    exactly the length vectors of prefix codes), by exhaustive search."""
    k = len(counts)
    best = None
    for ls in itertools.product(range(1, k + 1), repeat=k):
        if sum(2.0 ** -l for l in ls) <= 1.0 + 1e-12:
            c = sum(a * b for a, b in zip(counts, ls))
            best = c if best is None else min(best, c)
    return best


def test_huffman_textbook_example():
    h = {"a": 45, "b": 13, "c": 12, "d": 16, "e": 9, "f": 5}
    L = Hq.huffman_lengths(h)
    assert Hq.cost(h, L) == 224
    assert L["a"] == 1 and L["e"] == 4 and L["f"] == 4


@pytest.mark.parametrize("seed", range(12))
def test_huffman_is_optimal_against_exhaustive_search(seed):
    rng = np.random.default_rng(seed)
    k = int(rng.integers(2, 7))
    counts = [int(c) for c in rng.integers(1, 60, size=k)]
    h = {i: c for i, c in enumerate(counts)}
    L = Hq.huffman_lengths(h)
    assert Hq.cost(h, L) == _optimal_cost_by_search(counts)
    assert Hq.kraft(L) == pytest.approx(1.0, abs=1e-15)


def test_huffman_within_the_entropy_bounds():
    rng = np.random.default_rng(20)
    counts = rng.integers(1, 10_000, size=40)
    h = {i: int(c) for i, c in enumerate(counts)}
    L = Hq.huffman_lengths(h)
    p = counts / counts.sum()
    H = float(-(p * np.log2(p)).sum())
    avg = Hq.cost(h, L) / counts.sum()
    assert H <= avg < H + 1


def test_single_symbol_takes_one_bit():
    assert Hq.huffman_lengths({7: 100}) == {7: 1}


def test_canonical_code_is_prefix_free_and_round_trips():
    rng = np.random.default_rng(21)
    codes = rng.integers(-5, 9, size=(7, 23))
    codes[0, :5] = 40                                   # a rare far symbol
    L = Hq.huffman_lengths(Hq.histogram(codes))
    cb = Hq.canonical_codes(L)
    words = [format(c, f"0{ln}b") for c, ln in cb.values()]
    for a in words:
        for b in words:
            assert a == b or not b.startswith(a)
    row_off, stream = Hq.encode(codes, L)
    assert row_off[-1] == Hq.cost(Hq.histogram(codes), L)
    assert np.array_equal(Hq.decode(stream, row_off, L, 7, 23), codes)


# ---------------------------------------------------------------- the sweep

def _rtn_unclipped_by_loops(W, bits, group, alpha):
    """U = I: each weight's coordinate rint(w/s) on its group's lattice s·ℤ,
    s = α·(min-max step), by scalar float32 loops."""
    m, n = W.shape
    maxq = 2 ** bits - 1
    codes = np.zeros((m, n), np.int64)
    for r in range(m):
        for g0 in range(0, n, group):
            vals = [np.float32(W[r, c]) for c in range(g0, min(g0 + group, n))]
            lo = min(min(vals), np.float32(0))
            hi = max(max(vals), np.float32(0))
            if lo == 0 and hi == 0:
                lo, hi = np.float32(-1), np.float32(1)
            s0 = np.float32((hi - lo) / np.float32(maxq))
            s = np.float32(s0 * np.float32(alpha))
            for c in range(g0, min(g0 + group, n)):
                codes[r, c] = int(np.rint(np.float32(W[r, c]) / s))
    return codes


@pytest.mark.parametrize("alpha", [0.4, 1.0, 3.0])
def test_identity_factor_is_unclipped_rtn(alpha):
    rng = np.random.default_rng(1)
    W = _heavy(9, 64, rng)
    res = Hq.hptq_blocked(W, np.eye(64), 3, 16, 32, alpha)
    assert np.array_equal(res["codes"], _rtn_unclipped_by_loops(W, 3, 16, alpha))


def test_alpha_one_with_one_column_groups_is_gptq():
    """group = 1, α = 1: no weight leaves its own row's range, so GPTQ never
    clips and its q − z is the lattice coordinate k, error for error."""
    rng = np.random.default_rng(2)
    n = 40
    p = G.prepare(_spd(n, rng), 0.01, "act")
    Wp = _heavy(13, n, rng)[:, p["perm"]]
    a = Hq.hptq_blocked(Wp, p["U"], 3, 1, 8, 1.0)
    b = G.gptq_blocked(Wp, p["U"], 3, 1, 8)
    assert np.array_equal(a["codes"], b["codes"] - b["zero"].astype(np.int64))
    assert np.allclose(a["err"], b["err"], rtol=0, atol=1e-15)


def _half_step_holds(res, U, group):
    n = U.shape[0]
    s = res["scale"][:, np.arange(n) // group].astype(np.float64)
    return bool(np.all(np.abs(res["err"]) * np.diag(U)[None, :] <= s / 2.0 * (1 + 1e-12)))


@pytest.mark.parametrize("alpha", [0.5, 1.0, 2.5])
def test_satz5_half_step_for_every_alpha(alpha):
    rng = np.random.default_rng(3)
    n = 64
    p = G.prepare(_spd(n, rng), 0.01, "act")
    Wp = _heavy(25, n, rng)[:, p["perm"]]
    res = Hq.hptq_blocked(Wp, p["U"], 2, 16, 32, alpha)
    assert _half_step_holds(res, p["U"], 16)
    n_ = Wp.shape[1]
    g = np.arange(n_) // 16
    D = Wp - res["scale"][:, g].astype(np.float64) * res["codes"]
    lhs = np.einsum("ij,jk,ik->i", D, p["Hp"], D)
    assert np.allclose(lhs, np.sum(res["err"] ** 2, axis=1), rtol=1e-9)


def test_coarser_grids_code_in_fewer_bits_on_a_layer():
    rng = np.random.default_rng(4)
    n = 96
    p = G.prepare(_spd(n, rng), 0.01, "act")
    Wp = _heavy(40, n, rng)[:, p["perm"]]
    b = [Hq.coded_bits(Hq.hptq_blocked(Wp, p["U"], 4, 32, 32, a)) for a in (0.5, 1.0, 2.0, 4.0)]
    assert b[0] > b[1] > b[2] > b[3]


# ---------------------------------------------------------------- the search

def test_search_on_a_layer_meets_the_budget_with_the_finest_grid_found():
    rng = np.random.default_rng(5)
    n, m, T = 96, 40, 256
    X = rng.standard_normal((T, n)) * np.linspace(2.0, 0.3, n)
    H = G.hessian(X)
    W = _heavy(m, n, rng)
    out = Hq.hptq_layer(W, H, bits=4, group=32, block=64, budget=3.125, iters=12)
    b_max = Hq.max_bits(3.125, m, n)
    assert out["bits"] <= b_max
    rejected = [a for a, b in out["trace"] if b > b_max]
    assert rejected and max(rejected) < out["alpha"]
    assert out["alpha"] - max(rejected) <= (16.0 - 1.0 / 16) / 2 ** 12 * 1.0001
    # the codes decode back from their own stream
    ro, st = Hq.encode(out["codes"], out["lengths"])
    assert ro[-1] == out["bits"]
    assert np.array_equal(Hq.decode(st, ro, out["lengths"], m, n), out["codes"])


def test_search_stops_at_the_upper_end_when_it_is_over_budget():
    rng = np.random.default_rng(6)
    n = 64
    p = G.prepare(_spd(n, rng), 0.01, "act")
    Wp = _heavy(10, n, rng)[:, p["perm"]]
    alpha, res, trace = Hq.bisect_alpha(lambda a: Hq.hptq_blocked(Wp, p["U"], 4, 32, 32, a),
                                        0, 8, 0.5, 2.0)
    assert alpha == np.float32(2.0) and len(trace) == 1


def test_max_bits_is_the_floor():
    assert Hq.max_bits(3.125, 576, 576) == 1036800
    assert Hq.max_bits(3.125, 7, 3) == 65


def test_follow_accepts_its_own_codes_and_flags_a_planted_one():
    rng = np.random.default_rng(7)
    n = 64
    p = G.prepare(_spd(n, rng), 0.01, "act")
    Wp = _heavy(30, n, rng)[:, p["perm"]]
    ref = Hq.hptq_blocked(Wp, p["U"], 3, 32, 64, 1.5)
    ok = Hq.follow_hptq(Wp, p["U"], 3, 32, 64, 1.5, ref["codes"], ref["scale"])
    assert ok["n_diff"] == 0 and ok["n_bad"] == 0 and ok["max_scale_rel"] == 0.0
    frac = np.abs(ref["pre"] - np.floor(ref["pre"]) - 0.5)
    r, j = np.unravel_index(np.argmax(frac), frac.shape)
    bad = ref["codes"].copy()
    bad[r, j] += 1
    assert Hq.follow_hptq(Wp, p["U"], 3, 32, 64, 1.5, bad, ref["scale"])["n_bad"] >= 1


# ---------------------------------------------------------------- mutations

def _wrong_merge(hist):
    """Merges the two heaviest subtrees instead of the two lightest."""
    if len(hist) == 1:
        return {next(iter(hist)): 1}
    nodes = [(c, [s]) for s, c in hist.items()]
    depth = {s: 0 for s in hist}
    while len(nodes) > 1:
        nodes.sort(key=lambda t: -t[0])
        (c1, s1), (c2, s2) = nodes[0], nodes[1]
        for s in s1 + s2:
            depth[s] += 1
        nodes = nodes[2:] + [(c1 + c2, s1 + s2)]
    return depth


@pytest.mark.parametrize("kind", ["wrong_merge", "clipped", "zero_point_kept",
                                  "length_off_by_one"])
def test_pins_catch_planted_mistakes(kind, monkeypatch):
    failures = 0
    rng = np.random.default_rng(30)
    if kind in ("wrong_merge", "length_off_by_one"):
        if kind == "wrong_merge":
            monkeypatch.setattr(Hq, "huffman_lengths", _wrong_merge)
        else:
            orig = Hq.huffman_lengths
            monkeypatch.setattr(Hq, "huffman_lengths",
                                lambda h: {s: l + 1 for s, l in orig(h).items()})
        for seed in range(6):
            r2 = np.random.default_rng(seed)
            k = int(r2.integers(3, 7))
            counts = [int(c) for c in r2.integers(1, 60, size=k)]
            h = {i: c for i, c in enumerate(counts)}
            L = Hq.huffman_lengths(h)
            failures += Hq.cost(h, L) != _optimal_cost_by_search(counts)
    else:
        orig_k = Hq.lattice_column
        if kind == "clipped":               # the coordinate clamped to the nominal range
            monkeypatch.setattr(Hq, "lattice_column",
                                lambda cur, s: np.clip(orig_k(cur, s), -4, 3).astype(np.float32))
        else:                               # a zero point of 1 added to every code
            monkeypatch.setattr(Hq, "lattice_column",
                                lambda cur, s: (orig_k(cur, s) + 1).astype(np.float32))
        W = _heavy(9, 64, rng)
        res = Hq.hptq_blocked(W, np.eye(64), 3, 16, 32, 0.4)
        failures += not np.array_equal(res["codes"], _rtn_unclipped_by_loops(W, 3, 16, 0.4))
        n = 64
        p = G.prepare(_spd(n, rng), 0.01, "act")
        Wp = _heavy(25, n, rng)[:, p["perm"]]
        failures += not _half_step_holds(Hq.hptq_blocked(Wp, p["U"], 2, 16, 32, 0.5), p["U"], 16)
    assert failures >= 1, kind


def test_canonical_codes_golden(golden):
    """The canonical-code rule against the DEFLATE format's worked example."""
    for lens, codes in golden("canonical_code_deflate.txt"):
        lengths = {i: int(l) for i, l in enumerate(lens)}
        cb = Hq.canonical_codes(lengths)
        assert [format(cb[i][0], f"0{cb[i][1]}b") for i in range(len(lens))] == codes


@pytest.mark.parametrize("n,group,block,alpha", [(96, 32, 32, 1.0), (100, 32, 64, 0.6),
                                                 (64, 16, 64, 2.5)])
def test_blocked_equals_sequential(n, group, block, alpha):
    rng = np.random.default_rng(40)
    p = G.prepare(_spd(n, rng), 0.01, "act")
    Wp = _heavy(17, n, rng)[:, p["perm"]]
    a = Hq.hptq_sequential(Wp, p["U"], 3, group, alpha)
    b = Hq.hptq_blocked(Wp, p["U"], 3, group, block, alpha)
    assert np.array_equal(a["codes"], b["codes"]) and np.array_equal(a["scale"], b["scale"])
    assert np.allclose(a["err"], b["err"], rtol=0, atol=1e-12)


def test_hptq_is_ssqr_without_outliers():
    """One unbounded grid and the outlier-keeping grid coincide where nothing
    overflows: with one-column groups at α = 1 no weight leaves its range, and
    SSQR's code minus its zero point is HPTQ's lattice coordinate, error for
    error (the two oracles are written separately)."""
    from oracle import ssqr as Sq
    rng = np.random.default_rng(42)
    n = 48
    p = G.prepare(_spd(n, rng), 0.01, "act")
    Wp = _heavy(11, n, rng)[:, p["perm"]]
    a = Sq.ssqr_blocked(Wp, p["U"], 3, 1, 16, 1.0)
    b = Hq.hptq_blocked(Wp, p["U"], 3, 1, 16, 1.0)
    assert Sq.count(a) == 0
    assert np.array_equal(a["codes"] - a["zero"].astype(np.int64), b["codes"])
    assert np.allclose(a["err"], b["err"], rtol=0, atol=1e-15)


@pytest.mark.parametrize("alpha", [0.5, 1.0, 2.0])
def test_back_to_front_is_babai_without_clipping(alpha):
    """Satz 4 for the unbounded grid: with one group (its step taken at the
    first column, before any update, so from the original weights), HPTQ
    back to front is Babai's nearest plane on F·diag(s) with no clamp and no
    zero point (the separately written lattice oracle), identical integers."""
    from oracle import lattice as L
    rng = np.random.default_rng(50)
    for trial in range(40):
        n = int(rng.integers(2, 9))
        H = _spd(n, rng)
        w = rng.standard_normal(n) * 0.02
        p = G.prepare(H, 0.01, "reverse")
        r = Hq.hptq_blocked(w[None, p["perm"]], p["U"], 3, n, n, alpha)
        s = np.full(n, float(r["scale"][0, 0]))
        Hd, _, _ = G.damp_and_fix(H, 0.01)
        F = np.linalg.cholesky(Hd).T
        q_b = L.babai(F, F @ w, s, np.zeros(n), 3, clip=False)
        q_g = r["codes"][0][G.inverse_permutation(p["perm"])]
        assert np.array_equal(q_b, q_g), (trial, q_b, q_g)
