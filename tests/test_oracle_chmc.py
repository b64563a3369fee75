"""Pins of the CHMC frontend oracle against what the page and mathematics fix.

Page: "Warum Geometrie Gewichte nicht komprimiert", section "Methodik. Was ist
CHMC", Schritte 1–3.  Each pin checks the oracle against something other than
its own formula: a brute-force search, explicit loops, a matrix built with a
known answer, or an equivalent special case of the GPTQ oracle.
"""
import numpy as np
import pytest

from oracle import chmc as C
from oracle import gptq as G


# ------------------------------------------------------------ Schritt 3

@pytest.mark.parametrize("o,i,bits,gs,tgt", [
    (576, 576, 4, 128, 4.2875), (1536, 576, 4, 128, 4.2875), (576, 1536, 4, 128, 4.2875),
    (192, 576, 4, 128, 4.2875), (896, 4864, 4, 128, 4.2875), (64, 64, 3, 32, 3.6),
    (128, 128, 4, 128, 4.0)])
def test_rank_rule_is_the_largest_rank_within_budget(o, i, bits, gs, tgt):
    """Schritt 3: r is the largest rank whose CHMC bits per weight stay within
    the target (searched by brute force over the page's BPW formula)."""
    best = 0
    for r in range(0, min(o, i) + 1):
        bits_total = 16 * r * (o + i) + bits * o * i + 16 * (-(-o // gs)) * i
        if bits_total <= tgt * o * i:
            best = r
    assert C.chmc_rank(o, i, bits, gs, tgt) == best


def test_bpw_gptq_of_4bit_group128():
    """GPTQ's formula at 4 bits, group 128, gs | i: 4 + 16/128 = 4.125 (the
    page's 4.2875 does not follow from it; a reading)."""
    assert C.bpw_gptq(576, 1536, 4, 128) == pytest.approx(4.125, abs=1e-15)
    assert C.bpw_chmc(576, 1536, 0, 4, 128) == pytest.approx(4 + 16 * 5 / 576, abs=1e-15)


# ------------------------------------------------------------ Schritt 1

def test_activation_energy_by_loops():
    rng = np.random.default_rng(1)
    X = rng.standard_normal((5, 3))
    c0 = []
    for j in range(3):
        acc = 0.0
        for t in range(5):
            acc += X[t, j] * X[t, j]
        c0.append(acc / 5)
    mean = sum(c0) / 3
    want = [v + 0.05 * mean for v in c0]
    assert np.allclose(C.activation_energy(X, 0.05), want, rtol=1e-14, atol=0)


def test_activation_energy_from_hessian_equals_from_tokens():
    rng = np.random.default_rng(2)
    X = rng.standard_normal((37, 9))
    H = G.hessian(X)                      # 2·XᵀX
    assert np.allclose(C.activation_energy_from_hessian(H, 37, 0.05),
                       C.activation_energy(X, 0.05), rtol=1e-13, atol=0)


def test_lowrank_recovers_an_exactly_low_rank_matrix():
    """If rank(W) ≤ r the subspace iteration finds its whole range: W_lr = W."""
    rng = np.random.default_rng(3)
    o, i, r0, r = 40, 30, 3, 4
    W = rng.standard_normal((o, r0)) @ rng.standard_normal((r0, i))
    c = rng.uniform(0.1, 3.0, i)
    out = C.weighted_lowrank(W, c, rng.standard_normal((i, r)), niter=5)
    assert np.abs(out["Wlr"] - W).max() <= 1e-10 * np.abs(W).max()


def test_lowrank_is_the_truncated_weighted_svd_when_the_spectrum_has_a_gap():
    """Eckart–Young in the weighted norm: with σ_r/σ_{r+1} = 100 and five power
    iterations, W_lr equals the truncated SVD of W·diag(√c), scaled back."""
    rng = np.random.default_rng(4)
    o, i, r = 50, 36, 3
    Uo, _ = np.linalg.qr(rng.standard_normal((o, i)))
    Vo, _ = np.linalg.qr(rng.standard_normal((i, i)))
    sig = np.concatenate([[9.0, 5.0, 3.0], 0.03 * rng.uniform(0.2, 1.0, i - 3)])
    Wt = (Uo * sig) @ Vo.T
    c = rng.uniform(0.2, 2.0, i)
    W = Wt / np.sqrt(c)[None, :]
    best = (Uo[:, :r] * sig[:r]) @ Vo[:, :r].T / np.sqrt(c)[None, :]
    out = C.weighted_lowrank(W, c, rng.standard_normal((i, r)), niter=5)
    assert np.abs(out["Wlr"] - best).max() <= 1e-9 * np.abs(best).max()


def test_lowrank_factors_are_an_svd_of_the_approximation():
    rng = np.random.default_rng(5)
    o, i, r = 30, 20, 4
    W = rng.standard_normal((o, i))
    c = rng.uniform(0.5, 1.5, i)
    out = C.weighted_lowrank(W, c, rng.standard_normal((i, r)), niter=2)
    U, S, Vt = out["U"], out["S"], out["Vt"]
    assert np.allclose(U.T @ U, np.eye(r), atol=1e-12)
    assert np.allclose(Vt @ Vt.T, np.eye(r), atol=1e-12)
    assert np.all(np.diff(S) <= 0) and np.all(S >= 0)
    assert np.allclose((U * S) @ Vt / np.sqrt(c)[None, :], out["Wlr"], atol=1e-12)
    # the projector form: W_lr = Q·Qᵀ·W
    Q = out["Q"]
    assert np.allclose(Q @ (Q.T @ W), out["Wlr"], atol=1e-12)


# ------------------------------------------------------------ Schritt 2

def _rtn_rowgroups(W, bits, gs):
    """Round-to-nearest with row groups, by explicit loops (float32 decisions)."""
    m, n = W.shape
    maxq = 2 ** bits - 1
    codes = np.zeros((m, n), np.int64)
    for j in range(n):
        for g0 in range(0, m, gs):
            vals = [np.float32(W[r, j]) for r in range(g0, min(g0 + gs, m))]
            lo = min(min(vals), np.float32(0))
            hi = max(max(vals), np.float32(0))
            if lo == 0 and hi == 0:
                lo, hi = np.float32(-1), np.float32(1)
            s = np.float32((hi - lo) / np.float32(maxq))
            z = np.float32(np.rint(np.float32(-lo) / s))
            for r in range(g0, min(g0 + gs, m)):
                q = np.rint(np.float32(W[r, j]) / s) + z
                codes[r, j] = int(min(max(q, 0), maxq))
    return codes


def test_rowgroups_with_identity_factor_is_round_to_nearest():
    rng = np.random.default_rng(6)
    W = rng.standard_normal((21, 7)) * 0.05
    out = C.gptq_rowgroups_sequential(W, np.eye(7), 4, gs=8)
    assert np.array_equal(out["codes"], _rtn_rowgroups(W, 4, 8))


def test_rowgroups_of_one_row_equal_gptq_with_groups_of_one_column():
    """gs = 1: every (row, column) has its own min-max, exactly as the GPTQ
    oracle's input-channel groups of one column."""
    rng = np.random.default_rng(7)
    X = rng.standard_normal((64, 12))
    W = rng.standard_normal((9, 12)) * 0.03
    prep = G.prepare(G.hessian(X), 0.01, "act")
    Wp = W[:, prep["perm"]]
    a = C.gptq_rowgroups_sequential(Wp, prep["U"], 3, gs=1)
    b = G.gptq_sequential(Wp, prep["U"], 3, group=1)
    assert np.array_equal(a["codes"], b["codes"])
    assert np.array_equal(a["scale"], b["scale"])
    assert np.allclose(a["err"], b["err"], rtol=0, atol=1e-15)


def test_rowgroups_blocked_equals_sequential():
    rng = np.random.default_rng(8)
    X = rng.standard_normal((128, 40))
    W = rng.standard_normal((33, 40)) * 0.03
    prep = G.prepare(G.hessian(X), 0.01, "act")
    Wp = W[:, prep["perm"]]
    a = C.gptq_rowgroups_sequential(Wp, prep["U"], 4, gs=16)
    b = C.gptq_rowgroups_blocked(Wp, prep["U"], 4, gs=16, block=8)
    assert np.array_equal(a["codes"], b["codes"])
    assert np.allclose(a["err"], b["err"], rtol=0, atol=1e-10)


@pytest.mark.parametrize("seed", range(4))
def test_rowgroups_loss_below_round_to_nearest(seed):
    """On seeded layers the compensated residual quantization never loses to
    round-to-nearest with the same row-group quantizer (not a theorem for
    per-column scales; the measured ratio is ≈ 0.82)."""
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((256, 48)) * np.linspace(2, 0.2, 48) + 0.3 * rng.standard_normal((256, 1))
    W = rng.standard_normal((64, 48)) * 0.02
    H = G.hessian(X)
    prep = G.prepare(H, 0.01, "act")
    inv = G.inverse_permutation(prep["perm"])
    Wp = W[:, prep["perm"]]

    def deq(r):
        return G.dequantize(r["codes"], C._rows_matrix(r["scale"], 64, 16),
                            C._rows_matrix(r["zero"], 64, 16))[:, inv]

    l_gptq = G.layer_loss(W, deq(C.gptq_rowgroups_sequential(Wp, prep["U"], 4, 16)), H)
    l_rtn = G.layer_loss(W, deq(C.gptq_rowgroups_sequential(Wp, np.eye(48), 4, 16)), H)
    assert l_gptq < l_rtn


def test_follow_rowgroups_accepts_its_own_decisions_and_flags_a_planted_one():
    rng = np.random.default_rng(9)
    X = rng.standard_normal((128, 24))
    W = rng.standard_normal((40, 24)) * 0.03
    prep = G.prepare(G.hessian(X), 0.01, "act")
    Wp = W[:, prep["perm"]]
    ref = C.gptq_rowgroups_blocked(Wp, prep["U"], 4, gs=16, block=8)
    ok = C.follow_rowgroups(Wp, prep["U"], 4, 16, 8, ref["codes"], ref["scale"], ref["zero"])
    assert ok["n_diff"] == 0 and ok["n_bad"] == 0 and ok["max_scale_rel"] == 0.0
    # plant a wrong code far from any rounding boundary (in the oracle's output)
    frac = np.abs(ref["pre"] - np.floor(ref["pre"]) - 0.5)
    r, j = np.unravel_index(np.argmax(frac), frac.shape)
    bad = ref["codes"].copy()
    bad[r, j] = bad[r, j] + 1 if bad[r, j] < 15 else bad[r, j] - 1
    out = C.follow_rowgroups(Wp, prep["U"], 4, 16, 8, bad, ref["scale"], ref["zero"])
    assert out["n_bad"] >= 1


def test_chmc_layer_reconstructs_from_its_parts():
    rng = np.random.default_rng(10)
    o, i, T = 48, 32, 128
    X = rng.standard_normal((T, i)) * np.linspace(1.5, 0.3, i)
    W = rng.standard_normal((o, i)) * 0.02
    H = G.hessian(X)
    r = 3
    out = C.chmc_layer(W, H, T, rng.standard_normal((i, r)), rank=r, gs=16, block=16)
    assert np.allclose(out["Wcomp"], out["Wlr"] + out["Rq"], atol=1e-15)
    assert np.allclose(out["R"], W - out["Wlr"], atol=1e-15)
    assert out["scale"].shape == (3, i) and out["codes"].shape == (o, i)
    assert 0 <= out["codes"].min() and out["codes"].max() <= 15
    assert out["bpw"] == pytest.approx(C.bpw_chmc(o, i, r, 4, 16))


def test_follow_rowgroups_accepts_a_zero_point_flipped_at_a_tie():
    """A row group whose −xmin/s sits on a half-integer may take either zero
    point; the other side's codes of that column then sit one step over for
    every row of the group.  That is one allowed zero flip, no code
    difference."""
    W = np.array([[-1.0, 0.2], [5.0, -0.3], [0.3, 0.1], [2.0, 0.4]])
    s, z = C.rowgroup_params(W[:, 0], 4, 4)
    assert abs(1.0 / float(s[0]) - 2.5) < 1e-6          # −xmin/s = 2.5 up to rounding
    z2 = np.float32(z[0] + (1 if z[0] == 2 else -1))
    q0 = np.clip(np.rint(np.float32(W[:, 0]) / s[0]) + z2, 0, 15)
    s1, z1 = C.rowgroup_params(W[:, 1], 4, 4)
    q1 = np.clip(np.rint(np.float32(W[:, 1]) / s1[0]) + z1[0], 0, 15)
    codes = np.stack([q0, q1], axis=1).astype(np.int64)
    scale = np.array([[s[0], s1[0]]], np.float32)
    zero = np.array([[z2, z1[0]]], np.float32)
    f = C.follow_rowgroups(W, np.eye(2), 4, 4, 2, codes, scale, zero)
    assert f["z_diff"] == 1 and f["z_bad"] == 0
    assert f["n_bad"] == 0
