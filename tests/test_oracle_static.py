"""Pins of the static-group GPTQ oracle.

Static groups fix every group's scale and zero from the original weights of
`group` consecutive original columns before the sweep (the common GPTQ option
beside act-order; the pages define only the groups met in processing order).
Pinned against an independently written round-to-nearest, the pinned GPTQ
oracle's fixed-parameter mode, Babai's nearest-plane algorithm with per-column
scales (the Babai page, §2.2 Satz 4) and the loss identity; the last test
plants mistakes and checks that they are caught.
"""
import numpy as np
import pytest

from oracle import gptq as G
from oracle import lattice as L
from oracle import static as S


def _spd(n, rng):
    A = rng.standard_normal((n + 3, n))
    return A.T @ A + 0.05 * np.eye(n)


@pytest.mark.parametrize("bits,group", [(2, 16), (3, 32), (4, 64)])
def test_identity_hessian_is_rtn_in_any_order(bits, group):
    """H = I: no error feedback, so static-group GPTQ in act-order is the
    round-to-nearest of the original groups, codes and parameters bit for bit."""
    rng = np.random.default_rng(1)
    n = 200
    W = rng.standard_normal((30, n)) * 0.02
    H = np.diag(rng.uniform(0.5, 2.0, n))                 # act-order permutes the columns
    out = S.gptq_layer_static(W, H, bits, group, 64, 0.01, "act")
    assert not np.array_equal(out["perm"], np.arange(n))
    codes, scale, zero, _ = L.rtn(W, bits, group)
    assert np.array_equal(out["codes"], codes)
    assert np.array_equal(out["scale"], scale) and np.array_equal(out["zero"], zero)


def test_natural_order_equals_the_fixed_parameter_mode():
    rng = np.random.default_rng(2)
    n, group = 96, 32
    p = G.prepare(_spd(n, rng), 0.01, "natural")
    W = rng.standard_normal((17, n)) * 0.02
    scale, zero = S.static_params(W, 3, group)
    a = S.gptq_static_blocked(W, p["U"], 3, np.arange(n) // group, scale, zero, block=64)
    b = G.gptq_sequential(W, p["U"], 3, group, fixed=(scale, zero))
    assert np.array_equal(a["codes"], b["codes"])
    assert np.allclose(a["err"], b["err"], rtol=0, atol=1e-12)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_back_to_front_is_babai_with_per_column_scales(bits):
    """Satz 4 with static groups: GPTQ back to front on chol(H_d) is Babai's
    nearest plane on the basis F·diag(s), s and z per column from the column's
    original group; identical codes, n ≤ 8, two groups."""
    rng = np.random.default_rng(20 + bits)
    for trial in range(40):
        n = int(rng.integers(3, 9))
        H = _spd(n, rng)
        w = rng.standard_normal(n) * 0.02
        group = -(-n // 2)
        scale, zero = S.static_params(w[None, :], bits, group)
        s = scale[0, np.arange(n) // group].astype(np.float64)
        z = zero[0, np.arange(n) // group].astype(np.float64)
        Hd, _, _ = G.damp_and_fix(H, 0.01)
        F = np.linalg.cholesky(Hd).T
        q_b = L.babai(F, F @ w, s, z, bits)
        p = G.prepare(H, 0.01, "reverse")
        r = S.gptq_static_blocked(w[None, p["perm"]], p["U"], bits, p["perm"] // group, scale,
                                  zero, block=n)
        q_g = r["codes"][0][G.inverse_permutation(p["perm"])]
        assert np.array_equal(q_b, q_g), (trial, q_b, q_g)


def test_loss_identity_in_act_order():
    rng = np.random.default_rng(3)
    n = 80
    p = G.prepare(_spd(n, rng), 0.01, "act")
    W = rng.standard_normal((12, n)) * 0.02
    scale, zero = S.static_params(W, 3, 32)
    cg = p["perm"] // 32
    r = S.gptq_static_blocked(W[:, p["perm"]], p["U"], 3, cg, scale, zero, block=32)
    D = W[:, p["perm"]] - G.dequantize(r["codes"], scale[:, cg], zero[:, cg])
    lhs = np.einsum("ij,jk,ik->i", D, p["Hp"], D)
    assert np.allclose(lhs, np.sum(r["err"] ** 2, axis=1), rtol=1e-9)


def test_follow_accepts_its_own_codes_and_flags_a_planted_one():
    rng = np.random.default_rng(4)
    n = 64
    p = G.prepare(_spd(n, rng), 0.01, "act")
    W = rng.standard_normal((20, n)) * 0.02
    scale, zero = S.static_params(W, 4, 32)
    cg = p["perm"] // 32
    Wp = W[:, p["perm"]]
    ref = S.gptq_static_blocked(Wp, p["U"], 4, cg, scale, zero, block=32)
    ok = S.follow_static(Wp, p["U"], 4, cg, scale, zero, 32, ref["codes"])
    assert ok["n_diff"] == 0 and np.allclose(ok["err"], ref["err"], atol=1e-15)
    frac = np.abs(ref["pre"] - np.floor(ref["pre"]) - 0.5)
    r, j = np.unravel_index(np.argmax(frac), frac.shape)
    bad = ref["codes"].copy()
    bad[r, j] = bad[r, j] + 1 if bad[r, j] < 15 else bad[r, j] - 1
    assert S.follow_static(Wp, p["U"], 4, cg, scale, zero, 32, bad)["n_bad"] >= 1


@pytest.mark.parametrize("kind", ["processing_groups", "current_values"])
def test_pins_catch_planted_mistakes(kind, monkeypatch):
    """Two plausible mistakes: grouping by processing position instead of the
    original column, and taking the parameters from the current values."""
    orig = S.gptq_static_blocked

    def mutant(Wp, U, bits, col_group, scale, zero, block=128):
        n = np.asarray(Wp).shape[1]
        group = max(1, n // max(1, int(np.max(col_group)) + 1))
        if kind == "processing_groups":
            col_group = np.arange(n) // group
            return orig(Wp, U, bits, col_group, scale, zero, block)
        return G.gptq_blocked(Wp, U, bits, group, block if block % group == 0 else group)
    monkeypatch.setattr(S, "gptq_static_blocked", mutant)
    failures = 0
    rng = np.random.default_rng(5)
    n = 200
    W = rng.standard_normal((30, n)) * 0.02
    H = np.diag(rng.uniform(0.5, 2.0, n))
    out = S.gptq_layer_static(W, H, 3, 40, 40, 0.01, "act")
    failures += not np.array_equal(out["codes"], L.rtn(W, 3, 40)[0])
    for trial in range(20):
        n2 = 6
        H2 = _spd(n2, rng)
        w = rng.standard_normal(n2) * 0.02
        scale, zero = S.static_params(w[None, :], 3, 3)
        s = scale[0, np.arange(n2) // 3].astype(np.float64)
        z = zero[0, np.arange(n2) // 3].astype(np.float64)
        Hd, _, _ = G.damp_and_fix(H2, 0.01)
        F = np.linalg.cholesky(Hd).T
        p = G.prepare(H2, 0.01, "reverse")
        r = S.gptq_static_blocked(w[None, p["perm"]], p["U"], 3, p["perm"] // 3, scale, zero, 6)
        q_g = r["codes"][0][G.inverse_permutation(p["perm"])]
        failures += not np.array_equal(L.babai(F, F @ w, s, z, 3), q_g)
    assert failures >= 1, kind


@pytest.mark.parametrize("n,group,block", [(96, 32, 32), (100, 40, 64), (130, 17, 96)])
def test_blocked_equals_sequential_in_act_order(n, group, block):
    """Any block width with any group width: the lazy batch changes only the
    order of the float64 additions."""
    rng = np.random.default_rng(41)
    p = G.prepare(_spd(n, rng), 0.01, "act")
    W = rng.standard_normal((15, n)) * 0.02
    scale, zero = S.static_params(W, 3, group)
    cg = p["perm"] // group
    a = S.gptq_static_sequential(W[:, p["perm"]], p["U"], 3, cg, scale, zero)
    b = S.gptq_static_blocked(W[:, p["perm"]], p["U"], 3, cg, scale, zero, block)
    assert np.array_equal(a["codes"], b["codes"])
    assert np.allclose(a["err"], b["err"], rtol=0, atol=1e-12)


def test_requantizing_the_result_is_a_no_op():
    """Composition (the Babai page §2.2 reading of GPTQ as a lattice
    projection): the dequantized weights lie on the fixed grid, so a second
    static-group sweep over them, with the same parameters and order, returns
    the same codes and no error at all."""
    rng = np.random.default_rng(6)
    n = 120
    p = G.prepare(_spd(n, rng), 0.01, "act")
    W = rng.standard_normal((14, n)) * 0.02
    scale, zero = S.static_params(W, 3, 40)
    cg = p["perm"] // 40
    r1 = S.gptq_static_blocked(W[:, p["perm"]], p["U"], 3, cg, scale, zero, 64)
    Qp = G.dequantize(r1["codes"], scale[:, cg], zero[:, cg])
    r2 = S.gptq_static_blocked(Qp, p["U"], 3, cg, scale, zero, 64)
    assert np.array_equal(r2["codes"], r1["codes"])
    assert np.abs(r2["err"]).max() == 0.0
