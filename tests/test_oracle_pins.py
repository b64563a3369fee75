"""Pins of the float64 oracle against what the pages and the mathematics fix.

None of these tests re-types the oracle's formulas: each compares it with a
hand-computed fixture, a closed form, an independent algorithm (Babai's
nearest plane, brute-force CVP, a library LDL factorisation) or an invariant.
The last test plants plausible mistakes in copies of the sweep and checks that
the pins catch each of them.
"""
import numpy as np
import pytest
from scipy.linalg import ldl

from oracle import gptq as og
from oracle import lattice as ol
from workloads import problems_for


def _spd(n, rng, cond_scale=1.0):
    A = rng.standard_normal((n + 3, n))
    return A.T @ A + cond_scale * 0.05 * np.eye(n)


# ---------------------------------------------------------------- fixtures

def test_quantizer_golden(golden):
    for bits, vals, sz, codes in golden("quantizer_minmax.txt"):
        bits = int(bits[0])
        v = np.array([float(x) for x in vals])[None, :]
        s, z = og.group_params(v, bits)
        assert s[0] == np.float32(float(sz[0])), (vals, s)
        assert z[0] == float(sz[1])
        q = og.quantize_column(v[0], s[0], z[0], bits)
        assert [int(x) for x in q] == [int(c) for c in codes]
        # the independent RTN quantizer agrees with the fixture too
        s2, z2 = ol.minmax_params_row(v[0], bits)
        assert s2 == s[0] and z2 == z[0]


def test_two_column_closed_form(golden):
    H = np.array([[4.0, 2.0], [2.0, 3.0]])
    U = og.inverse_cholesky_upper(H)
    assert np.allclose(U, [[np.sqrt(3 / 8), -1 / (4 * np.sqrt(3 / 8))],
                           [0.0, 1 / np.sqrt(3)]], atol=1e-15)
    for w, q, e, loss in golden("two_column.txt"):
        w = np.array([[float(x) for x in w]])
        fixed = (np.full((1, 1), 0.25, np.float32), np.full((1, 1), 8, np.float32))
        r = og.gptq_sequential(w, U, 4, 2, fixed=fixed)
        assert [int(x) for x in r["codes"][0]] == [int(x) for x in q]
        assert np.allclose(r["err"][0], [float(x) for x in e], rtol=1e-12)
        qhat = og.dequantize(r["codes"], 0.25, 8)
        assert np.isclose(og.layer_loss(w, qhat, H), float(loss[0]), rtol=1e-12)


def test_pack_golden(golden):
    for bits, codes, words in golden("pack_lsb_first.txt"):
        bits = int(bits[0])
        c = np.array([[int(x) for x in codes]])
        got = og.pack_rows(c, bits)[0]
        assert [f"{int(x):08X}" for x in got] == words


def test_pack_matches_bigint_stream():
    rng = np.random.default_rng(1)
    for bits in (2, 3, 4, 8):
        codes = rng.integers(0, 2 ** bits, size=(3, 77))
        got = og.pack_rows(codes, bits)
        for r in range(3):
            stream = 0
            for c in reversed(range(77)):
                stream = (stream << bits) | int(codes[r, c])
            words = [(stream >> (32 * k)) & 0xFFFFFFFF for k in range(got.shape[1])]
            assert words == [int(x) for x in got[r]]


# ---------------------------------------------------------------- prepare

def test_prepare_factor_definition():
    rng = np.random.default_rng(2)
    H = _spd(40, rng)
    for order in ("natural", "act", "reverse"):
        p = og.prepare(H, 0.01, order)
        U, Hp = p["U"], p["Hp"]
        assert np.allclose(np.tril(U, -1), 0)
        assert np.all(np.diag(U) > 0)
        assert np.allclose(U.T @ U @ Hp, np.eye(40), atol=1e-9)
        d = np.mean(np.diag(H))
        assert np.allclose(np.diag(p["Hd"]), np.diag(H) + 0.01 * d)
    # act-order: descending diagonal, equal entries keep ascending index
    H2 = np.diag([1.0, 3.0, 2.0, 3.0, 0.5])
    assert list(og.prepare(H2, 0.01, "act")["perm"]) == [1, 3, 2, 0, 4]


def test_dead_columns():
    rng = np.random.default_rng(3)
    X = rng.standard_normal((50, 12))
    X[:, 4] = 0.0
    H = og.hessian(X)
    W = rng.standard_normal((5, 12)) * 0.02
    r = og.gptq_layer(W, H, 4, 4, 4, 0.01, "act")
    assert r["dead"][4] and r["dead"].sum() == 1
    # dead column: its weight is zeroed, so its code is the zero point
    assert np.all(r["Q"][:, 4] == 0.0)
    # the damping mean is taken before the fix (the dead entry counts as 0)
    Hd, dead, d = og.damp_and_fix(H, 0.01)
    assert d == np.mean(np.diag(H)) and Hd[4, 4] == 1.0 + 0.01 * d


def test_ldl_pivots_are_inverse_squared_diagonal():
    """Satz 5's D: 1/U_jj² equals the LDL pivots of the permuted Hessian.

    GPTQ front to back pivots from the last column (H_p = R̃R̃ᵀ with R̃ = U⁻¹
    upper), i.e. an LDLᵀ of the reversed matrix.  scipy's LDL is the check.
    """
    rng = np.random.default_rng(4)
    H = _spd(30, rng)
    for order in ("natural", "act"):
        p = og.prepare(H, 0.01, order)
        J = p["Hp"][::-1, ::-1]
        _, D, _ = ldl(J, lower=True)
        assert np.allclose(np.diag(D)[::-1], 1.0 / np.diag(p["U"]) ** 2, rtol=1e-10)


# ---------------------------------------------------------------- sweep forms

@pytest.mark.parametrize("n,group,block", [(64, 16, 32), (200, 32, 64), (512, 128, 128)])
def test_blocked_equals_sequential(n, group, block):
    rng = np.random.default_rng(n)
    H = _spd(n, rng)
    U = og.prepare(H, 0.01)["U"]
    W = rng.standard_normal((20, n)) * 0.02
    a = og.gptq_sequential(W, U, 4, group)
    b = og.gptq_blocked(W, U, 4, group, block)
    assert np.array_equal(a["codes"], b["codes"])
    assert np.max(np.abs(a["pre"] - b["pre"])) <= 1e-10
    assert np.array_equal(a["scale"], b["scale"])


def test_downdated_inverse_equals_sequential():
    rng = np.random.default_rng(5)
    for n, group in ((8, 8), (33, 16), (64, 32)):
        H = _spd(n, rng)
        p = og.prepare(H, 0.01)
        W = rng.standard_normal((10, n)) * 0.02
        a = og.gptq_sequential(W, p["U"], 3, group)
        b = og.gptq_downdated_inverse(W, p["Hp"], 3, group)
        assert np.array_equal(a["codes"], b["codes"])
        assert np.allclose(a["pre"], b["pre"], atol=1e-10)
        assert np.allclose(a["err"], b["err"], atol=1e-10)


def test_identity_hessian_is_round_to_nearest():
    """H = I: no error feedback, so GPTQ is RTN bit for bit."""
    rng = np.random.default_rng(6)
    n = 300
    W = rng.standard_normal((40, n)) * 0.02
    for bits in (2, 3, 4, 8):
        for group in (32, 64, 128):
            r = og.gptq_layer(W, np.eye(n), bits, group, 128, 0.01, "natural")
            c, s, z, Q = ol.rtn(W, bits, group)
            assert np.array_equal(r["codes"], c)
            assert np.array_equal(r["scale"], s)
            assert np.array_equal(r["zero"], z)


def test_loss_identity():
    """(w − q̂)ᵀH_d(w − q̂) = Σ_j e_j² per row, for any rounding decisions."""
    rng = np.random.default_rng(7)
    n = 96
    H = _spd(n, rng)
    W = rng.standard_normal((12, n)) * 0.02
    for order in ("natural", "act"):
        p = og.prepare(H, 0.01, order)
        Wp = W[:, p["perm"]]
        r = og.gptq_blocked(Wp, p["U"], 3, 32, 64)
        g = np.arange(n) // 32
        D = Wp - og.dequantize(r["codes"], r["scale"][:, g], r["zero"][:, g])
        lhs = np.einsum("ij,jk,ik->i", D, p["Hp"], D)
        assert np.allclose(lhs, np.sum(r["err"] ** 2, axis=1), rtol=1e-9)


def test_satz5_bound_without_clipping():
    """[P2] §2.3 Satz 5: unclipped error ≤ ¼·Σ s_j²·D_jj per row."""
    rng = np.random.default_rng(8)
    n = 64
    H = _spd(n, rng)
    p = og.prepare(H, 0.01, "act")
    W = rng.standard_normal((30, n)) * 0.02
    Wp = W[:, p["perm"]]
    r = og.gptq_blocked(Wp, p["U"], 2, 16, 32, clip=False)
    s = r["scale"][:, np.arange(n) // 16].astype(np.float64)
    bound = 0.25 * np.sum(s ** 2 / np.diag(p["U"])[None, :] ** 2, axis=1)
    loss = np.sum(r["err"] ** 2, axis=1)
    assert np.all(loss <= bound * (1 + 1e-12))


# ---------------------------------------------------------------- lattice view

def _single_group_params(w, bits):
    s, z = ol.minmax_params_row(w, bits)
    return np.full(w.size, s), np.full(w.size, z)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_back_to_front_is_babai(bits):
    """[P2] §2.2 Satz 4: GPTQ back to front ≡ Babai on chol(H_d); natural order
    ≡ Babai on the reversed basis.  Identical codes, many seeds, n ≤ 8."""
    rng = np.random.default_rng(10 + bits)
    for trial in range(60):
        n = int(rng.integers(2, 9))
        H = _spd(n, rng, cond_scale=rng.uniform(0.1, 3))
        w = rng.standard_normal(n) * 0.02
        s, z = _single_group_params(w, bits)
        Hd, _, _ = og.damp_and_fix(H, 0.01)
        F = np.linalg.cholesky(Hd).T                      # FᵀF = H_d
        q_b = ol.babai(F, F @ w, s, z, bits)
        p = og.prepare(H, 0.01, "reverse")
        r = og.gptq_sequential(w[None, p["perm"]], p["U"], bits, n)
        q_g = r["codes"][0][og.inverse_permutation(p["perm"])]
        assert np.array_equal(q_b, q_g), (trial, q_b, q_g)
        # natural order = Babai on the reversed lattice
        J = np.arange(n)[::-1]
        Fr = np.linalg.cholesky(Hd[np.ix_(J, J)]).T
        q_br = ol.babai(Fr, Fr @ w[J], s[J], z[J], bits)[np.argsort(J)]
        p2 = og.prepare(H, 0.01, "natural")
        r2 = og.gptq_sequential(w[None, :], p2["U"], bits, n)
        assert np.array_equal(q_br, r2["codes"][0])


def test_satz1_any_factor_of_the_hessian():
    """[P2] §2.1 Satz 1: Babai on X (stacked with √(λ)·I for the damping)
    gives the same codes as Babai on the square Cholesky factor."""
    rng = np.random.default_rng(20)
    for trial in range(30):
        n = int(rng.integers(2, 8))
        X = rng.standard_normal((40, n)) * rng.uniform(0.5, 2, n)
        H = og.hessian(X)
        Hd, _, mean_diag = og.damp_and_fix(H, 0.01)
        lam = 0.01 * mean_diag
        Xa = np.vstack([np.sqrt(2.0) * X, np.sqrt(lam) * np.eye(n)])
        w = rng.standard_normal(n) * 0.02
        s, z = _single_group_params(w, 3)
        F = np.linalg.cholesky(Hd).T
        assert np.array_equal(ol.babai(Xa, Xa @ w, s, z, 3),
                              ol.babai(F, F @ w, s, z, 3))


def test_bruteforce_cvp_bounds_gptq():
    """Exact CVP optimum ≤ GPTQ loss, and GPTQ back to front = Babai (n ≤ 4)."""
    rng = np.random.default_rng(21)
    for trial in range(25):
        n = int(rng.integers(2, 5))
        H = _spd(n, rng)
        w = rng.standard_normal(n) * 0.02
        s, z = _single_group_params(w, 2)
        Hd, _, _ = og.damp_and_fix(H, 0.01)
        _, best = ol.cvp_bruteforce(Hd, w, s, z, 2)
        p = og.prepare(H, 0.01, "reverse")
        r = og.gptq_sequential(w[None, p["perm"]], p["U"], 2, n)
        assert best <= np.sum(r["err"] ** 2) * (1 + 1e-12)
        q_g = r["codes"][0][og.inverse_permutation(p["perm"])]
        F = np.linalg.cholesky(Hd).T
        assert np.array_equal(q_g, ol.babai(F, F @ w, s, z, 2))


def test_composition_is_a_no_op():
    """[P2] §2.2: GPTQ on its own dequantized output, same scales, changes
    nothing: identical codes and all errors zero."""
    rng = np.random.default_rng(22)
    n = 160
    H = _spd(n, rng)
    p = og.prepare(H, 0.01, "act")
    W = rng.standard_normal((16, n)) * 0.02
    Wp = W[:, p["perm"]]
    r = og.gptq_blocked(Wp, p["U"], 4, 32, 64)
    g = np.arange(n) // 32
    Qp = og.dequantize(r["codes"], r["scale"][:, g], r["zero"][:, g])
    r2 = og.gptq_blocked(Qp, p["U"], 4, 32, 64, fixed=(r["scale"], r["zero"]))
    assert np.array_equal(r2["codes"], r["codes"])
    assert np.max(np.abs(r2["err"])) < 1e-12


def test_order_equivariance():
    rng = np.random.default_rng(23)
    n = 70
    H = _spd(n, rng)
    W = rng.standard_normal((9, n)) * 0.02
    pi = rng.permutation(n)
    a = og.gptq_layer(W, H, 4, 16, 32, 0.01, "custom", perm=pi)
    b = og.gptq_layer(W[:, pi], H[np.ix_(pi, pi)], 4, 16, 32, 0.01, "natural")
    assert np.array_equal(a["codes"][:, pi], b["codes"])
    assert np.array_equal(a["scale"], b["scale"])


def test_hessian_scale_invariance():
    """Codes do not depend on the Hessian's scale (2·XᵀX vs XᵀX/n readings)."""
    p = problems_for(0)[0]
    X = p.X.float().numpy()[:512]
    W = p.W.numpy()[:64]
    H = og.hessian(X)
    a = og.gptq_layer(W, H, 4, 128, 128, 0.01, "act")
    b = og.gptq_layer(W, 4.0 * H, 4, 128, 128, 0.01, "act")
    assert np.array_equal(a["codes"], b["codes"])
    assert np.array_equal(a["scale"], b["scale"])


def test_objective_is_layer_output_error():
    """[P2] §2.1: tr((W−Q)H(W−Q)ᵀ) with H = 2XᵀX is twice the squared L2
    error of the layer output X·(W−Q)ᵀ."""
    rng = np.random.default_rng(24)
    X = rng.standard_normal((100, 20))
    W = rng.standard_normal((6, 20))
    Q = np.round(W * 4) / 4
    direct = 2.0 * np.sum((X @ (W - Q).T) ** 2)
    assert np.isclose(og.layer_loss(W, Q, og.hessian(X)), direct, rtol=1e-12)


def test_hessian_blocks_tile_the_hessian():
    """Blocks of 2·XᵀX from column subsets are the matching entries of the
    whole product (the tile check of large Hessians relies on it)."""
    rng = np.random.default_rng(26)
    X = rng.standard_normal((50, 30))
    H = og.hessian(X)
    I, J = np.arange(3, 17), np.arange(20, 30)
    assert np.allclose(og.hessian_block(X[:, I], X[:, J]), H[np.ix_(I, J)], rtol=1e-13)
    assert np.allclose(og.hessian_block(X[:, J], X[:, I]), H[np.ix_(I, J)].T, rtol=1e-13)


def test_gptq_beats_rtn_on_cone_layer():
    """Layer loss of GPTQ never exceeds round-to-nearest on the cone workload."""
    p = problems_for(0)[0]
    X = p.X.float().numpy()
    W = p.W.numpy()[:128]
    H = og.hessian(X)
    r = og.gptq_layer(W, H, 4, 128, 128, 0.01, "natural")
    _, _, _, Q = ol.rtn(W, 4, 128)
    assert r["loss"] < og.layer_loss(W, Q, H)


def test_rtn_dequant_equals_element_loop():
    """The whole-array round-to-nearest used at layer sizes gives exactly the
    element loop's dequantized weights (ragged last group, an all-zero group,
    same-sign groups, every bit width)."""
    rng = np.random.default_rng(31)
    for m, n, g, b in [(5, 37, 16, 4), (7, 128, 128, 3), (6, 200, 64, 2), (4, 64, 32, 8)]:
        W = (rng.standard_normal((m, n)) * 0.02).astype(np.float32)
        W[1, :g] = 0.0
        W[2, :g] = np.abs(W[2, :g])
        W[3, :g] = -np.abs(W[3, :g])
        _, _, _, Q = ol.rtn(W, b, g)
        assert np.array_equal(ol.rtn_dequant(W, b, g), Q)


@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("order", ["natural", "act", "reverse"])
def test_gptq_never_worse_than_rtn_across_seeds(bits, order):
    """The layer loss tr((W−Q)H(W−Q)ᵀ) of GPTQ does not exceed round-to-nearest's
    on the same inputs, over seeds, shapes (ragged groups and blocks), cone and
    heavy-tailed activations.

    Not a theorem once codes are clipped (the Babai page's Satz 5 bounds the
    unclipped error only): at 2 bits on heavy-tailed Student-t activations run
    back to front, seed 1 of this set gives 1.12× the round-to-nearest loss.
    So 2 bits is checked on the cone activations the workloads use, 3 and 4
    bits on both kinds."""
    from workloads import cone_activations, gaussian_weights, student_t_activations
    cases = [(512, 320, 96, 128, "cone"), (384, 200, 48, 64, "t")]
    for seed in range(4):
        for T, n, m, group, kind in cases if bits > 2 else cases[:1]:
            if kind == "cone":
                X = cone_activations(T, n, 500 + seed)
            else:
                X = student_t_activations(T, n, 500 + seed)
            X = X.to(dtype=__import__("torch").bfloat16).float().numpy()
            W = gaussian_weights(m, n, 600 + seed).numpy()
            H = og.hessian(X)
            r = og.gptq_layer(W, H, bits, group, 128, 0.01, order)
            rtn_loss = og.layer_loss(W, ol.rtn_dequant(W, bits, group), H)
            assert r["loss"] <= rtn_loss, (seed, kind, r["loss"], rtn_loss)


@pytest.mark.parametrize("cid,bits,rows", [(0, 4, None), (1, 4, None), (2, 4, 128),
                                           (3, 4, 128), (3, 3, 128)])
def test_gptq_never_worse_than_rtn_on_workloads(cid, bits, rows):
    """The same on every problem of the workloads' layers (the single layer and
    the SmolLM layer in full; the first 128 rows of each Qwen2.5-0.5B and
    TinyLlama-1.1B problem, a layer of their own since rows are independent).
    The 8192² stress layer is checked on the GPU's result, in full."""
    for p in problems_for(cid, bits=bits):
        X = p.X.float().numpy()
        W = p.W.float().numpy() if rows is None else p.W[:rows].float().numpy()
        H = og.hessian(X)
        r = og.gptq_layer(W, H, bits, p.group, p.block, p.damp, p.order)
        rtn_loss = og.layer_loss(W, ol.rtn_dequant(W, bits, p.group), H)
        assert r["loss"] <= rtn_loss, (p.name, r["loss"], rtn_loss)


# ---------------------------------------------------------------- follow mode

def test_follow_mode_on_own_decisions():
    rng = np.random.default_rng(25)
    n = 200
    H = _spd(n, rng)
    p = og.prepare(H, 0.01, "act")
    W = rng.standard_normal((20, n)) * 0.02
    Wp = W[:, p["perm"]]
    r = og.gptq_blocked(Wp, p["U"], 4, 64, 128)
    f = og.follow(Wp, p["U"], 4, 64, 128, r["codes"], r["scale"], r["zero"])
    assert f["code_diff"] == 0 and f["zero_diff"] == 0 and f["max_scale_rel"] == 0
    assert np.allclose(f["loss_rows"], np.sum(r["err"] ** 2, axis=1))
    # a planted wrong code far from any boundary is reported as disallowed
    codes = r["codes"].copy()
    i = np.argmax(np.abs(r["pre"][:, 5] - np.floor(r["pre"][:, 5]) - 0.5) < 0.3)
    codes[i, 5] = (codes[i, 5] + 1) % 16
    f2 = og.follow(Wp, p["U"], 4, 64, 128, codes, r["scale"], r["zero"])
    assert f2["code_diff_disallowed"] >= 1


# ---------------------------------------------------------------- mutations

def _mutant_sweep(kind):
    """Copies of the sequential sweep with one plausible mistake each."""
    def sweep(Wp, U, bits, group, fixed=None):
        W = np.array(Wp, dtype=np.float64, copy=True)
        m, n = W.shape
        codes = np.zeros((m, n), np.int64)
        err = np.zeros((m, n))
        s = z = None
        for j in range(n):
            if j % group == 0:
                if fixed is None:
                    s, z = og.group_params(W[:, j:j + group], bits)
                else:
                    s, z = fixed[0][:, j // group], fixed[1][:, j // group]
            q = og.quantize_column(W[:, j], s, z, bits)
            e = (W[:, j] - og.dequantize(q, s, z)) / U[j, j]
            row = U[j, j + 1:]
            if kind == "sign":
                W[:, j + 1:] += np.outer(e, row)
            elif kind == "skip_next":
                W[:, j + 2:] -= np.outer(e, U[j, j + 2:])
            elif kind == "no_diag":
                W[:, j + 1:] -= np.outer(e * U[j, j], row)
            elif kind == "drop_update":
                pass
            codes[:, j] = q
            err[:, j] = e
        return {"codes": codes, "err": err}
    return sweep


@pytest.mark.parametrize("kind", ["sign", "skip_next", "no_diag", "drop_update",
                                  "factor_of_H"])
def test_pins_catch_planted_mistakes(kind):
    """Each plausible sweep mistake fails the Babai pin or the loss identity."""
    rng = np.random.default_rng(30)
    bad = _mutant_sweep(kind)
    caught = False
    for trial in range(40):
        n = 6
        H = _spd(n, rng)
        w = rng.standard_normal(n) * 0.02
        s, z = _single_group_params(w, 3)
        Hd, _, _ = og.damp_and_fix(H, 0.01)
        F = np.linalg.cholesky(Hd).T
        p = og.prepare(H, 0.01, "reverse")
        fixed = (s[None, :1].astype(np.float32), z[None, :1].astype(np.float32))
        U = p["U"]
        if kind == "factor_of_H":      # the factor of H instead of its inverse
            U = np.linalg.cholesky(p["Hp"]).T
        r = bad(w[None, p["perm"]], U, 3, n, fixed)
        q = r["codes"][0][og.inverse_permutation(p["perm"])]
        if not np.array_equal(q, ol.babai(F, F @ w, s, z, 3)):
            caught = True
            break
        D = w[p["perm"]] - og.dequantize(r["codes"][0], s[0], z[0])
        if not np.isclose(D @ p["Hp"] @ D, np.sum(r["err"] ** 2), rtol=1e-9):
            caught = True
            break
    assert caught, kind


# ---------------------------------------------------------------- min-pivot order

def _schur_diagonal(H, eliminated):
    """diag(H_RR − H_RE·H_EE⁻¹·H_ER) over the remaining columns R, by a solve."""
    n = H.shape[0]
    E = np.array(eliminated, dtype=np.int64)
    R = np.array([i for i in range(n) if i not in set(eliminated)], dtype=np.int64)
    if len(E) == 0:
        return R, np.diag(H)[R].copy()
    X = np.linalg.solve(H[np.ix_(E, E)], H[np.ix_(E, R)])
    return R, np.diag(H[np.ix_(R, R)] - H[np.ix_(R, E)] @ X).copy()


def test_min_pivot_golden(golden):
    for (n,), flat, want in golden("min_pivot_order.txt"):
        n = int(n)
        H = np.array([float(v) for v in flat]).reshape(n, n)
        want = [int(v) for v in want]
        assert og.min_pivot_order(H).tolist() == want
        assert og.prepare(H, 0.0, "minpivot")["perm"].tolist() == want


def test_min_pivot_diagonal_is_act_order():
    """On a diagonal H (ties and a dead column included) min-pivot = act-order."""
    rng = np.random.default_rng(41)
    for trial in range(20):
        n = 40
        d = rng.choice([0.5, 1.0, 2.0, 3.5, 7.0], size=n)
        d[rng.integers(n)] = 0.0                      # a dead column
        H = np.diag(d)
        a = og.prepare(H, 0.01, "act")["perm"]
        b = og.prepare(H, 0.01, "minpivot")["perm"]
        assert np.array_equal(a, b)


def test_min_pivot_takes_the_schur_minimum():
    """Every step eliminates the smallest Schur-complement diagonal.

    The Schur complements are recomputed from scratch with a linear solve
    (not the oracle's rank-1 updates), and the LDL pivots 1/U_jj² of the
    resulting order are those minima.
    """
    rng = np.random.default_rng(42)
    for trial in range(6):
        n = 14
        H = _spd(n, rng)
        p = og.prepare(H, 0.01, "minpivot")
        Hd = p["Hd"]
        elim = p["perm"][::-1]
        pivots = []
        for t in range(n):
            R, sd = _schur_diagonal(Hd, list(elim[:t]))
            k = int(np.flatnonzero(R == elim[t])[0])
            assert sd[k] <= sd.min() * (1 + 1e-12)
            pivots.append(sd[k])
        assert np.allclose(1.0 / np.diag(p["U"]) ** 2, np.array(pivots)[::-1], rtol=1e-9)


def test_min_pivot_catches_planted_mistakes(golden):
    """A largest-pivot rule or a rule on the undamped, un-updated diagonal fails."""
    rows = golden("min_pivot_order.txt")
    (n,), flat, want = rows[1]
    H = np.array([float(v) for v in flat]).reshape(int(n), int(n))
    want = [int(v) for v in want]

    def largest(Hd):
        S = np.array(Hd, dtype=np.float64, copy=True)
        alive = np.ones(S.shape[0], bool)
        elim = []
        for _ in range(S.shape[0]):
            d = np.where(alive, np.diag(S), -np.inf)
            j = int(np.flatnonzero(d == d.max())[-1])
            elim.append(j)
            alive[j] = False
            c = S[:, j].copy()
            S -= np.outer(c, c) / c[j]
        return elim[::-1]

    def static_diagonal(Hd):                     # no Schur updates
        return list(np.argsort(np.diag(Hd), kind="stable")[::-1])

    assert largest(H) != want
    assert static_diagonal(H) != want


def test_follow_accepts_a_zero_point_flipped_at_a_tie():
    """A zero point decided at a near-tie may go either way; the other side's
    codes then sit one step over for the whole group.  Follow mode must count
    the one allowed zero flip and no code difference (the codes are the same
    grid, shifted)."""
    W = np.array([[-1.0, 5.0, 0.3, 2.0, -0.7, 4.1, 1.1, 3.3]])
    s, z = og.group_params(W[:, :4], 4)                  # −xmin/s = 2.5 up to rounding
    zpre = 1.0 / float(s[0])
    assert abs(zpre - 2.5) < 1e-6
    z2 = np.float32(z[0] + (1 if z[0] == 2 else -1))
    s2, zb = og.group_params(W[:, 4:], 4)
    q = np.concatenate([
        np.clip(np.rint(np.float32(W[0, :4]) / s[0]) + z2, 0, 15),
        np.clip(np.rint(np.float32(W[0, 4:]) / s2[0]) + zb[0], 0, 15)])[None, :]
    scale = np.stack([s, s2], axis=1)
    zero = np.array([[z2, zb[0]]], np.float32)
    f = og.follow(W, np.eye(8), 4, 4, 8, q.astype(np.int64), scale, zero)
    assert f["zero_diff"] == 1 and f["zero_diff_disallowed"] == 0
    assert f["code_diff_disallowed"] == 0
