"""CHMC frontend oracle: plain float64 numpy, written from the pages.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  It shares no code
with the CUDA path.

Sources (page title, then the place on the page)
------------------------------------------------
[P1] "Warum Geometrie Gewichte nicht komprimiert" (nonndazone.ru article),
     section "Methodik. Was ist CHMC":
     * Schritt 1: damped activation energies c_j = (1/n)·Σ_t x²_tj + λ·mean(c)
       with λ = 0.05; the weighted truncated SVD of W̃ = W·diag(√c) by a
       randomized SVD with rank q = r and 5 power iterations; W_lr =
       (U·S)·Vᵀ·diag(1/√c).
     * Schritt 2: the residual R = W − W_lr quantized by GPTQ with act-order,
       the Hessian from the calibration activations, scales shared by groups
       of output channels (rows).
     * Schritt 3: bits per weight, BPW_CHMC = [16·r·(o+i) + b·o·i +
       16·⌈o/gs⌉·i]/(o·i) against BPW_GPTQ = [b·o·i + 16·o·⌈i/gs⌉]/(o·i), and
       the rank rule r = floor((BPW_tgt·o·i − b·o·i − 16·⌈o/gs⌉·i)/(16·(o+i))).
     * The result is W_comp = W_lr + R_q.

Readings taken where the page is silent or ambiguous
----------------------------------------------------
* The randomized SVD is the randomized subspace iteration (Halko, Martinsson
  and Tropp, "Finding structure with randomness", 2011, Algorithm 4.4): Q =
  orth(W̃·Ω), then per power iteration Q = orth(W̃ᵀ·Q), Q = orth(W̃·Q); then
  B = Qᵀ·W̃ and the SVD of the small B.  Ω (i × r, standard normal) is an
  input, drawn by the caller from a seeded generator.  Since B has exactly r
  rows, (U·S)·Vᵀ = Q·Qᵀ·W̃ and W_lr = Q·Qᵀ·W: the SVD of B only normalises
  the stored factors.
* "(1/n)·Σ_t" averages over the n calibration tokens; mean(c) is the mean of
  the undamped energies.
* The residual quantizer is the hot path's asymmetric min-max quantizer
  (integer zero point, float32 decisions), applied per column to groups of
  ``gs`` consecutive rows, with the group's parameters taken from the
  column's current (error-updated) values when the column is processed.  The
  last row group may be partial.
* R is taken against the unrounded W_lr; the factors would be stored in FP16
  (Schritt 3 counts 16 bits per factor entry), which the accounting reflects.
* The rank is clamped to [0, min(o, i)].
"""
from __future__ import annotations

import numpy as np

from . import gptq as G


# --------------------------------------------------------------------------
# Schritt 3: the bit budget
# --------------------------------------------------------------------------

def bpw_gptq(o: int, i: int, bits: int = 4, gs: int = 128) -> float:
    """[P1] Schritt 3: GPTQ's bits per weight, scales along the input channels."""
    return (bits * o * i + 16 * o * (-(-i // gs))) / (o * i)


def bpw_chmc(o: int, i: int, r: int, bits: int = 4, gs: int = 128) -> float:
    """[P1] Schritt 3: CHMC's bits per weight for rank r, scales along the rows."""
    return (16 * r * (o + i) + bits * o * i + 16 * (-(-o // gs)) * i) / (o * i)


def chmc_rank(o: int, i: int, bits: int = 4, gs: int = 128,
              bpw_target: float = 4.2875) -> int:
    """[P1] Schritt 3, the rank rule, clamped to [0, min(o, i)]."""
    num = bpw_target * o * i - bits * o * i - 16 * (-(-o // gs)) * i
    r = int(np.floor(num / (16 * (o + i))))
    return max(0, min(r, o, i))


# --------------------------------------------------------------------------
# Schritt 1: activation energies and the weighted low-rank part
# --------------------------------------------------------------------------

def activation_energy(X, lam: float = 0.05) -> np.ndarray:
    """c_j = (1/n)·Σ_t x_tj² + λ·mean(c) over the n rows (tokens) of X."""
    X = np.asarray(X, dtype=np.float64)
    c0 = np.mean(X * X, axis=0)
    return c0 + lam * np.mean(c0)


def activation_energy_from_hessian(H, tokens: int, lam: float = 0.05) -> np.ndarray:
    """The same energies from H = 2·XᵀX over ``tokens`` rows: diag(H)/(2·tokens)."""
    c0 = np.diag(np.asarray(H, dtype=np.float64)) / (2.0 * tokens)
    return c0 + lam * np.mean(c0)


def orth(A) -> np.ndarray:
    """An orthonormal basis of the columns of A (thin QR)."""
    q, _ = np.linalg.qr(np.asarray(A, dtype=np.float64), mode="reduced")
    return q


def weighted_lowrank(W, c, Omega, niter: int = 5) -> dict:
    """[P1] Schritt 1: rank-r approximation of W in the norm weighted by √c.

    ``Omega``: i × r test matrix.  Returns Q (o × r, the basis found), the
    SVD factors U (o × r), S (r), Vt (r × i) of W̃'s approximation, and
    W_lr = (U·S)·Vt·diag(1/√c).
    """
    W = np.asarray(W, dtype=np.float64)
    c = np.asarray(c, dtype=np.float64)
    Om = np.asarray(Omega, dtype=np.float64)
    sq = np.sqrt(c)
    Wt = W * sq[None, :]
    Q = orth(Wt @ Om)
    for _ in range(niter):
        Q = orth(Wt.T @ Q)
        Q = orth(Wt @ Q)
    B = Q.T @ Wt
    Ub, S, Vt = np.linalg.svd(B, full_matrices=False)
    U = Q @ Ub
    Wlr = ((U * S[None, :]) @ Vt) / sq[None, :]
    return {"Q": Q, "U": U, "S": S, "Vt": Vt, "Wlr": Wlr}


# --------------------------------------------------------------------------
# Schritt 2: GPTQ on the residual with output-channel (row) groups
# --------------------------------------------------------------------------

def rowgroup_params(col, gs: int, bits: int):
    """Scale and zero of every row group of one column, each of shape (⌈m/gs⌉,)."""
    col = np.asarray(col, dtype=np.float64)
    m = col.shape[0]
    ng = -(-m // gs)
    s = np.empty(ng, np.float32)
    z = np.empty(ng, np.float32)
    for g in range(ng):
        sg, zg = G.group_params(col[None, g * gs:min((g + 1) * gs, m)], bits)
        s[g], z[g] = sg[0], zg[0]
    return s, z


def _rows(vec_per_group, m: int, gs: int) -> np.ndarray:
    """Expand a per-row-group vector to one value per row."""
    return np.repeat(np.asarray(vec_per_group), gs)[:m]


def gptq_rowgroups_sequential(Wp, U, bits: int, gs: int = 128) -> dict:
    """The column sweep of [P1] Schritt 2 with row groups, one column at a time.

    ``Wp``: the residual with its columns in processing order; ``U``: the
    upper inverse-Cholesky factor in that order.  Returns codes, scale and
    zero (⌈m/gs⌉ × n, processing order), the errors and the pre-rounding
    values in code units.
    """
    W = np.array(Wp, dtype=np.float64, copy=True)
    U = np.asarray(U, dtype=np.float64)
    m, n = W.shape
    if gs < 1:
        raise ValueError("gs must be >= 1")
    ng = -(-m // gs)
    out = {"codes": np.zeros((m, n), np.int64),
           "scale": np.zeros((ng, n), np.float32),
           "zero": np.zeros((ng, n), np.float32),
           "err": np.zeros((m, n), np.float64),
           "pre": np.zeros((m, n), np.float64)}
    for j in range(n):
        sg, zg = rowgroup_params(W[:, j], gs, bits)
        out["scale"][:, j], out["zero"][:, j] = sg, zg
        s, z = _rows(sg, m, gs), _rows(zg, m, gs)
        out["pre"][:, j] = W[:, j] / s.astype(np.float64)
        q = G.quantize_column(W[:, j], s, z, bits)
        e = (W[:, j] - G.dequantize(q, s, z)) / U[j, j]
        W[:, j + 1:] -= np.outer(e, U[j, j + 1:])
        out["codes"][:, j] = q.astype(np.int64)
        out["err"][:, j] = e
    return out


def gptq_rowgroups_blocked(Wp, U, bits: int, gs: int = 128, block: int = 128) -> dict:
    """Lazy-batch form of :func:`gptq_rowgroups_sequential` (inside a block per
    column, one product for the later columns after it); equal up to float64
    rounding order."""
    W = np.array(Wp, dtype=np.float64, copy=True)
    U = np.asarray(U, dtype=np.float64)
    m, n = W.shape
    ng = -(-m // gs)
    out = {"codes": np.zeros((m, n), np.int64),
           "scale": np.zeros((ng, n), np.float32),
           "zero": np.zeros((ng, n), np.float32),
           "err": np.zeros((m, n), np.float64),
           "pre": np.zeros((m, n), np.float64)}
    for b0 in range(0, n, block):
        b1 = min(b0 + block, n)
        for j in range(b0, b1):
            sg, zg = rowgroup_params(W[:, j], gs, bits)
            out["scale"][:, j], out["zero"][:, j] = sg, zg
            s, z = _rows(sg, m, gs), _rows(zg, m, gs)
            out["pre"][:, j] = W[:, j] / s.astype(np.float64)
            q = G.quantize_column(W[:, j], s, z, bits)
            e = (W[:, j] - G.dequantize(q, s, z)) / U[j, j]
            W[:, j + 1:b1] -= np.outer(e, U[j, j + 1:b1])
            out["codes"][:, j] = q.astype(np.int64)
            out["err"][:, j] = e
        if b1 < n:
            W[:, b1:] -= out["err"][:, b0:b1] @ U[b0:b1, b1:]
    return out


def follow_rowgroups(Wp, U, bits: int, gs: int, block: int, codes_p, scale, zero,
                     tol: float = 1e-4) -> dict:
    """Walk the row-group sweep with another implementation's decisions.

    As :func:`oracle.gptq.follow`: at each column the oracle forms its own
    current values (from the other side's earlier codes, scales and zeros),
    its own row-group scale/zero and its own codes, then continues with the
    other side's codes.  A differing code or zero is *allowed* only if the
    oracle's pre-rounding value lies within ``tol`` code units of a rounding
    boundary.  ``scale``/``zero``: (⌈m/gs⌉, n) in processing order.
    """
    W = np.array(Wp, dtype=np.float64, copy=True)
    U = np.asarray(U, dtype=np.float64)
    m, n = W.shape
    codes_p = np.asarray(codes_p, dtype=np.int64)
    scale = np.asarray(scale, dtype=np.float32)
    zero = np.asarray(zero, dtype=np.float32)
    maxq = 2 ** bits - 1
    ng = -(-m // gs)
    n_diff = n_bad = z_diff = z_bad = 0
    max_scale_rel = 0.0
    err = np.zeros((m, n))
    for b0 in range(0, n, block):
        b1 = min(b0 + block, n)
        for j in range(b0, b1):
            s_o, z_o = rowgroup_params(W[:, j], gs, bits)
            s_g, z_g = scale[:, j], zero[:, j]
            rel = np.abs(s_g.astype(np.float64) - s_o) / np.abs(s_o)
            max_scale_rel = max(max_scale_rel, float(rel.max()))
            zd = z_g != z_o
            if zd.any():
                xmin = np.array([min(float(np.asarray(W[g * gs:min((g + 1) * gs, m), j],
                                                      np.float32).min()), 0.0)
                                 for g in range(ng)])
                zpre = -xmin / s_o.astype(np.float64)
                near_z = np.abs(zpre - np.floor(zpre) - 0.5) <= tol
                z_diff += int(zd.sum())
                z_bad += int((zd & ~near_z).sum())
                # a zero point flipped at a near-tie shifts the row group's codes
                # in this column by one: decide them with the other side's zero
                z_o = np.where(zd & near_z, z_g, z_o).astype(np.float32)
            so, zo = _rows(s_o, m, gs), _rows(z_o, m, gs)
            x = W[:, j] / so.astype(np.float64)
            q_o = G.quantize_column(W[:, j], so, zo, bits).astype(np.int64)
            q_g = codes_p[:, j]
            d = q_o != q_g
            if d.any():
                near = np.abs(x - np.floor(x) - 0.5) <= tol
                n_diff += int(d.sum())
                n_bad += int((d & ~near).sum())
            n_bad += int(np.sum((q_g < 0) | (q_g > maxq)))
            sgr, zgr = _rows(s_g, m, gs), _rows(z_g, m, gs)
            e = (W[:, j] - G.dequantize(q_g, sgr, zgr)) / U[j, j]
            W[:, j + 1:b1] -= np.outer(e, U[j, j + 1:b1])
            err[:, j] = e
        if b1 < n:
            W[:, b1:] -= err[:, b0:b1] @ U[b0:b1, b1:]
    return {"n_diff": n_diff, "n_bad": n_bad, "z_diff": z_diff, "z_bad": z_bad,
            "max_scale_rel": max_scale_rel, "err": err}


# --------------------------------------------------------------------------
# The whole CHMC layer
# --------------------------------------------------------------------------

def chmc_layer(W, H, tokens: int, Omega=None, rank: int | None = None, bits: int = 4,
               gs: int = 128, bpw_target: float = 4.2875, lam: float = 0.05,
               damp: float = 0.05, order: str = "act", niter: int = 5,
               block: int = 128) -> dict:
    """[P1] Schritte 1–3 on one layer W (o × i) with H = 2·XᵀX over ``tokens``.

    ``Omega`` (i × rank) is the randomized SVD's test matrix; ``rank`` defaults
    to the rank rule.  Returns the low-rank part, the residual's codes
    (original column order), scale/zero (⌈o/gs⌉ × i, original column order),
    the reconstruction W_comp = W_lr + R_q and the layer losses.
    """
    W = np.asarray(W, dtype=np.float64)
    o, i = W.shape
    r = chmc_rank(o, i, bits, gs, bpw_target) if rank is None else int(rank)
    c = activation_energy_from_hessian(H, tokens, lam)
    if r > 0:
        if Omega is None or np.asarray(Omega).shape != (i, r):
            raise ValueError("Omega must be i x rank")
        lr = weighted_lowrank(W, c, Omega, niter)
        Wlr = lr["Wlr"]
    else:
        lr = {"Q": np.zeros((o, 0)), "U": np.zeros((o, 0)), "S": np.zeros(0),
              "Vt": np.zeros((0, i))}
        Wlr = np.zeros_like(W)
    R = W - Wlr
    prep = G.prepare(H, damp, order)
    perm = prep["perm"]
    Rz = R.copy()
    Rz[:, prep["dead"]] = 0.0
    res = gptq_rowgroups_blocked(Rz[:, perm], prep["U"], bits, gs, block)
    inv = G.inverse_permutation(perm)
    codes = res["codes"][:, inv]
    scale = res["scale"][:, inv]
    zero = res["zero"][:, inv]
    Rq = G.dequantize(codes, _rows_matrix(scale, o, gs), _rows_matrix(zero, o, gs))
    Wc = Wlr + Rq
    return {"rank": r, "c": c, "Wlr": Wlr, "R": R, "codes": codes, "scale": scale,
            "zero": zero, "perm": perm, "dead": prep["dead"], "U": prep["U"],
            "codes_p": res["codes"], "scale_p": res["scale"], "zero_p": res["zero"],
            "err": res["err"], "Rq": Rq, "Wcomp": Wc, "lowrank": lr,
            "loss": G.layer_loss(W, Wc, H),
            "bpw": bpw_chmc(o, i, r, bits, gs)}


def _rows_matrix(per_group, m: int, gs: int) -> np.ndarray:
    """(⌈m/gs⌉, n) → (m, n): every row takes its group's row."""
    return np.repeat(np.asarray(per_group), gs, axis=0)[:m]
