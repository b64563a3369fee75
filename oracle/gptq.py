"""GPTQ oracle: plain float64 numpy, written from the pages.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  It shares no code
with the CUDA path.

Sources (page title, then the place on the page)
------------------------------------------------
[P1] "Warum Geometrie Gewichte nicht komprimiert" (nonndazone.ru article),
     section "Methodik. Was ist CHMC", Schritt 2: the Hessian XᵀX/n plus a
     relative damping λ·mean(diag H)·I, its inverse through the Cholesky
     factorisation, columns in act-order, and for each column j: quantize with
     the group's scale, err_j = (col_j − q_j)/H⁻¹[j,j], then subtract
     err_j·H⁻¹[j, j+1:] from the columns not yet quantized.  The same section
     calls the one-column-at-a-time form with the full row of H⁻¹
     "strict_sequential" and says it is the real GPTQ update.  Schritt 3: GPTQ
     groups run along the input channels (o·⌈i/gs⌉ scales).  Table 1: GPTQ
     stores INT4 indices plus group scales.
[P2] "The Geometry of LLM Quantization: GPTQ as Babai's Nearest Plane
     Algorithm" (gist.science summary), §2.1 (layer-output L2 error as a CVP
     on the lattice B = X·diag(s), Satz 1), §2.2 (Satz 4: GPTQ run back to
     front is Babai's nearest-plane algorithm), §2.3 (Satz 5 bound; act-order
     is the descending Hessian diagonal; the min-pivot order takes the
     smallest diagonal entry at every LDL step, to shrink the trace of D).

Readings taken where the pages are silent or disagree
-----------------------------------------------------
* H = 2·XᵀX instead of XᵀX/n.  Codes do not change under H → cH because the
  damping is relative to mean(diag H).
* "H⁻¹[j, j:]" is the inverse restricted to the columns not yet quantized.
  Its row j divided by its diagonal equals U[j, j:]/U[j,j] with U the upper
  Cholesky factor of H⁻¹ (UᵀU = H⁻¹).  The per-column error is therefore
  e_j = (w_j − q̂_j)/U[j,j] and the update is w[j+1:] −= e_j·U[j, j+1:].
* Asymmetric min-max quantizer with an integer zero point (the workloads ask
  for 4-bit asymmetric).  The range always contains 0; an all-zero group uses
  [−1, 1]; ties round half to even.
* A group's scale and zero are taken at its first column in processing order,
  from the group's current (error-updated) values.  Groups are consecutive
  runs of ``group`` columns in processing order; the last may be partial.
* Where floating point decides an integer (scale → zero, value → code) the
  decision is taken in IEEE float32, the precision of the CUDA path.  Error
  propagation is float64.
* Dead columns (diag H = 0): H_jj := 1 and W[:, j] := 0.  mean(diag H) for
  the damping is taken before that fix.
* act-order sorts the Hessian diagonal (dead entries read as 1) in descending
  order; equal entries keep ascending column index.
* min-pivot order: the D of Satz 5 comes from the LDL factorisation that
  eliminates the last processed column first (1/U_jj² are its pivots), so the
  column eliminated at step t is processed at position n−1−t.  Each step takes
  the smallest diagonal entry of the current Schur complement of the damped,
  dead-fixed H_d; equal entries go to the larger column index, so that a
  diagonal H gives act-order and H = I the natural order.
"""
from __future__ import annotations

import numpy as np
from scipy.linalg import solve_triangular

ORDERS = ("natural", "act", "reverse", "custom", "minpivot")


# --------------------------------------------------------------------------
# Hessian, damping, ordering, inverse Cholesky
# --------------------------------------------------------------------------

def hessian(X) -> np.ndarray:
    """H = 2·XᵀX in float64 from the calibration activations X (T × n).

    [P1] Schritt 2 (XᵀX/n; the factor is a reading, see module docstring);
    [P2] §2.1: XᵀX is the Gram matrix of the lattice basis.
    """
    X = np.asarray(X, dtype=np.float64)
    return 2.0 * (X.T @ X)


def hessian_block(A, B) -> np.ndarray:
    """One block of H = 2·XᵀX: rows from the columns A = X[:, I], columns
    from B = X[:, J] (float64), for checking a large H tile by tile."""
    return 2.0 * (np.asarray(A, dtype=np.float64).T @ np.asarray(B, dtype=np.float64))


def damp_and_fix(H, damp: float):
    """Relative damping and the dead-column fix.

    [P1] Schritt 2: H + λ·mean(diag H)·I.  Returns (H_d, dead mask, mean).
    """
    H = np.array(H, dtype=np.float64, copy=True)
    diag = np.diag(H).copy()
    mean_diag = diag.mean()
    dead = diag == 0.0
    idx = np.nonzero(dead)[0]
    H[idx, idx] = 1.0
    H[np.diag_indices_from(H)] += float(damp) * mean_diag
    return H, dead, mean_diag


def min_pivot_order(Hd) -> np.ndarray:
    """Processing order of the min-pivot rule ([P2] §2.3, "Rolle der Reihenfolge").

    Symmetric elimination of H_d, one column at a time: take the remaining
    column with the smallest Schur-complement diagonal (ties: the larger
    column index), then S ← S − s_j·s_jᵀ/S_jj.  The column eliminated at step t
    is processed at position n−1−t.  Raises LinAlgError on a pivot ≤ 0.
    """
    S = np.array(Hd, dtype=np.float64, copy=True)
    n = S.shape[0]
    alive = np.ones(n, dtype=bool)
    elim = np.empty(n, dtype=np.int64)
    for t in range(n):
        d = np.where(alive, np.diag(S), np.inf)
        dmin = d.min()
        if not dmin > 0.0:
            raise np.linalg.LinAlgError(f"min-pivot order: pivot {dmin} at step {t}")
        j = int(np.flatnonzero(d == dmin)[-1])
        elim[t] = j
        alive[j] = False
        col = S[:, j].copy()
        S -= np.outer(col, col) / col[j]
    return elim[::-1].copy()


def order_permutation(H, dead, order: str, perm=None, Hd=None) -> np.ndarray:
    """Processing order: perm[p] = original column processed at position p.

    natural: 0..n−1.  reverse: n−1..0 ([P2] §2.2, Satz 4).  act: descending
    Hessian diagonal ([P1] Schritt 2 "act-order"; [P2] §2.3).  custom: given.
    minpivot: the min-pivot rule on the damped H_d ([P2] §2.3).
    """
    n = H.shape[0]
    if order == "minpivot":
        if Hd is None:
            raise ValueError("the min-pivot order needs the damped Hessian")
        return min_pivot_order(Hd)
    if order == "natural":
        return np.arange(n, dtype=np.int64)
    if order == "reverse":
        return np.arange(n - 1, -1, -1, dtype=np.int64)
    if order == "act":
        key = np.diag(np.asarray(H, dtype=np.float64)).copy()
        key[dead] = 1.0
        return np.argsort(-key, kind="stable").astype(np.int64)
    if order == "custom":
        perm = np.asarray(perm, dtype=np.int64)
        if perm.shape != (n,) or not np.array_equal(np.sort(perm), np.arange(n)):
            raise ValueError("custom order is not a permutation of 0..n-1")
        return perm.copy()
    raise ValueError(f"unknown order {order!r}")


def inverse_cholesky_upper(Hp) -> np.ndarray:
    """Upper U with UᵀU = Hp⁻¹, by the textbook route.

    [P1] Schritt 2 ("H⁻¹ über die Cholesky-Zerlegung"): L = chol(Hp),
    Hinv = L⁻ᵀL⁻¹, U = upper Cholesky factor of Hinv.
    """
    n = Hp.shape[0]
    L = np.linalg.cholesky(Hp)
    Linv = solve_triangular(L, np.eye(n), lower=True)
    Hinv = Linv.T @ Linv
    Hinv = 0.5 * (Hinv + Hinv.T)
    return np.linalg.cholesky(Hinv).T.copy()


def prepare(H, damp: float = 0.01, order: str = "natural", perm=None) -> dict:
    """Damp, fix dead columns, order, and factor: the whole prepare step."""
    H = np.asarray(H, dtype=np.float64)
    Hd, dead, mean_diag = damp_and_fix(H, damp)
    perm = order_permutation(H, dead, order, perm, Hd=Hd)
    Hp = Hd[np.ix_(perm, perm)]
    U = inverse_cholesky_upper(Hp)
    return {"U": U, "perm": perm, "dead": dead, "Hd": Hd, "Hp": Hp,
            "mean_diag": mean_diag}


# --------------------------------------------------------------------------
# Quantizer (decisions in float32)
# --------------------------------------------------------------------------

def group_params(cur, bits: int):
    """Scale and zero of one group from its current values, shape (m, g).

    Min-max over the group with 0 inside the range; s = (xmax − xmin)/maxq,
    z = rint(−xmin/s).  float32 arithmetic.
    """
    maxq = np.float32(2 ** bits - 1)
    v = np.asarray(cur, dtype=np.float32)
    xmin = np.minimum(v.min(axis=1), np.float32(0.0))
    xmax = np.maximum(v.max(axis=1), np.float32(0.0))
    empty = (xmin == 0) & (xmax == 0)
    xmin = np.where(empty, np.float32(-1.0), xmin)
    xmax = np.where(empty, np.float32(1.0), xmax)
    scale = ((xmax - xmin) / maxq).astype(np.float32)
    zero = np.rint((-xmin) / scale).astype(np.float32)
    return scale, zero


def quantize_column(cur, scale, zero, bits: int, clip: bool = True):
    """Integer code of each row's current value: clamp(rint(w/s) + z, 0, maxq).

    float32 arithmetic; ``clip=False`` gives the unclipped grid of [P2] §2.3.
    """
    q = np.rint(np.asarray(cur, dtype=np.float32) / scale) + zero
    if clip:
        q = np.clip(q, np.float32(0), np.float32(2 ** bits - 1))
    return q.astype(np.float32)


def dequantize(q, scale, zero):
    """q̂ = s·(q − z) in float64 (exact for these operands)."""
    return np.asarray(scale, np.float64) * (np.asarray(q, np.float64)
                                            - np.asarray(zero, np.float64))


# --------------------------------------------------------------------------
# The column sweep: definition and equivalent forms
# --------------------------------------------------------------------------

def _empty_result(m, n, group):
    ng = -(-n // group)
    return {
        "codes": np.zeros((m, n), np.int64),
        "scale": np.zeros((m, ng), np.float32),
        "zero": np.zeros((m, ng), np.float32),
        "err": np.zeros((m, n), np.float64),
        "pre": np.zeros((m, n), np.float64),
    }


def _check_args(n, bits, group):
    if bits < 1 or bits > 8:
        raise ValueError("bits must be in 1..8")
    if group < 1:
        raise ValueError("group must be >= 1")


def gptq_sequential(Wp, U, bits: int, group: int, clip: bool = True,
                    fixed=None) -> dict:
    """The definition: one column at a time with the full row of U.

    [P1] Schritt 2 ("strict_sequential": eine Spalte nach der anderen,
    vollständige Zeile).  ``Wp`` is W with its columns already in processing
    order; ``U`` the matching upper inverse-Cholesky factor.  ``fixed`` =
    (scale, zero) per (row, group) replaces the min-max step.

    Returns codes (int, −1 never occurs), scale, zero (float32 values), the
    per-column errors e_j and the pre-rounding values w_j/s in code units.
    """
    W = np.array(Wp, dtype=np.float64, copy=True)
    U = np.asarray(U, dtype=np.float64)
    m, n = W.shape
    _check_args(n, bits, group)
    out = _empty_result(m, n, group)
    s = z = None
    for j in range(n):
        g = j // group
        if j % group == 0:
            if fixed is None:
                s, z = group_params(W[:, j:j + group], bits)
            else:
                s = np.asarray(fixed[0][:, g], np.float32)
                z = np.asarray(fixed[1][:, g], np.float32)
            out["scale"][:, g], out["zero"][:, g] = s, z
        out["pre"][:, j] = W[:, j] / s.astype(np.float64)
        q = quantize_column(W[:, j], s, z, bits, clip)
        e = (W[:, j] - dequantize(q, s, z)) / U[j, j]
        W[:, j + 1:] -= np.outer(e, U[j, j + 1:])
        out["codes"][:, j] = q.astype(np.int64)
        out["err"][:, j] = e
    return out


def gptq_blocked(Wp, U, bits: int, group: int, block: int = 128,
                 clip: bool = True, fixed=None) -> dict:
    """Lazy-batch form: updates inside a block per column, one product after.

    Same arithmetic as :func:`gptq_sequential` up to float64 rounding order:
    inside block [b0, b1) each column updates only columns < b1; after the
    block, W[:, b1:] −= E[:, b0:b1]·U[b0:b1, b1:].  Requires block % group == 0
    so that a group never straddles a block.
    """
    W = np.array(Wp, dtype=np.float64, copy=True)
    U = np.asarray(U, dtype=np.float64)
    m, n = W.shape
    _check_args(n, bits, group)
    if block % group != 0:
        raise ValueError("block must be a multiple of group")
    out = _empty_result(m, n, group)
    s = z = None
    for b0 in range(0, n, block):
        b1 = min(b0 + block, n)
        for j in range(b0, b1):
            g = j // group
            if j % group == 0:
                if fixed is None:
                    s, z = group_params(W[:, j:min(j + group, n)], bits)
                else:
                    s = np.asarray(fixed[0][:, g], np.float32)
                    z = np.asarray(fixed[1][:, g], np.float32)
                out["scale"][:, g], out["zero"][:, g] = s, z
            out["pre"][:, j] = W[:, j] / s.astype(np.float64)
            q = quantize_column(W[:, j], s, z, bits, clip)
            e = (W[:, j] - dequantize(q, s, z)) / U[j, j]
            W[:, j + 1:b1] -= np.outer(e, U[j, j + 1:b1])
            out["codes"][:, j] = q.astype(np.int64)
            out["err"][:, j] = e
        if b1 < n:
            W[:, b1:] -= out["err"][:, b0:b1] @ U[b0:b1, b1:]
    return out


def gptq_downdated_inverse(Wp, Hp, bits: int, group: int,
                           clip: bool = True) -> dict:
    """The page's literal form with an explicitly down-dated inverse.

    [P1] Schritt 2: err_j = (col_j − q_j)/H⁻¹[j,j] and
    R[:, j+1:] −= err_j·H⁻¹[j, j+1:], where H⁻¹ is the inverse over the
    columns not yet quantized; after column j it is down-dated by
    H⁻¹ ← H⁻¹ − H⁻¹[:, j]H⁻¹[j, :]/H⁻¹[j,j].  Brute force, small n only.
    ``err`` is reported as (w_j − q̂_j)/sqrt(H⁻¹[j,j]) to match the U form.
    """
    W = np.array(Wp, dtype=np.float64, copy=True)
    m, n = W.shape
    _check_args(n, bits, group)
    Hinv = np.linalg.inv(np.asarray(Hp, dtype=np.float64))
    out = _empty_result(m, n, group)
    s = z = None
    for j in range(n):
        g = j // group
        if j % group == 0:
            s, z = group_params(W[:, j:j + group], bits)
            out["scale"][:, g], out["zero"][:, g] = s, z
        out["pre"][:, j] = W[:, j] / s.astype(np.float64)
        q = quantize_column(W[:, j], s, z, bits, clip)
        delta = W[:, j] - dequantize(q, s, z)
        err = delta / Hinv[j, j]
        W[:, j + 1:] -= np.outer(err, Hinv[j, j + 1:])
        out["codes"][:, j] = q.astype(np.int64)
        out["err"][:, j] = delta / np.sqrt(Hinv[j, j])
        Hinv = Hinv - np.outer(Hinv[:, j], Hinv[j, :]) / Hinv[j, j]
    return out


# --------------------------------------------------------------------------
# Whole layer, packing, losses
# --------------------------------------------------------------------------

def inverse_permutation(perm) -> np.ndarray:
    perm = np.asarray(perm, dtype=np.int64)
    inv = np.empty_like(perm)
    inv[perm] = np.arange(perm.size, dtype=np.int64)
    return inv


def pack_rows(codes, bits: int) -> np.ndarray:
    """Per row, an LSB-first bit stream of ``bits``-bit codes in uint32 words.

    Column c occupies stream bits [c·bits, (c+1)·bits); word k holds stream
    bits [32k, 32k+32).  [P1] Table 1 (INT indices) with this layout as the
    reading of an unspecified format.
    """
    codes = np.asarray(codes, dtype=np.uint64)
    m, n = codes.shape
    nwords = -(-n * bits // 32)
    out = np.zeros((m, nwords + 1), dtype=np.uint64)
    for c in range(n):
        off = c * bits
        w, sh = divmod(off, 32)
        v = codes[:, c]
        out[:, w] |= (v << np.uint64(sh)) & np.uint64(0xFFFFFFFF)
        if sh + bits > 32:
            out[:, w + 1] |= v >> np.uint64(32 - sh)
    return out[:, :nwords].astype(np.uint32)


def layer_loss(W, Q, H) -> float:
    """tr((W − Q)·H·(W − Q)ᵀ): the layer-output objective ([P2] §2.1)."""
    D = np.asarray(W, np.float64) - np.asarray(Q, np.float64)
    return float(np.sum((D @ np.asarray(H, np.float64)) * D))


def gptq_layer(W, H, bits: int = 4, group: int = 128, block: int = 128,
               damp: float = 0.01, order: str = "natural", perm=None,
               form: str = "blocked", clip: bool = True) -> dict:
    """GPTQ on one layer from (W, H), in the original column order.

    Outputs mirror the library's: codes (m × n, original order), scale and
    zero (m × ⌈n/group⌉, processing-order groups), g_idx (group of each
    original column), qweight (packed), Q (dequantized), losses.
    """
    W = np.asarray(W, dtype=np.float64)
    prep = prepare(H, damp, order, perm)
    perm = prep["perm"]
    Wz = W.copy()
    Wz[:, prep["dead"]] = 0.0
    Wp = Wz[:, perm]
    if form == "blocked":
        res = gptq_blocked(Wp, prep["U"], bits, group, block, clip)
    elif form == "sequential":
        res = gptq_sequential(Wp, prep["U"], bits, group, clip)
    else:
        raise ValueError(form)
    inv = inverse_permutation(perm)
    codes = res["codes"][:, inv]
    g_idx = (inv // group).astype(np.int64)
    Q = dequantize(codes, res["scale"][:, g_idx], res["zero"][:, g_idx])
    out = {
        "codes": codes, "scale": res["scale"], "zero": res["zero"],
        "g_idx": g_idx, "Q": Q, "perm": perm, "dead": prep["dead"],
        "U": prep["U"], "err": res["err"], "pre_p": res["pre"],
        "codes_p": res["codes"],
        "loss_rows": np.sum(res["err"] ** 2, axis=1),
        "loss": layer_loss(W, Q, H),
        "loss_damped": float(np.sum(res["err"] ** 2)),
    }
    if 1 <= bits <= 8 and clip:
        out["qweight"] = pack_rows(codes, bits)
    return out


# --------------------------------------------------------------------------
# Follow mode: the parity checker
# --------------------------------------------------------------------------

def follow(Wp, U, bits: int, group: int, block: int, codes_p, scale, zero,
           tol: float = 1e-4) -> dict:
    """Walk the sweep with another implementation's decisions.

    At each column the oracle forms its own current value (float64 from the
    other side's earlier codes, scales and zeros), its own group scale/zero at
    group starts, and its own code.  It then continues with the other side's
    code so that one legitimate flip does not cascade.  A code that differs is
    *allowed* only if the oracle's pre-rounding value w/s lies within ``tol``
    code units of a rounding boundary; likewise a differing zero point.

    ``codes_p``: (m, n) codes in processing order; ``scale``/``zero``: (m, ng).
    """
    W = np.array(Wp, dtype=np.float64, copy=True)
    U = np.asarray(U, dtype=np.float64)
    m, n = W.shape
    codes_p = np.asarray(codes_p, dtype=np.int64)
    scale = np.asarray(scale, dtype=np.float32)
    zero = np.asarray(zero, dtype=np.float32)
    maxq = 2 ** bits - 1
    n_diff = n_bad = 0
    z_diff = z_bad = 0
    max_scale_rel = 0.0
    err = np.zeros((m, n))
    for b0 in range(0, n, block):
        b1 = min(b0 + block, n)
        for j in range(b0, b1):
            g = j // group
            if j % group == 0:
                s_o, z_o = group_params(W[:, j:min(j + group, n)], bits)
                cur = np.asarray(W[:, j:min(j + group, n)], np.float32)
                xmin = np.minimum(cur.min(axis=1), 0).astype(np.float64)
                zpre = -xmin / s_o.astype(np.float64)
                s_g, z_g = scale[:, g], zero[:, g]
                rel = np.abs(s_g.astype(np.float64) - s_o) / np.abs(s_o)
                max_scale_rel = max(max_scale_rel, float(rel.max()))
                zd = z_g != z_o
                z_diff += int(zd.sum())
                near_z = np.abs(zpre - np.floor(zpre) - 0.5) <= tol
                z_bad += int((zd & ~near_z).sum())
                # a zero point flipped at a near-tie shifts the group's codes by
                # one: decide this group's codes with the other side's zero, so
                # that the one allowed flip does not count once per column
                z_o = np.where(zd & near_z, z_g, z_o).astype(np.float32)
            x = W[:, j] / s_o.astype(np.float64)
            q_o = quantize_column(W[:, j], s_o, z_o, bits).astype(np.int64)
            q_g = codes_p[:, j]
            d = q_o != q_g
            if d.any():
                near = np.abs(x - np.floor(x) - 0.5) <= tol
                n_diff += int(d.sum())
                n_bad += int((d & ~near).sum())
            if np.any((q_g < 0) | (q_g > maxq)):
                n_bad += int(np.sum((q_g < 0) | (q_g > maxq)))
            e = (W[:, j] - dequantize(q_g, s_g, z_g)) / U[j, j]
            W[:, j + 1:b1] -= np.outer(e, U[j, j + 1:b1])
            err[:, j] = e
        if b1 < n:
            W[:, b1:] -= err[:, b0:b1] @ U[b0:b1, b1:]
    return {
        "codes": m * n, "code_diff": n_diff, "code_diff_disallowed": n_bad,
        "max_scale_rel": max_scale_rel, "zero_diff": z_diff,
        "zero_diff_disallowed": z_bad, "loss_rows": np.sum(err ** 2, axis=1),
    }
