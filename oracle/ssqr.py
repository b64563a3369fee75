"""SSQR oracle: GPTQ with full-precision outliers, plain float64 numpy.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  It shares no code
with the CUDA path.

Source (page title, then the place on the page)
-----------------------------------------------
[P2] "The Geometry of LLM Quantization: GPTQ as Babai's Nearest Plane
     Algorithm" (gist.science summary), §3 "Praktische Anwendungen und
     Algorithmen": scale-adjusted SpQR (SSQR) tolerates overflow instead of
     clipping it.  A small share of the weights (the outliers) is kept in full
     precision as a sparse floating-point part, the rest (the inliers) is
     quantized to a low bit width, and a binary search moves the scales until
     the outlier density reaches a target.  The same section motivates it:
     clipping an overflowing weight breaks the error bound of Satz 5 (§2.3).

Readings taken where the page is silent
---------------------------------------
* The scales are adjusted by one factor α for the whole layer: each group's
  min-max step s₀ (the hot path's quantizer, taken at the group's first
  column from its current values) becomes s = α·s₀, rounded to float32.  The
  zero point z = rint(−xmin/s₀) stays, so for α < 1 the grid
  s·([0, 2^b − 1] − z) shrinks towards 0 and keeps 0 on it.
* An outlier is a weight whose unclipped code rint(w/s) + z falls outside
  [0, 2^b − 1] when its column is processed (decided in float32, like every
  code).  It keeps its current value exactly, so its error is 0 and nothing
  propagates from it; the layer stores it as (row, original column, value).
  Its packed code is the clipped one, which dequantization ignores.
* The binary search evaluates α_hi first.  If more than
  N_max = floor(target·m·n) weights are outliers there, it stops with α_hi.
  Otherwise it bisects [α_lo, α_hi] for ``iters`` steps: the midpoint
  (lo + hi)/2 rounded to float32 becomes the new hi when it has at most N_max
  outliers, else the new lo; it stops early when the midpoint equals lo or
  hi.  The result is hi: the finest grid found whose outliers stay within the
  budget.  The outlier count need not fall monotonically as α grows (the
  errors that propagate change with α); the search is defined by these steps.
"""
from __future__ import annotations

import numpy as np

from . import gptq as G


def max_outliers(target: float, m: int, n: int) -> int:
    """N_max = floor(target·m·n): the largest outlier count the target allows."""
    return int(np.floor(float(target) * float(m) * float(n)))


def adjusted_params(cur, bits: int, alpha):
    """(s, z) of one group: s = fl32(α·s₀), z from s₀ (min-max of ``cur``)."""
    s0, z = G.group_params(cur, bits)
    return (s0 * np.float32(alpha)).astype(np.float32), z, s0


def quantize_column_outliers(cur, scale, zero, bits: int):
    """(clipped code, outlier flag, pre-rounding value w/s) of each row."""
    q = np.rint(np.asarray(cur, dtype=np.float32) / scale) + zero
    maxq = np.float32(2 ** bits - 1)
    out = (q < 0) | (q > maxq)
    return np.clip(q, np.float32(0), maxq).astype(np.float32), out


def _result(m, n, group):
    ng = -(-n // group)
    return {"codes": np.zeros((m, n), np.int64), "mask": np.zeros((m, n), bool),
            "value": np.zeros((m, n), np.float64),
            "scale": np.zeros((m, ng), np.float32), "zero": np.zeros((m, ng), np.float32),
            "err": np.zeros((m, n), np.float64), "pre": np.zeros((m, n), np.float64)}


def _column(W, j, s, z, bits, U, out):
    """Quantize column j of W (current values) and return its error."""
    out["pre"][:, j] = W[:, j] / s.astype(np.float64)
    q, o = quantize_column_outliers(W[:, j], s, z, bits)
    qhat = np.where(o, W[:, j], G.dequantize(q, s, z))
    e = (W[:, j] - qhat) / U[j, j]
    out["codes"][:, j] = q.astype(np.int64)
    out["mask"][:, j] = o
    out["value"][:, j] = np.where(o, W[:, j], 0.0)
    out["err"][:, j] = e
    return e


def ssqr_sequential(Wp, U, bits: int, group: int, alpha) -> dict:
    """The definition: one column at a time, each error pushed onto every
    later column with the full row of U (columns in processing order)."""
    W = np.array(Wp, dtype=np.float64, copy=True)
    U = np.asarray(U, dtype=np.float64)
    m, n = W.shape
    out = _result(m, n, group)
    s = z = None
    for j in range(n):
        if j % group == 0:
            s, z, _ = adjusted_params(W[:, j:j + group], bits, alpha)
            out["scale"][:, j // group], out["zero"][:, j // group] = s, z
        e = _column(W, j, s, z, bits, U, out)
        W[:, j + 1:] -= np.outer(e, U[j, j + 1:])
    return out


def ssqr_blocked(Wp, U, bits: int, group: int, block: int, alpha) -> dict:
    """Lazy-batch form: inside block [b0, b1) each column updates the block's
    later columns; after the block, W[:, b1:] −= E[:, b0:b1]·U[b0:b1, b1:].
    Requires block % group == 0."""
    if block % group != 0:
        raise ValueError("block must be a multiple of group")
    W = np.array(Wp, dtype=np.float64, copy=True)
    U = np.asarray(U, dtype=np.float64)
    m, n = W.shape
    out = _result(m, n, group)
    s = z = None
    for b0 in range(0, n, block):
        b1 = min(b0 + block, n)
        for j in range(b0, b1):
            if j % group == 0:
                s, z, _ = adjusted_params(W[:, j:min(j + group, n)], bits, alpha)
                out["scale"][:, j // group], out["zero"][:, j // group] = s, z
            e = _column(W, j, s, z, bits, U, out)
            W[:, j + 1:b1] -= np.outer(e, U[j, j + 1:b1])
        if b1 < n:
            W[:, b1:] -= out["err"][:, b0:b1] @ U[b0:b1, b1:]
    return out


def count(res) -> int:
    return int(np.count_nonzero(res["mask"]))


def bisect_alpha(run, n_max: int, iters: int = 16, alpha_lo: float = 1.0 / 16,
                 alpha_hi: float = 1.0):
    """The binary search on α (module readings).  ``run(α)`` takes a float32 α
    and returns a result with a "mask".  Returns (α, result at α, trace of
    (α, outlier count) per evaluation)."""
    hi = np.float32(alpha_hi)
    lo = np.float32(alpha_lo)
    res_hi = run(hi)
    trace = [(float(hi), count(res_hi))]
    if count(res_hi) > n_max:
        return hi, res_hi, trace
    for _ in range(iters):
        mid = np.float32((float(lo) + float(hi)) / 2.0)
        if mid <= lo or mid >= hi:
            break
        res = run(mid)
        trace.append((float(mid), count(res)))
        if count(res) <= n_max:
            hi, res_hi = mid, res
        else:
            lo = mid
    return hi, res_hi, trace


def ssqr_layer(W, H, bits: int = 3, group: int = 128, block: int = 128, damp: float = 0.01,
               order: str = "act", target: float = 0.01, iters: int = 16,
               alpha_lo: float = 1.0 / 16, alpha_hi: float = 1.0, prep=None) -> dict:
    """SSQR on one layer: the hot path's preparation, the binary search, and
    the chosen sweep's outputs in original column order, with the outliers as
    (row, column, value) lists in row-major order."""
    W = np.asarray(W, dtype=np.float64)
    m, n = W.shape
    if prep is None:
        prep = G.prepare(H, damp, order)
    perm = prep["perm"]
    Wz = W.copy()
    Wz[:, prep["dead"]] = 0.0
    Wp = Wz[:, perm]
    alpha, res, trace = bisect_alpha(
        lambda a: ssqr_blocked(Wp, prep["U"], bits, group, block, a),
        max_outliers(target, m, n), iters, alpha_lo, alpha_hi)
    inv = G.inverse_permutation(perm)
    codes = res["codes"][:, inv]
    mask = res["mask"][:, inv]
    value = res["value"][:, inv]
    g_idx = (inv // group).astype(np.int64)
    Q = np.where(mask, value, G.dequantize(codes, res["scale"][:, g_idx], res["zero"][:, g_idx]))
    rows, cols = np.nonzero(mask)
    return {"alpha": alpha, "trace": trace, "codes": codes, "mask": mask,
            "scale": res["scale"], "zero": res["zero"], "g_idx": g_idx, "Q": Q,
            "outlier_rows": rows, "outlier_cols": cols, "outlier_vals": value[rows, cols],
            "count": int(mask.sum()), "perm": perm, "dead": prep["dead"], "U": prep["U"],
            "res_p": res, "loss": G.layer_loss(W, Q, H)}


def follow_ssqr(Wp, U, bits: int, group: int, block: int, alpha, codes_p, mask_p, vals_p,
                scale, zero, tol: float = 1e-4, scale_rtol: float = 1e-5) -> dict:
    """Walk the SSQR sweep with another implementation's decisions.

    At each column the oracle forms its own current values (float64, from the
    other side's earlier decisions), its own scale and zero at group starts,
    and its own (code, outlier flag).  A (code, flag) pair that differs is
    allowed only where the oracle's pre-rounding value w/s lies within ``tol``
    code units of a rounding boundary.  It then continues with the other
    side's decision: an outlier contributes no error.  ``vals_p`` holds the
    other side's stored outlier values; their largest deviation from the
    oracle's current value is reported relative to |w| + s₀·(2^b − 1).

    Scales: ``scale_rtol`` relative, or, where the group's own float32
    working precision is coarser, the forward-error bound of the float32
    propagation that built its current values: |Δs| ≤ 2·γ_K·M/(2^b − 1)·α
    with M the largest |w| + Σ|e_k·U_kj| over the group at its start, K the
    columns processed before it and γ_K = 2⁻²¹ + K·2⁻²⁴ (a three-term TF32
    product and K float32 additions).  ``scale_bad`` counts groups beyond both;
    ``scale_wide_over`` counts groups of at least 32 columns beyond
    ``scale_rtol`` alone.  Kept values likewise: ``val_bad`` counts those off
    by more than both 1e-5·(|w| + s₀·(2^b − 1)) and γ_j·M_j (j their column).

    Arrays in processing order: codes_p, mask_p, vals_p (m × n); scale and
    zero (m × ngroups).
    """
    W = np.array(Wp, dtype=np.float64, copy=True)
    U = np.asarray(U, dtype=np.float64)
    m, n = W.shape
    codes_p = np.asarray(codes_p, dtype=np.int64)
    mask_p = np.asarray(mask_p, dtype=bool)
    scale = np.asarray(scale, dtype=np.float32)
    zero = np.asarray(zero, dtype=np.float32)
    maxq = 2 ** bits - 1
    n_diff = n_bad = z_diff = z_bad = scale_bad = scale_wide_over = val_bad = 0
    max_scale_rel = max_val_rel = 0.0
    worst = None
    err = np.zeros((m, n))
    mag = np.abs(W)                   # |w| + Σ|e_k·U_kj| of the updates so far
    s_o = z_o = s0 = None
    for b0 in range(0, n, block):
        b1 = min(b0 + block, n)
        for j in range(b0, b1):
            g = j // group
            if j % group == 0:
                cur = W[:, j:min(j + group, n)]
                s_o, z_o, s0 = adjusted_params(cur, bits, alpha)
                c32 = np.asarray(cur, np.float32)
                zpre = -np.minimum(c32.min(axis=1), 0).astype(np.float64) / s0.astype(np.float64)
                rel = np.abs(scale[:, g].astype(np.float64) - s_o) / np.abs(s_o)
                width = cur.shape[1]
                M = mag[:, j:j + width].max(axis=1)
                gam = 2.0 ** -21 + j * 2.0 ** -24
                bound = 2.0 * gam * M / maxq * float(alpha) / np.abs(s_o)
                scale_bad += int(np.sum(rel > np.maximum(scale_rtol, bound)))
                if width >= 32:
                    scale_wide_over += int(np.sum(rel > scale_rtol))
                if float(rel.max()) > max_scale_rel:
                    r = int(np.argmax(rel))
                    rng = float(s0[r]) * maxq
                    worst = {"row": r, "group": g, "cols": cur.shape[1],
                             "mag_over_range": float(mag[r, j:j + cur.shape[1]].max()) / rng}
                max_scale_rel = max(max_scale_rel, float(rel.max()))
                zd = zero[:, g] != z_o
                near_z = np.abs(zpre - np.floor(zpre) - 0.5) <= tol
                z_diff += int(zd.sum())
                z_bad += int((zd & ~near_z).sum())
                # a zero point flipped at a near-tie shifts the group's codes by
                # one: decide this group's codes with the other side's zero
                z_o = np.where(zd & near_z, zero[:, g], z_o).astype(np.float32)
            s_g, z_g = scale[:, g], zero[:, g]
            x = W[:, j] / s_o.astype(np.float64)
            q_o, o_o = quantize_column_outliers(W[:, j], s_o, z_o, bits)
            q_g, o_g = codes_p[:, j], mask_p[:, j]
            d = (q_o.astype(np.int64) != q_g) | (o_o != o_g)
            if d.any():
                near = np.abs(x - np.floor(x) - 0.5) <= tol
                n_diff += int(d.sum())
                n_bad += int((d & ~near).sum())
            n_bad += int(np.sum((q_g < 0) | (q_g > maxq)))
            if o_g.any():
                v = np.asarray(vals_p[:, j], np.float64)[o_g]
                ref = W[o_g, j]
                den = np.abs(ref) + s0[o_g].astype(np.float64) * maxq
                dv = np.abs(v - ref)
                max_val_rel = max(max_val_rel, float(np.max(dv / den)))
                gam = 2.0 ** -21 + j * 2.0 ** -24
                val_bad += int(np.sum(dv > np.maximum(1e-5 * den, gam * mag[o_g, j])))
            qhat = np.where(o_g, W[:, j], G.dequantize(q_g, s_g, z_g))
            e = (W[:, j] - qhat) / U[j, j]
            W[:, j + 1:b1] -= np.outer(e, U[j, j + 1:b1])
            mag[:, j + 1:b1] += np.outer(np.abs(e), np.abs(U[j, j + 1:b1]))
            err[:, j] = e
        if b1 < n:
            W[:, b1:] -= err[:, b0:b1] @ U[b0:b1, b1:]
            mag[:, b1:] += np.abs(err[:, b0:b1]) @ np.abs(U[b0:b1, b1:])
    return {"n_diff": n_diff, "n_bad": n_bad, "z_diff": z_diff, "z_bad": z_bad,
            "max_scale_rel": max_scale_rel,
            "scale_bad": scale_bad, "scale_wide_over": scale_wide_over, "worst_scale": worst,
            "val_bad": val_bad, "max_val_rel": max_val_rel, "err": err,
            "count": int(mask_p.sum())}
