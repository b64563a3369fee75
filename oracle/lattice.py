"""Independent pins for the GPTQ oracle: lattice algorithms and RTN.

TEST INFRASTRUCTURE ONLY.  Written separately from ``oracle.gptq`` (no shared
helpers) so that a mistake in one is caught by the other.

[P2] "The Geometry of LLM Quantization: GPTQ as Babai's Nearest Plane
Algorithm" (gist.science summary):
  §2.1  minimising the layer-output L2 error is the closest-vector problem on
        the lattice with basis B = X·diag(s) and target y = X·w; Satz 1: any
        factor F with FᵀF = XᵀX gives an equivalent instance.
  §2.2  Babai's nearest-plane algorithm walks the basis from the last vector
        to the first, projects the residual target on the current Gram–Schmidt
        direction, rounds the coefficient and subtracts; Satz 4: GPTQ run back
        to front does exactly this.
  §2.3  Satz 5: without clipping the error is at most ¼·Σ s_j²·D_jj, D the
        diagonal of the LDL factorisation of the permuted Hessian.
[P1] "Warum Geometrie Gewichte nicht komprimiert", Teil 2 (scalar_q4):
        plain round-to-nearest with group scales is the baseline GPTQ beats.
"""
from __future__ import annotations

import itertools

import numpy as np


def _rint32(x):
    # Nearest integer of a float32 value, ties to even (IEEE roundTiesToEven).
    return np.rint(np.float32(x))


def minmax_params_row(values, bits: int):
    """Scale and zero of one row-group, one row at a time (no vectorisation).

    Same definition as the sweep's quantizer, written independently: the range
    [min(0, min v), max(0, max v)] split into 2^bits − 1 steps; zero point
    rint(−xmin/s); an all-zero group uses [−1, 1].  float32 arithmetic.
    """
    lo = np.float32(0.0)
    hi = np.float32(0.0)
    for v in np.asarray(values, dtype=np.float32).ravel():
        if v < lo:
            lo = v
        if v > hi:
            hi = v
    if lo == 0 and hi == 0:
        lo, hi = np.float32(-1.0), np.float32(1.0)
    s = np.float32(np.float32(hi - lo) / np.float32(2 ** bits - 1))
    z = _rint32(np.float32(-lo) / s)
    return s, z


def rtn(W, bits: int, group: int):
    """Round-to-nearest with min-max groups along the input channels.

    Returns (codes, scale, zero, Q) with natural-order groups of the original
    W; no error feedback.
    """
    W = np.asarray(W, dtype=np.float64)
    m, n = W.shape
    ng = -(-n // group)
    maxq = 2 ** bits - 1
    codes = np.zeros((m, n), np.int64)
    scale = np.zeros((m, ng), np.float32)
    zero = np.zeros((m, ng), np.float32)
    Q = np.zeros((m, n))
    for r in range(m):
        for g in range(ng):
            c0, c1 = g * group, min((g + 1) * group, n)
            s, z = minmax_params_row(W[r, c0:c1], bits)
            scale[r, g], zero[r, g] = s, z
            for c in range(c0, c1):
                q = _rint32(np.float32(np.float32(W[r, c]) / s)) + z
                q = min(max(int(q), 0), maxq)
                codes[r, c] = q
                Q[r, c] = float(s) * (q - float(z))
    return codes, scale, zero, Q


def rtn_dequant(W, bits: int, group: int) -> np.ndarray:
    """The dequantized weights of :func:`rtn`, all rows and groups at once.

    The same float32 steps as ``rtn`` (range [min(0, min v), max(0, max v)],
    an all-zero group on [−1, 1], scale (hi − lo)/(2^bits − 1), zero point and
    codes rounded half to even, codes clamped to [0, 2^bits − 1]) on whole
    arrays, for layers too large for the element loop; pinned equal to it.
    """
    W32 = np.asarray(W, dtype=np.float32)
    m, n = W32.shape
    maxq = np.float32(2 ** bits - 1)
    Q = np.zeros((m, n))
    for c0 in range(0, n, group):
        v = W32[:, c0:c0 + group]
        lo = np.minimum(v.min(axis=1), np.float32(0))
        hi = np.maximum(v.max(axis=1), np.float32(0))
        empty = (lo == 0) & (hi == 0)
        lo = np.where(empty, np.float32(-1), lo)
        hi = np.where(empty, np.float32(1), hi)
        s = ((hi - lo) / maxq).astype(np.float32)
        z = np.rint((-lo) / s).astype(np.float32)
        q = np.clip(np.rint(v / s[:, None]) + z[:, None], 0, maxq)
        Q[:, c0:c0 + group] = s[:, None].astype(np.float64) * (
            q.astype(np.float64) - z[:, None].astype(np.float64))
    return Q


def babai(B, y, scale, zero, bits: int, clip: bool = True):
    """Babai's nearest-plane algorithm, basis vectors processed last to first.

    ``B`` (d × n) holds the *unscaled* basis columns (e.g. X, or a square factor
    F with FᵀF = H); the lattice is B·diag(s) shifted by the zero points, i.e.
    points B·(s ⊙ (q − z)).  ``y`` is the target, B·w for weights w.  The
    Gram–Schmidt directions come from a QR factorisation of B·diag(s).
    Returns integer codes q (length n).
    """
    B = np.asarray(B, dtype=np.float64)
    s = np.asarray(scale, dtype=np.float64)
    z = np.asarray(zero, dtype=np.float64)
    n = B.shape[1]
    maxq = 2 ** bits - 1
    Bs = B * s[None, :]
    Qm, R = np.linalg.qr(Bs, mode="reduced")
    t = Qm.T @ np.asarray(y, dtype=np.float64)   # residual target, GS coords
    q = np.zeros(n, dtype=np.int64)
    for k in range(n - 1, -1, -1):
        coeff = t[k] / R[k, k]                   # coefficient along b*_k
        a = int(np.rint(coeff + z[k]))
        if clip:
            a = min(max(a, 0), maxq)
        q[k] = a
        t[: k + 1] -= (a - z[k]) * R[: k + 1, k]  # subtract the chosen b_k
    return q


def cvp_bruteforce(H, w, scale, zero, bits: int):
    """Exact minimiser of (w − q̂)ᵀH(w − q̂) over every code vector (tiny n)."""
    H = np.asarray(H, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    s = np.asarray(scale, dtype=np.float64)
    z = np.asarray(zero, dtype=np.float64)
    n = w.size
    best, best_q = np.inf, None
    for q in itertools.product(range(2 ** bits), repeat=n):
        d = w - s * (np.asarray(q, np.float64) - z)
        v = float(d @ H @ d)
        if v < best:
            best, best_q = v, np.asarray(q, np.int64)
    return best_q, best
