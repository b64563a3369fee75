"""Static-group GPTQ oracle: group parameters fixed from the original weights.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  It shares no code
with the CUDA path.

Source (page title, then the place on the page)
-----------------------------------------------
The pages define GPTQ's groups as they are met in processing order ("Warum
Geometrie Gewichte nicht komprimiert", Methodik, Schritt 2 and 3: a scale per
group of input channels).  The static variant is not on the pages; it is the
common GPTQ option that fixes every group's scale and zero before the sweep,
from the original weights of ``group`` consecutive ORIGINAL columns, so that
act-order (the same section; the Babai page, §2.3) changes only the order in
which the columns are quantized, not which columns share a scale.

Readings
--------
* A group's parameters: the hot path's min-max quantizer (0 inside the range,
  an all-zero group → [−1, 1], float32 decisions) over the original values of
  its columns, dead columns reading 0.
* The sweep is GPTQ's column loop with those parameters: column j (processing
  order) uses the parameters of group perm[j] // group.  Nothing is
  recomputed from the current values.
* g_idx[c] = c // group.
"""
from __future__ import annotations

import numpy as np

from . import gptq as G


def static_params(Wz, bits: int, group: int):
    """(scale, zero), m × ceil(n/group): min-max of each original group."""
    Wz = np.asarray(Wz, dtype=np.float64)
    m, n = Wz.shape
    ng = -(-n // group)
    scale = np.zeros((m, ng), np.float32)
    zero = np.zeros((m, ng), np.float32)
    for g in range(ng):
        scale[:, g], zero[:, g] = G.group_params(Wz[:, g * group:min((g + 1) * group, n)], bits)
    return scale, zero


def gptq_static_sequential(Wp, U, bits: int, col_group, scale, zero) -> dict:
    """The definition: one column at a time with the full row of U, the
    parameters of each column's original group."""
    W = np.array(Wp, dtype=np.float64, copy=True)
    U = np.asarray(U, dtype=np.float64)
    m, n = W.shape
    col_group = np.asarray(col_group, dtype=np.int64)
    out = {"codes": np.zeros((m, n), np.int64), "err": np.zeros((m, n))}
    for j in range(n):
        s = np.asarray(scale[:, col_group[j]], np.float32)
        z = np.asarray(zero[:, col_group[j]], np.float32)
        q = G.quantize_column(W[:, j], s, z, bits)
        e = (W[:, j] - G.dequantize(q, s, z)) / U[j, j]
        W[:, j + 1:] -= np.outer(e, U[j, j + 1:])
        out["codes"][:, j] = q.astype(np.int64)
        out["err"][:, j] = e
    return out


def gptq_static_blocked(Wp, U, bits: int, col_group, scale, zero, block: int = 128) -> dict:
    """The lazy-batch sweep with fixed parameters; ``col_group[j]`` is the
    group of processing column j.  Any block width."""
    W = np.array(Wp, dtype=np.float64, copy=True)
    U = np.asarray(U, dtype=np.float64)
    m, n = W.shape
    col_group = np.asarray(col_group, dtype=np.int64)
    out = {"codes": np.zeros((m, n), np.int64), "err": np.zeros((m, n)),
           "pre": np.zeros((m, n))}
    for b0 in range(0, n, block):
        b1 = min(b0 + block, n)
        for j in range(b0, b1):
            s = np.asarray(scale[:, col_group[j]], np.float32)
            z = np.asarray(zero[:, col_group[j]], np.float32)
            out["pre"][:, j] = W[:, j] / s.astype(np.float64)
            q = G.quantize_column(W[:, j], s, z, bits)
            e = (W[:, j] - G.dequantize(q, s, z)) / U[j, j]
            W[:, j + 1:b1] -= np.outer(e, U[j, j + 1:b1])
            out["codes"][:, j] = q.astype(np.int64)
            out["err"][:, j] = e
        if b1 < n:
            W[:, b1:] -= out["err"][:, b0:b1] @ U[b0:b1, b1:]
    return out


def gptq_layer_static(W, H, bits: int = 4, group: int = 128, block: int = 128,
                      damp: float = 0.01, order: str = "act") -> dict:
    """Static-group GPTQ on one layer; outputs in original column order."""
    W = np.asarray(W, dtype=np.float64)
    prep = G.prepare(H, damp, order)
    perm = prep["perm"]
    Wz = W.copy()
    Wz[:, prep["dead"]] = 0.0
    scale, zero = static_params(Wz, bits, group)
    res = gptq_static_blocked(Wz[:, perm], prep["U"], bits, perm // group, scale, zero, block)
    inv = G.inverse_permutation(perm)
    codes = res["codes"][:, inv]
    g_idx = np.arange(W.shape[1]) // group
    Q = G.dequantize(codes, scale[:, g_idx], zero[:, g_idx])
    return {"codes": codes, "scale": scale, "zero": zero, "g_idx": g_idx, "Q": Q,
            "perm": perm, "dead": prep["dead"], "U": prep["U"], "res_p": res,
            "loss": G.layer_loss(W, Q, H)}


def follow_static(Wp, U, bits: int, col_group, scale, zero, block: int, codes_p,
                  tol: float = 1e-4) -> dict:
    """Walk the static sweep with another implementation's codes (its scales
    and zeros are compared exactly, elsewhere): the oracle's own code from its
    own current value, a difference allowed only within ``tol`` code units of
    a rounding boundary, then the other side's code carried on."""
    W = np.array(Wp, dtype=np.float64, copy=True)
    U = np.asarray(U, dtype=np.float64)
    m, n = W.shape
    codes_p = np.asarray(codes_p, dtype=np.int64)
    col_group = np.asarray(col_group, dtype=np.int64)
    n_diff = n_bad = 0
    err = np.zeros((m, n))
    for b0 in range(0, n, block):
        b1 = min(b0 + block, n)
        for j in range(b0, b1):
            s = np.asarray(scale[:, col_group[j]], np.float32)
            z = np.asarray(zero[:, col_group[j]], np.float32)
            x = W[:, j] / s.astype(np.float64)
            q_o = G.quantize_column(W[:, j], s, z, bits).astype(np.int64)
            d = q_o != codes_p[:, j]
            if d.any():
                near = np.abs(x - np.floor(x) - 0.5) <= tol
                n_diff += int(d.sum())
                n_bad += int((d & ~near).sum())
            e = (W[:, j] - G.dequantize(codes_p[:, j], s, z)) / U[j, j]
            W[:, j + 1:b1] -= np.outer(e, U[j, j + 1:b1])
            err[:, j] = e
        if b1 < n:
            W[:, b1:] -= err[:, b0:b1] @ U[b0:b1, b1:]
    return {"n_diff": n_diff, "n_bad": n_bad, "err": err}
