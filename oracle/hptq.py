"""HPTQ oracle: unclipped GPTQ codes, Huffman-coded to a bit budget.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  It shares no code
with the CUDA path.

Source (page title, then the place on the page)
-----------------------------------------------
[P2] "The Geometry of LLM Quantization: GPTQ as Babai's Nearest Plane
     Algorithm" (gist.science summary), §3 "Praktische Anwendungen und
     Algorithmen": Huffman-encoded PTQ (HPTQ) puts inliers and outliers on one
     unbounded integer grid and Huffman-codes the resulting integers, so that
     the bit width adapts to the weight distribution while a given compression
     budget is met.  §4 reports 3.125 bits per weight as its sweet spot.  §2.3
     (Satz 5): without clipping, GPTQ keeps its error bound.

Readings taken where the page is silent
---------------------------------------
* The grid is the lattice s·ℤ of each group: the group's min-max step s₀
  (the hot path's, from ``bits`` nominal bits, taken at the group's first
  column from its current values) becomes s = fl32(α·s₀), and a weight's
  integer is k = rint(w/s), any integer, decided in float32.  Its error is
  w − s·k (no clipping, so |error| ≤ s/2).  With no clamp a zero point has no
  role (rint(w/s) + z − z = rint(w/s) for an integer z), so the integers are
  the lattice coordinates themselves, centred on 0, and one code serves every
  group: "one unbounded integer grid".
* One Huffman code per weight matrix over its integers k.  The budget counts
  the coded payload: Σ_q count(q)·len(q) ≤ B_max = floor(budget·m·n) bits.
  The scales and the code table are stored beside it and not counted.
* A matrix whose codes take one value only codes it with 1 bit.
* Huffman lengths are not unique where counts tie; the optimal total cost is.
  Both sides' decisions use the cost; a code table is checked as valid (Kraft
  sum 1) and optimal (its cost equals the optimum).
* The binary search is SSQR's with "admissible" meaning cost ≤ B_max: α_hi
  (the coarsest grid) first, over budget there ends the search with α_hi;
  then ``iters`` bisection steps on [α_lo, α_hi] with float32 midpoints; the
  result is hi, the finest grid found within budget.
* The bit stream: canonical Huffman codes (assigned in order of (length,
  symbol)), each weight's code written most significant bit first, rows one
  after another in original column order, the stream packed into 32-bit
  words most significant bit first.  Row r starts at bit row_off[r].
"""
from __future__ import annotations

import heapq

import numpy as np

from . import gptq as G


def max_bits(budget: float, m: int, n: int) -> int:
    """B_max = floor(budget·m·n)."""
    return int(np.floor(float(budget) * float(m) * float(n)))


def lattice_column(cur, scale):
    """k = rint(w/s) in float32: the weight's coordinate on s·ℤ."""
    return np.rint(np.asarray(cur, dtype=np.float32) / scale).astype(np.float32)


def hptq_sequential(Wp, U, bits: int, group: int, alpha) -> dict:
    """The definition: one column at a time, each error pushed onto every
    later column with the full row of U (columns in processing order)."""
    W = np.array(Wp, dtype=np.float64, copy=True)
    U = np.asarray(U, dtype=np.float64)
    m, n = W.shape
    ng = -(-n // group)
    out = {"codes": np.zeros((m, n), np.int64), "scale": np.zeros((m, ng), np.float32),
           "err": np.zeros((m, n))}
    s = None
    for j in range(n):
        if j % group == 0:
            s0, _ = G.group_params(W[:, j:j + group], bits)
            s = (s0 * np.float32(alpha)).astype(np.float32)
            out["scale"][:, j // group] = s
        q = lattice_column(W[:, j], s)
        e = (W[:, j] - s.astype(np.float64) * q.astype(np.float64)) / U[j, j]
        W[:, j + 1:] -= np.outer(e, U[j, j + 1:])
        out["codes"][:, j] = q.astype(np.int64)
        out["err"][:, j] = e
    return out


def hptq_blocked(Wp, U, bits: int, group: int, block: int, alpha) -> dict:
    """The unclipped sweep, lazy-batch form, columns in processing order;
    codes are the unbounded lattice coordinates k."""
    if block % group != 0:
        raise ValueError("block must be a multiple of group")
    W = np.array(Wp, dtype=np.float64, copy=True)
    U = np.asarray(U, dtype=np.float64)
    m, n = W.shape
    ng = -(-n // group)
    out = {"codes": np.zeros((m, n), np.int64), "scale": np.zeros((m, ng), np.float32),
           "err": np.zeros((m, n)), "pre": np.zeros((m, n))}
    s = None
    a32 = np.float32(alpha)
    for b0 in range(0, n, block):
        b1 = min(b0 + block, n)
        for j in range(b0, b1):
            g = j // group
            if j % group == 0:
                s0, _ = G.group_params(W[:, j:min(j + group, n)], bits)
                s = (s0 * a32).astype(np.float32)
                out["scale"][:, g] = s
            out["pre"][:, j] = W[:, j] / s.astype(np.float64)
            q = lattice_column(W[:, j], s)
            e = (W[:, j] - s.astype(np.float64) * q.astype(np.float64)) / U[j, j]
            W[:, j + 1:b1] -= np.outer(e, U[j, j + 1:b1])
            out["codes"][:, j] = q.astype(np.int64)
            out["err"][:, j] = e
        if b1 < n:
            W[:, b1:] -= out["err"][:, b0:b1] @ U[b0:b1, b1:]
    return out


def histogram(codes) -> dict:
    vals, cnt = np.unique(np.asarray(codes, np.int64), return_counts=True)
    return {int(v): int(c) for v, c in zip(vals, cnt)}


def huffman_lengths(hist: dict) -> dict:
    """Code length per symbol of an optimal prefix code (Huffman's merge of
    the two lightest subtrees, with a heap; ties broken by insertion order)."""
    if not hist:
        return {}
    if len(hist) == 1:
        return {next(iter(hist)): 1}
    heap = []
    for i, (sym, c) in enumerate(sorted(hist.items())):
        heapq.heappush(heap, (c, i, [sym]))
    depth = {sym: 0 for sym in hist}
    k = len(hist)
    while len(heap) > 1:
        c1, _, s1 = heapq.heappop(heap)
        c2, _, s2 = heapq.heappop(heap)
        for sym in s1 + s2:
            depth[sym] += 1
        heapq.heappush(heap, (c1 + c2, k, s1 + s2))
        k += 1
    return depth


def cost(hist: dict, lengths: dict) -> int:
    return int(sum(c * lengths[s] for s, c in hist.items()))


def kraft(lengths: dict) -> float:
    return float(sum(2.0 ** -l for l in lengths.values()))


def canonical_codes(lengths: dict) -> dict:
    """symbol → (code, length): codes assigned in order of (length, symbol),
    each the previous one plus one, shifted left when the length grows."""
    order = sorted(lengths.items(), key=lambda kv: (kv[1], kv[0]))
    out, code, prev = {}, 0, None
    for sym, ln in order:
        if prev is not None:
            code = (code + 1) << (ln - prev)
        out[sym] = (code, ln)
        prev = ln
    return out


def encode(codes, lengths: dict):
    """Rows of ``codes`` (original column order) → (row_off[m+1], words)."""
    cb = canonical_codes(lengths)
    codes = np.asarray(codes, np.int64)
    m, n = codes.shape
    bits = []
    row_off = [0]
    for r in range(m):
        for q in codes[r]:
            c, ln = cb[int(q)]
            bits.extend((c >> (ln - 1 - i)) & 1 for i in range(ln))
        row_off.append(len(bits))
    nw = -(-len(bits) // 32)
    words = np.zeros(nw, np.uint32)
    for p, b in enumerate(bits):
        if b:
            words[p // 32] |= np.uint32(1) << np.uint32(31 - p % 32)
    return np.array(row_off, np.int64), words


def decode(words, row_off, lengths: dict, m: int, n: int):
    """The inverse of :func:`encode` (walks each row's bits)."""
    cb = canonical_codes(lengths)
    table = {(c, ln): s for s, (c, ln) in cb.items()}
    words = np.asarray(words, np.uint32)
    out = np.zeros((m, n), np.int64)
    for r in range(m):
        p = int(row_off[r])
        for j in range(n):
            c = ln = 0
            while True:
                c = (c << 1) | int((int(words[p // 32]) >> (31 - p % 32)) & 1)
                p += 1
                ln += 1
                if (c, ln) in table:
                    out[r, j] = table[(c, ln)]
                    break
                if ln > 64:
                    raise ValueError("not a code word")
        if p != int(row_off[r + 1]):
            raise ValueError("row length mismatch")
    return out


def coded_bits(res) -> int:
    h = histogram(res["codes"])
    return cost(h, huffman_lengths(h))


def bisect_alpha(run, b_max: int, iters: int = 16, alpha_lo: float = 1.0 / 16,
                 alpha_hi: float = 16.0):
    """SSQR's search with the coded size as the constraint.  ``run(α)``
    returns a result with "codes".  Returns (α, result, trace of (α, bits))."""
    hi = np.float32(alpha_hi)
    lo = np.float32(alpha_lo)
    res_hi = run(hi)
    b = coded_bits(res_hi)
    trace = [(float(hi), b)]
    if b > b_max:
        return hi, res_hi, trace
    for _ in range(iters):
        mid = np.float32((float(lo) + float(hi)) / 2.0)
        if mid <= lo or mid >= hi:
            break
        res = run(mid)
        b = coded_bits(res)
        trace.append((float(mid), b))
        if b <= b_max:
            hi, res_hi = mid, res
        else:
            lo = mid
    return hi, res_hi, trace


def hptq_layer(W, H, bits: int = 4, group: int = 128, block: int = 128, damp: float = 0.01,
               order: str = "act", budget: float = 3.125, iters: int = 16,
               alpha_lo: float = 1.0 / 16, alpha_hi: float = 16.0, prep=None) -> dict:
    """HPTQ on one layer: the search, then the chosen sweep's codes in
    original column order, their Huffman code and the layer loss."""
    W = np.asarray(W, dtype=np.float64)
    m, n = W.shape
    if prep is None:
        prep = G.prepare(H, damp, order)
    perm = prep["perm"]
    Wz = W.copy()
    Wz[:, prep["dead"]] = 0.0
    Wp = Wz[:, perm]
    alpha, res, trace = bisect_alpha(
        lambda a: hptq_blocked(Wp, prep["U"], bits, group, block, a),
        max_bits(budget, m, n), iters, alpha_lo, alpha_hi)
    inv = G.inverse_permutation(perm)
    codes = res["codes"][:, inv]
    g_idx = (inv // group).astype(np.int64)
    Q = res["scale"][:, g_idx].astype(np.float64) * codes
    hist = histogram(codes)
    lengths = huffman_lengths(hist)
    return {"alpha": alpha, "trace": trace, "codes": codes, "scale": res["scale"],
            "g_idx": g_idx, "Q": Q, "hist": hist, "lengths": lengths,
            "bits": cost(hist, lengths), "perm": perm, "dead": prep["dead"], "U": prep["U"],
            "res_p": res, "loss": G.layer_loss(W, Q, H)}


def follow_hptq(Wp, U, bits: int, group: int, block: int, alpha, codes_p, scale,
                tol: float = 1e-4, scale_rtol: float = 1e-5) -> dict:
    """Walk the unclipped sweep with another implementation's codes.

    As the SSQR checker: the oracle forms its own current values from the
    other side's earlier decisions, its own scale at group starts and
    its own code; a differing code is allowed only within ``tol`` code units
    of a rounding boundary; scales are held to ``scale_rtol`` or, in a group
    narrower than 32 columns, to the float32 forward-error bound of the
    propagation (2·γ_K·M/(2^b − 1)·α, γ_K = 2⁻²¹ + K·2⁻²⁴, M the largest
    |w| + Σ|e_k·U_kj| of the group).  Arrays in processing order.
    """
    W = np.array(Wp, dtype=np.float64, copy=True)
    U = np.asarray(U, dtype=np.float64)
    m, n = W.shape
    codes_p = np.asarray(codes_p, dtype=np.int64)
    scale = np.asarray(scale, dtype=np.float32)
    maxq = 2 ** bits - 1
    n_diff = n_bad = scale_bad = scale_wide_over = 0
    max_scale_rel = 0.0
    err = np.zeros((m, n))
    mag = np.abs(W)
    s_o = None
    a32 = np.float32(alpha)
    for b0 in range(0, n, block):
        b1 = min(b0 + block, n)
        for j in range(b0, b1):
            g = j // group
            if j % group == 0:
                cur = W[:, j:min(j + group, n)]
                s0, _ = G.group_params(cur, bits)
                s_o = (s0 * a32).astype(np.float32)
                rel = np.abs(scale[:, g].astype(np.float64) - s_o) / np.abs(s_o)
                width = cur.shape[1]
                M = mag[:, j:j + width].max(axis=1)
                bound = 2.0 * (2.0 ** -21 + j * 2.0 ** -24) * M / maxq * float(a32) / np.abs(s_o)
                scale_bad += int(np.sum(rel > np.maximum(scale_rtol, bound)))
                if width >= 32:
                    scale_wide_over += int(np.sum(rel > scale_rtol))
                max_scale_rel = max(max_scale_rel, float(rel.max()))
            s_g = scale[:, g]
            x = W[:, j] / s_o.astype(np.float64)
            q_o = lattice_column(W[:, j], s_o).astype(np.int64)
            q_g = codes_p[:, j]
            d = q_o != q_g
            if d.any():
                near = np.abs(x - np.floor(x) - 0.5) <= tol
                n_diff += int(d.sum())
                n_bad += int((d & ~near).sum())
            e = (W[:, j] - s_g.astype(np.float64) * q_g) / U[j, j]
            W[:, j + 1:b1] -= np.outer(e, U[j, j + 1:b1])
            mag[:, j + 1:b1] += np.outer(np.abs(e), np.abs(U[j, j + 1:b1]))
            err[:, j] = e
        if b1 < n:
            W[:, b1:] -= err[:, b0:b1] @ U[b0:b1, b1:]
            mag[:, b1:] += np.abs(err[:, b0:b1]) @ np.abs(U[b0:b1, b1:])
    return {"n_diff": n_diff, "n_bad": n_bad, "max_scale_rel": max_scale_rel,
            "scale_bad": scale_bad, "scale_wide_over": scale_wide_over, "err": err}
