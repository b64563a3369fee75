"""GPU-vs-oracle parity checks shared by the GPU tests.

Tolerances (written here, each derived from the arithmetic it checks):
  * H: |ΔH_ij| ≤ 2·T·2⁻²⁴·S_ij with S = 2·|X|ᵀ|X| — the float32 summation
    bound γ_T of a length-T dot product (bf16 products are exact in float32).
  * U: the library computes in float64 and rounds once to float32, so
    |ΔU_ij| ≤ 2⁻²²·|U_ij| + n·κ(H_d)·2⁻⁵³·max_k|U_ik| (four float32 ulps plus
    the forward-error scale of two float64 factorisations).
  * quantize (oracle in follow mode on the GPU's own H/U): a code may differ
    only where the oracle's pre-rounding value lies within 1e-4 code units of
    a rounding boundary, and such codes are at most 0.1 % of all codes;
    scales agree to 1e-5 relative; zeros are equal unless at such a near-tie,
    and such zero flips are at most 0.1 % of the (row, group) pairs (the same
    cap as codes: a flipped zero is a rounding decision of the same kind);
    the layer loss agrees to 1e-3 relative.
  * round-to-nearest dominance: the GPU result's layer loss tr((W−Q)H(W−Q)ᵀ)
    does not exceed that of round-to-nearest with the same groups.
  * end to end (oracle from X alone, float64 throughout): layer loss to 1e-3
    relative.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import gptq as og

CODE_TOL = 1e-4
CODE_FRAC = 1e-3
ZERO_FRAC = 1e-3
SCALE_RTOL = 1e-5
LOSS_RTOL = 1e-3


def unpack_rows(qweight: np.ndarray, bits: int, n: int) -> np.ndarray:
    """Codes (m × n) from the LSB-first uint32 bit stream of each row."""
    w = np.asarray(qweight).view(np.uint32).astype(np.uint64)
    m = w.shape[0]
    out = np.zeros((m, n), dtype=np.int64)
    mask = np.uint64((1 << bits) - 1)
    for c in range(n):
        off = c * bits
        k, sh = divmod(off, 32)
        v = w[:, k] >> np.uint64(sh)
        if sh + bits > 32:
            v |= w[:, k + 1] << np.uint64(32 - sh)
        out[:, c] = (v & mask).astype(np.int64)
    return out


def run_gpu(X, W, bits=4, group=128, block=128, damp=0.01, order="natural",
            perm=None, device="cuda:0", qdq=True):
    """The whole path on the GPU; returns numpy copies of every output."""
    import post_weight_quantization_08_b200 as g
    dev = torch.device(device)
    Xd = X.to(device=dev, dtype=torch.bfloat16).contiguous()
    Wd = W.to(device=dev).contiguous()
    H = g.hessian(Xd)
    pin = None if perm is None else torch.as_tensor(perm, dtype=torch.int32, device=dev)
    prep = g.prepare(H, damp, order, perm=pin)
    q = g.quantize(Wd, prep, bits, group, block, want_loss=True, want_qdq=qdq)
    torch.cuda.synchronize(dev)
    out = {k: v.cpu().numpy() for k, v in q.items() if v is not None}
    out.update(H=H.cpu().numpy(), U=prep["U"].cpu().numpy(),
               perm=prep["perm"].cpu().numpy().astype(np.int64),
               dead=prep["dead"].cpu().numpy().astype(bool))
    out["codes"] = unpack_rows(out["qweight"], bits, W.shape[1])
    return out


def check_hessian(X, H_gpu):
    Xf = X.to(torch.bfloat16).to(torch.float64).numpy()
    T = Xf.shape[0]
    H = og.hessian(Xf)
    S = 2.0 * (np.abs(Xf).T @ np.abs(Xf))
    tol = 2.0 * T * 2.0 ** -24 * S + 1e-30
    err = np.abs(H_gpu.astype(np.float64) - H)
    ratio = float(np.max(err / tol))
    assert ratio <= 1.0, f"Hessian outside the float32 summation bound: {ratio}"
    assert np.array_equal(H_gpu, H_gpu.T), "Hessian not symmetric"
    return {"hessian_err_over_bound": ratio,
            "hessian_max_rel": float(np.max(err / (np.sqrt(np.outer(np.diag(H), np.diag(H))) + 1e-300)))}


def check_prepare(H_gpu, out, damp, order, perm=None):
    ref = og.prepare(H_gpu.astype(np.float64), damp, order, perm)
    assert np.array_equal(out["perm"], ref["perm"]), "permutation differs"
    assert np.array_equal(out["dead"], ref["dead"]), "dead mask differs"
    U, Ur = out["U"].astype(np.float64), ref["U"]
    assert np.all(np.tril(U, -1) == 0), "U has a non-zero below the diagonal"
    rowmax = np.max(np.abs(Ur), axis=1, keepdims=True)
    # float32 rounding (4 ulps) + the float64 forward-error scale n·κ·2⁻⁵³
    ev = np.linalg.eigvalsh(ref["Hp"])
    kappa = float(ev[-1] / ev[0])
    n = Ur.shape[0]
    tol = 2.0 ** -22 * np.abs(Ur) + n * kappa * 2.0 ** -53 * rowmax
    ratio = float(np.max(np.abs(U - Ur) / (tol + 1e-300)))
    assert ratio <= 1.0, f"U outside tolerance: {ratio}"
    return ref, {"U_err_over_tol": ratio, "kappa": kappa}


def check_quantize(W, out, ref_prep_U, bits, group, block, rows=None):
    """Follow-mode parity of the sweep on the GPU's own U and permutation."""
    Wf = W.to(torch.float64).numpy() if isinstance(W, torch.Tensor) else np.asarray(W, np.float64)
    perm, dead = out["perm"], out["dead"]
    sel = slice(None) if rows is None else rows
    Wz = Wf[sel].copy()
    Wz[:, dead] = 0.0
    Wp = Wz[:, perm]
    codes_p = out["codes"][sel][:, perm]
    f = og.follow(Wp, out["U"].astype(np.float64), bits, group, block, codes_p,
                  out["scale"][sel], out["zero"][sel], CODE_TOL)
    assert f["code_diff_disallowed"] == 0, f
    assert f["code_diff"] <= CODE_FRAC * f["codes"], f
    assert f["max_scale_rel"] <= SCALE_RTOL, f
    assert f["zero_diff_disallowed"] == 0, f
    assert f["zero_diff"] <= ZERO_FRAC * out["scale"][sel].size, f
    lg = out["loss_row"][sel].astype(np.float64)
    lo = f["loss_rows"]
    assert abs(lg.sum() - lo.sum()) <= LOSS_RTOL * lo.sum(), (lg.sum(), lo.sum())
    # g_idx: processing-order groups mapped back to original columns
    inv = og.inverse_permutation(perm)
    assert np.array_equal(out["g_idx"], inv // group)
    # the packed words are exactly the oracle's packing of the GPU codes
    assert np.array_equal(og.pack_rows(out["codes"][sel], bits).view(np.int32),
                          out["qweight"][sel])
    if "Qdq" in out:
        g = out["g_idx"]
        Q = out["scale"][sel][:, g].astype(np.float64) * (
            out["codes"][sel] - out["zero"][sel][:, g].astype(np.float64))
        assert np.allclose(out["Qdq"][sel], Q, rtol=2 ** -23, atol=0)
    return {"codes": f["codes"], "code_diff": f["code_diff"],
            "max_scale_rel": f["max_scale_rel"], "zero_diff": f["zero_diff"],
            "damped_loss_gpu": float(lg.sum()), "damped_loss_oracle": float(lo.sum())}


def check_layer_loss(X, W, out, bits, group, block, damp, order, perm=None):
    """End to end: undamped layer loss of the GPU result vs the oracle's own
    run from X alone (float64 throughout)."""
    Xf = X.to(torch.bfloat16).to(torch.float64).numpy()
    Wf = W.to(torch.float64).numpy()
    H = og.hessian(Xf)
    ref = og.gptq_layer(Wf, H, bits, group, block, damp, order, perm)
    lg = og.layer_loss(Wf, dequantized(out), H)
    rel = abs(lg - ref["loss"]) / ref["loss"]
    assert rel <= LOSS_RTOL, (lg, ref["loss"], rel)
    return {"loss_gpu": lg, "loss_oracle": ref["loss"], "loss_rel": rel,
            "code_agree": float(np.mean(ref["codes"] == out["codes"]))}


def dequantized(out):
    """Q = s·(q − z) in float64 from the GPU's codes, scales, zeros and g_idx."""
    g = out["g_idx"]
    return out["scale"][:, g].astype(np.float64) * (
        out["codes"] - out["zero"][:, g].astype(np.float64))


def check_rtn_dominance(W, out, H, bits, group):
    """The GPU result's layer loss does not exceed round-to-nearest's (min-max
    groups of the original W along the input channels), both measured with
    the same float64 H."""
    from oracle import lattice as ol
    Wf = W.to(torch.float64).numpy() if isinstance(W, torch.Tensor) else np.asarray(W, np.float64)
    H = np.asarray(H, dtype=np.float64)
    lg = og.layer_loss(Wf, dequantized(out), H)
    lr = og.layer_loss(Wf, ol.rtn_dequant(Wf, bits, group), H)
    assert lg <= lr, (lg, lr)
    return {"loss_gpu_undamped": lg, "loss_rtn": lr, "loss_over_rtn": lg / lr}
