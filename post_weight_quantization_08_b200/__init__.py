"""B200-native GPTQ: Hessian → inverse-Cholesky → column sweep → packed codes.

The C ABI (include/gptq_b200.h) is exposed under the same names by
:mod:`._binding`.  The helpers below only allocate the output tensors with
torch (device memory is the caller's) and call those functions; every step of
the path runs in the library's CUDA kernels.

  hessian, prepare, quantize       the path (quantize(static_groups=True):
                                   group parameters fixed from the original
                                   weights; prepare(order="minpivot"))
  chmc_lowrank, quantize_rowgroups,
  chmc_layer                       the CHMC frontend ("Warum Geometrie Gewichte
                                   nicht komprimiert", Methodik)
  ssqr_quantize                    GPTQ with full-precision outliers and a
                                   binary search on the scales ("The Geometry
                                   of LLM Quantization", §3)
  hptq_quantize                    GPTQ on one unbounded integer grid,
                                   Huffman-coded to a bit budget (same, §3)
"""
from __future__ import annotations

import torch

from ._binding import (DTYPES, ORDERS, GptqError, exported_symbols,
                       gptq_check, gptq_chmc_lowrank, gptq_chmc_rank,
                       gptq_chmc_workspace_bytes, gptq_hessian_accumulate,
                       gptq_launch_count, gptq_prepare, gptq_prepare_workspace_bytes,
                       gptq_profile_start, gptq_profile_stop, gptq_quantize,
                       gptq_quantize_rowgroups, gptq_quantize_workspace_bytes,
                       gptq_ssqr_quantize, gptq_ssqr_workspace_bytes, gptq_hptq_quantize,
                       gptq_hptq_workspace_bytes, HPTQ_SYMBOLS, HPTQ_SYMBOL_OFFSET,
                       kernel_names, lib)

__all__ = [
    "GptqError", "ORDERS", "DTYPES", "lib", "exported_symbols", "kernel_names",
    "gptq_hessian_accumulate", "gptq_prepare", "gptq_quantize", "gptq_check",
    "gptq_prepare_workspace_bytes", "gptq_quantize_workspace_bytes",
    "gptq_launch_count", "gptq_profile_start", "gptq_profile_stop",
    "gptq_quantize_rowgroups", "gptq_chmc_rank", "gptq_chmc_workspace_bytes",
    "gptq_chmc_lowrank", "gptq_ssqr_quantize", "gptq_ssqr_workspace_bytes",
    "gptq_hptq_quantize", "gptq_hptq_workspace_bytes", "HPTQ_SYMBOLS", "HPTQ_SYMBOL_OFFSET",
    "hessian", "prepare", "quantize", "workspace",
    "chmc_lowrank", "quantize_rowgroups", "chmc_layer", "ssqr_quantize", "hptq_quantize",
]


def workspace(nbytes: int, device) -> torch.Tensor:
    """A device byte buffer for the library's workspace (256-byte aligned)."""
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def _raise_info(info, stream, what):
    st, idx = gptq_check(info, stream)
    if st != 0:
        raise GptqError(st, f"{what}: device reported index {idx}")


def hessian(X: torch.Tensor, H: torch.Tensor | None = None, stream=None,
            check: bool = True) -> torch.Tensor:
    """H += 2·XᵀX; allocates a zero H when none is given."""
    if H is None:
        n = X.shape[1]
        H = torch.zeros(n, n, dtype=torch.float32, device=X.device)
    info = torch.zeros(2, dtype=torch.int32, device=X.device) if check else None
    gptq_hessian_accumulate(X, H, info, stream)
    if check:
        _raise_info(info, stream, "gptq_hessian_accumulate")
    return H


def prepare(H: torch.Tensor, damp: float = 0.01, order: str = "natural",
            perm: torch.Tensor | None = None, ws: torch.Tensor | None = None,
            stream=None, check: bool = True) -> dict:
    """Returns {"U", "perm", "dead", "info"} on H's device."""
    n = H.shape[0]
    dev = H.device
    if perm is None:
        perm = torch.empty(n, dtype=torch.int32, device=dev)
    U = torch.empty(n, n, dtype=torch.float32, device=dev)
    dead = torch.empty(n, dtype=torch.uint8, device=dev)
    info = torch.zeros(2, dtype=torch.int32, device=dev)
    if ws is None:
        ws = workspace(gptq_prepare_workspace_bytes(n), dev)
    gptq_prepare(H, damp, order, perm, U, dead, info, ws, stream)
    if check:
        _raise_info(info, stream, "gptq_prepare")
    return {"U": U, "perm": perm, "dead": dead, "info": info}


def quantize(W: torch.Tensor, prep: dict, bits: int = 4, group: int = 128,
             block: int = 128, want_loss: bool = True, want_qdq: bool = False,
             ws: torch.Tensor | None = None, stream=None, check: bool = True,
             static_groups: bool = False) -> dict:
    """Returns qweight (int32 bit patterns of the uint32 words), scale, zero,
    g_idx and optionally loss_row / Qdq.  ``static_groups``: every group's
    parameters fixed from the original weights of consecutive original
    columns (gptq_quantize_static)."""
    m, n = W.shape
    dev = W.device
    ng = -(-n // max(group, 1))             # the library rejects group < 1 itself
    nwords = -(-n * bits // 32)
    out = {
        "qweight": torch.empty(m, nwords, dtype=torch.int32, device=dev),
        "scale": torch.empty(m, ng, dtype=torch.float32, device=dev),
        "zero": torch.empty(m, ng, dtype=torch.uint8, device=dev),
        "g_idx": torch.empty(n, dtype=torch.int32, device=dev),
        "loss_row": torch.empty(m, dtype=torch.float32, device=dev) if want_loss else None,
        "Qdq": torch.empty(m, n, dtype=torch.float32, device=dev) if want_qdq else None,
        "info": torch.zeros(2, dtype=torch.int32, device=dev),
    }
    if ws is None:
        ws = workspace(gptq_quantize_workspace_bytes(m, n, block), dev)
    gptq_quantize(W, prep["U"], prep["perm"], prep["dead"], bits, group, block,
                  out["qweight"], out["scale"], out["zero"], out["g_idx"],
                  out["loss_row"], out["Qdq"], out["info"], ws, stream, static_groups)
    if check:
        _raise_info(out["info"], stream, "gptq_quantize")
    return out


# ---- CHMC frontend ("Warum Geometrie Gewichte nicht komprimiert", Methodik)

def chmc_lowrank(W: torch.Tensor, H: torch.Tensor, tokens: int, Omega: torch.Tensor | None,
                 r: int, lam: float = 0.05, niter: int = 5, ws: torch.Tensor | None = None,
                 stream=None, check: bool = True) -> dict:
    """Schritt 1: returns {"Q", "P", "R"} with W_lr = Q·P and R = W − W_lr."""
    o, i = W.shape
    dev = W.device
    out = {
        "Q": torch.empty(o, r, dtype=torch.float32, device=dev) if r > 0 else None,
        "P": torch.empty(r, i, dtype=torch.float32, device=dev) if r > 0 else None,
        "R": torch.empty(o, i, dtype=torch.float32, device=dev),
        "info": torch.zeros(2, dtype=torch.int32, device=dev),
    }
    if ws is None:
        ws = workspace(gptq_chmc_workspace_bytes(o, i, r), dev)
    gptq_chmc_lowrank(W, H, tokens, lam, Omega, r, niter, out["Q"], out["P"], out["R"],
                      out["info"], ws, stream)
    if check:
        _raise_info(out["info"], stream, "gptq_chmc_lowrank")
    return out


def quantize_rowgroups(W: torch.Tensor, prep: dict, bits: int = 4, gs: int = 128,
                       block: int = 128, want_loss: bool = True, want_qdq: bool = False,
                       ws: torch.Tensor | None = None, stream=None, check: bool = True) -> dict:
    """Schritt 2: GPTQ with scales along the output channels; scale and zero
    are ⌈m/gs⌉ × n in the original column order."""
    m, n = W.shape
    dev = W.device
    ngr = -(-m // gs)
    nwords = -(-n * bits // 32)
    out = {
        "qweight": torch.empty(m, nwords, dtype=torch.int32, device=dev),
        "scale": torch.empty(ngr, n, dtype=torch.float32, device=dev),
        "zero": torch.empty(ngr, n, dtype=torch.uint8, device=dev),
        "loss_row": torch.empty(m, dtype=torch.float32, device=dev) if want_loss else None,
        "Qdq": torch.empty(m, n, dtype=torch.float32, device=dev) if want_qdq else None,
        "info": torch.zeros(2, dtype=torch.int32, device=dev),
    }
    if ws is None:
        ws = workspace(gptq_quantize_workspace_bytes(m, n, block), dev)
    gptq_quantize_rowgroups(W, prep["U"], prep["perm"], prep["dead"], bits, gs, block,
                            out["qweight"], out["scale"], out["zero"], out["loss_row"],
                            out["Qdq"], out["info"], ws, stream)
    if check:
        _raise_info(out["info"], stream, "gptq_quantize_rowgroups")
    return out


def chmc_layer(W: torch.Tensor, H: torch.Tensor, tokens: int, Omega: torch.Tensor | None,
               r: int | None = None, bits: int = 4, gs: int = 128, bpw_target: float = 4.2875,
               lam: float = 0.05, damp: float = 0.05, order: str = "act", niter: int = 5,
               block: int = 128, stream=None) -> dict:
    """Schritte 1–3 on one layer: the low-rank part, then GPTQ of the residual
    with output-channel scales.  ``r`` defaults to the rank rule."""
    o, i = W.shape
    if r is None:
        r = gptq_chmc_rank(o, i, bits, gs, bpw_target)
    lr = chmc_lowrank(W, H, tokens, Omega, r, lam, niter, stream=stream)
    prep = prepare(H, damp, order, stream=stream)
    q = quantize_rowgroups(lr["R"], prep, bits, gs, block, want_qdq=True, stream=stream)
    return {"rank": r, **lr, **{"prep_" + k: v for k, v in prep.items()}, **q}


# ---- SSQR ("The Geometry of LLM Quantization: GPTQ as Babai's Nearest Plane
# Algorithm", §3)

def ssqr_quantize(W: torch.Tensor, prep: dict, bits: int = 3, group: int = 128,
                  block: int = 128, target: float = 0.01, iters: int = 16,
                  alpha_lo: float = 1.0 / 16, alpha_hi: float = 1.0, nnz_cap: int | None = None,
                  want_loss: bool = True, want_qdq: bool = False, want_trace: bool = False,
                  ws: torch.Tensor | None = None, stream=None, check: bool = True,
                  lookahead: bool = True) -> dict:
    """GPTQ with the overflowing weights kept: packed inlier codes, scales,
    zeros, g_idx and the outliers in CSR (row_ptr, col_idx, val, original
    columns).  ``nnz_cap`` (default floor(target·m·n), at least 1) sizes the
    CSR arrays; with ``check`` the arrays are trimmed to the outlier count."""
    m, n = W.shape
    dev = W.device
    ng = -(-n // group)
    nwords = -(-n * bits // 32)
    if nnz_cap is None:
        nnz_cap = max(int(target * m * n), 1)
    out = {
        "qweight": torch.empty(m, nwords, dtype=torch.int32, device=dev),
        "scale": torch.empty(m, ng, dtype=torch.float32, device=dev),
        "zero": torch.empty(m, ng, dtype=torch.uint8, device=dev),
        "g_idx": torch.empty(n, dtype=torch.int32, device=dev),
        "row_ptr": torch.empty(m + 1, dtype=torch.int64, device=dev),
        "col_idx": torch.empty(nnz_cap, dtype=torch.int32, device=dev),
        "val": torch.empty(nnz_cap, dtype=torch.float32, device=dev),
        "alpha": torch.empty(1, dtype=torch.float32, device=dev),
        "trace_alpha": torch.empty(iters + 1, dtype=torch.float32, device=dev) if want_trace else None,
        "trace_count": torch.empty(iters + 1, dtype=torch.int64, device=dev) if want_trace else None,
        "loss_row": torch.empty(m, dtype=torch.float32, device=dev) if want_loss else None,
        "Qdq": torch.empty(m, n, dtype=torch.float32, device=dev) if want_qdq else None,
        "info": torch.zeros(2, dtype=torch.int32, device=dev),
    }
    if ws is None:
        ws = workspace(gptq_ssqr_workspace_bytes(m, n, block), dev)
    gptq_ssqr_quantize(W, prep["U"], prep["perm"], prep["dead"], bits, group, block, target,
                       iters, alpha_lo, alpha_hi, out["qweight"], out["scale"], out["zero"],
                       out["g_idx"], out["row_ptr"], out["col_idx"], out["val"], out["alpha"],
                       out["trace_alpha"], out["trace_count"], out["loss_row"], out["Qdq"],
                       out["info"], ws, stream, lookahead)
    if check:
        _raise_info(out["info"], stream, "gptq_ssqr_quantize")
        nnz = int(out["row_ptr"][-1])
        out["col_idx"] = out["col_idx"][:nnz]
        out["val"] = out["val"][:nnz]
    return out


# ---- HPTQ ("The Geometry of LLM Quantization: GPTQ as Babai's Nearest Plane
# Algorithm", §3)

def hptq_quantize(W: torch.Tensor, prep: dict, bits: int = 4, group: int = 128,
                  block: int = 128, budget: float = 3.125, iters: int = 16,
                  alpha_lo: float = 1.0 / 16, alpha_hi: float = 16.0,
                  stream_cap: int | None = None, want_loss: bool = True,
                  want_qdq: bool = False, want_codes: bool = True, want_trace: bool = False,
                  ws: torch.Tensor | None = None, stream=None, check: bool = True,
                  lookahead: bool = True) -> dict:
    """GPTQ on the unbounded lattice s·ℤ, Huffman-coded: the integers
    (original column order), scales, g_idx, the code table (length and canonical word
    per symbol), the row bit offsets and the bit stream.  ``stream_cap``
    (default: the budget's bits, in 32-bit words, plus one word per row)
    sizes the stream; with ``check`` it is trimmed to the coded length."""
    m, n = W.shape
    dev = W.device
    ng = -(-n // group)
    if stream_cap is None:
        stream_cap = int(budget * m * n) // 32 + m + 1
    out = {
        "codes": torch.empty(m, n, dtype=torch.int16, device=dev) if want_codes else None,
        "scale": torch.empty(m, ng, dtype=torch.float32, device=dev),
        "g_idx": torch.empty(n, dtype=torch.int32, device=dev),
        "code_len": torch.empty(HPTQ_SYMBOLS, dtype=torch.uint8, device=dev),
        "code_word": torch.empty(HPTQ_SYMBOLS, dtype=torch.int64, device=dev),
        "row_off": torch.empty(m + 1, dtype=torch.int64, device=dev),
        "stream": torch.empty(max(stream_cap, 1), dtype=torch.int32, device=dev),
        "alpha": torch.empty(1, dtype=torch.float32, device=dev),
        "trace_alpha": torch.empty(iters + 1, dtype=torch.float32, device=dev) if want_trace else None,
        "trace_bits": torch.empty(iters + 1, dtype=torch.int64, device=dev) if want_trace else None,
        "loss_row": torch.empty(m, dtype=torch.float32, device=dev) if want_loss else None,
        "Qdq": torch.empty(m, n, dtype=torch.float32, device=dev) if want_qdq else None,
        "info": torch.zeros(2, dtype=torch.int32, device=dev),
    }
    if ws is None:
        ws = workspace(gptq_hptq_workspace_bytes(m, n, block), dev)
    gptq_hptq_quantize(W, prep["U"], prep["perm"], prep["dead"], bits, group, block, budget,
                       iters, alpha_lo, alpha_hi, out["codes"], out["scale"],
                       out["g_idx"], out["code_len"], out["code_word"], out["row_off"],
                       out["stream"] if stream_cap > 0 else None, out["alpha"],
                       out["trace_alpha"], out["trace_bits"], out["loss_row"], out["Qdq"],
                       out["info"], ws, stream, lookahead)
    if check:
        _raise_info(out["info"], stream, "gptq_hptq_quantize")
        nbits = int(out["row_off"][-1])
        out["stream"] = out["stream"][:-(-nbits // 32)]
    return out
