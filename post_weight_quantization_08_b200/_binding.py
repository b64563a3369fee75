"""ctypes binding of libgptq_b200.so: argument marshalling only.

The C functions keep their names; each wrapper checks dtypes, shapes and
devices of the torch tensors it is given, passes their data pointers and the
CUDA stream, and turns a non-OK status into :class:`GptqError`.  All
computation happens in the library's CUDA kernels.  There is no fallback: if
the library is missing, every call raises.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgptq_b200.so")

STATUS = {0: "GPTQ_OK", 1: "GPTQ_ERR_INVALID_ARG", 2: "GPTQ_ERR_NOT_PD",
          3: "GPTQ_ERR_NONFINITE", 4: "GPTQ_ERR_UNSUPPORTED",
          5: "GPTQ_ERR_TIMEOUT", 6: "GPTQ_ERR_CUDA", 7: "GPTQ_ERR_CAPACITY"}
ORDERS = {"natural": 0, "act": 1, "reverse": 2, "custom": 3, "minpivot": 4}
DTYPES = {torch.float32: 0, torch.bfloat16: 1}

# name: (restype, argtypes)
_SIGS = {
    "gptq_hessian_accumulate": (C.c_int, [C.c_void_p, C.c_int64, C.c_int64, C.c_void_p,
                                          C.c_void_p, C.c_void_p]),
    "gptq_prepare_workspace_bytes": (C.c_size_t, [C.c_int64]),
    "gptq_prepare": (C.c_int, [C.c_void_p, C.c_int64, C.c_double, C.c_int, C.c_void_p,
                               C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_size_t,
                               C.c_void_p]),
    "gptq_prepare_noalloc": (C.c_int, [C.c_void_p, C.c_int64, C.c_double, C.c_int,
                                       C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p,
                                       C.c_void_p]),
    "gptq_quantize_workspace_bytes": (C.c_size_t, [C.c_int64, C.c_int64, C.c_int]),
    "gptq_quantize": (C.c_int, [C.c_void_p, C.c_int, C.c_int64, C.c_int64, C.c_void_p,
                                C.c_void_p, C.c_void_p, C.c_int, C.c_int, C.c_int,
                                C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p,
                                C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p,
                                C.c_size_t, C.c_void_p]),
    "gptq_quantize_static": (C.c_int, [C.c_void_p, C.c_int, C.c_int64, C.c_int64, C.c_void_p,
                                       C.c_void_p, C.c_void_p, C.c_int, C.c_int, C.c_int,
                                       C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p,
                                       C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p,
                                       C.c_size_t, C.c_void_p]),
    "gptq_quantize_rowgroups": (C.c_int, [C.c_void_p, C.c_int, C.c_int64, C.c_int64,
                                          C.c_void_p, C.c_void_p, C.c_void_p, C.c_int,
                                          C.c_int, C.c_int, C.c_void_p, C.c_void_p,
                                          C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p,
                                          C.c_void_p, C.c_size_t, C.c_void_p]),
    "gptq_chmc_rank": (C.c_int, [C.c_int64, C.c_int64, C.c_int, C.c_int, C.c_double]),
    "gptq_chmc_workspace_bytes": (C.c_size_t, [C.c_int64, C.c_int64, C.c_int]),
    "gptq_chmc_lowrank": (C.c_int, [C.c_void_p, C.c_int, C.c_int64, C.c_int64, C.c_void_p,
                                    C.c_int64, C.c_double, C.c_void_p, C.c_int, C.c_int,
                                    C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p,
                                    C.c_void_p, C.c_size_t, C.c_void_p]),
    "gptq_ssqr_workspace_bytes": (C.c_size_t, [C.c_int64, C.c_int64, C.c_int]),
    "gptq_ssqr_quantize": (C.c_int, [C.c_void_p, C.c_int, C.c_int64, C.c_int64, C.c_void_p,
                                     C.c_void_p, C.c_void_p, C.c_int, C.c_int, C.c_int,
                                     C.c_double, C.c_int, C.c_float, C.c_float, C.c_int,
                                     C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p,
                                     C.c_void_p, C.c_void_p, C.c_void_p, C.c_int64,
                                     C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p,
                                     C.c_void_p, C.c_void_p, C.c_void_p, C.c_size_t,
                                     C.c_void_p]),
    "gptq_hptq_workspace_bytes": (C.c_size_t, [C.c_int64, C.c_int64, C.c_int]),
    "gptq_hptq_quantize": (C.c_int, [C.c_void_p, C.c_int, C.c_int64, C.c_int64, C.c_void_p,
                                     C.c_void_p, C.c_void_p, C.c_int, C.c_int, C.c_int,
                                     C.c_double, C.c_int, C.c_float, C.c_float, C.c_int,
                                     C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p,
                                     C.c_void_p, C.c_void_p, C.c_void_p,
                                     C.c_int64, C.c_void_p, C.c_void_p, C.c_void_p,
                                     C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p,
                                     C.c_size_t, C.c_void_p]),
    "gptq_set_wait_limit": (None, [C.c_uint32]),
    "gptq_set_factor_workers": (None, [C.c_int]),
    "gptq_peak_probe": (C.c_int, [C.c_int, C.c_int64, C.POINTER(C.c_double), C.c_void_p,
                                  C.c_void_p, C.c_void_p]),
    "gptq_check": (C.c_int, [C.c_void_p, C.POINTER(C.c_int32), C.c_void_p]),
    "gptq_last_error": (C.c_char_p, []),
    "gptq_status_string": (C.c_char_p, [C.c_int]),
    "gptq_launch_count": (C.c_uint64, []),
    "gptq_kernel_kinds": (C.c_int, []),
    "gptq_kernel_name": (C.c_char_p, [C.c_int]),
    "gptq_profile_start": (C.c_int, [C.c_int]),
    "gptq_profile_stop": (C.c_int, []),
    "gptq_profile_get": (C.c_int, [C.c_int, C.POINTER(C.c_double), C.POINTER(C.c_int64)]),
}

_lib = None


class GptqError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status


def lib() -> C.CDLL:
    """The loaded library (loaded on first use; raises if it is missing)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m post_weight_quantization_08_b200.build` (nvcc, sm_100a)")
        handle = C.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(handle, name)
            f.restype, f.argtypes = res, args
        _lib = handle
    return _lib


def exported_symbols() -> list[str]:
    return list(_SIGS)


def _raise(status: int):
    if status != 0:
        msg = lib().gptq_last_error().decode(errors="replace")
        raise GptqError(status, msg)


def _stream(stream, device) -> int:
    if stream is None:
        return torch.cuda.current_stream(device).cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t):
    return None if t is None else t.data_ptr()


def _need(t, name, dtype, shape=None, device=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


# ---------------------------------------------------------------- C calls

def gptq_hessian_accumulate(X, H, info=None, stream=None):
    """H += 2·XᵀX (X: T×n bf16, H: n×n float32; both on the same GPU)."""
    _need(X, "X", torch.bfloat16)
    T, n = X.shape
    _need(H, "H", torch.float32, (n, n), X.device)
    if info is not None:
        _need(info, "info", torch.int32, (2,), X.device)
    _raise(lib().gptq_hessian_accumulate(_ptr(X), T, n, _ptr(H), _ptr(info),
                                         _stream(stream, X.device)))


def gptq_prepare_workspace_bytes(n: int) -> int:
    return int(lib().gptq_prepare_workspace_bytes(n))


def gptq_quantize_workspace_bytes(m: int, n: int, block: int) -> int:
    return int(lib().gptq_quantize_workspace_bytes(m, n, block))


def gptq_prepare(H, damp, order, perm, U, dead, info, ws, stream=None):
    """Damp, order and factor H into U (see include/gptq_b200.h)."""
    _need(H, "H", torch.float32)
    n = H.shape[0]
    dev = H.device
    _need(perm, "perm", torch.int32, (n,), dev)
    _need(U, "U", torch.float32, (n, n), dev)
    _need(dead, "dead", torch.uint8, (n,), dev)
    _need(info, "info", torch.int32, (2,), dev)
    _need(ws, "ws", torch.uint8, None, dev)
    order = ORDERS[order] if isinstance(order, str) else int(order)
    _raise(lib().gptq_prepare(_ptr(H), n, float(damp), order, _ptr(perm), _ptr(U),
                              _ptr(dead), _ptr(info), _ptr(ws), ws.numel(),
                              _stream(stream, dev)))


def gptq_quantize(W, U, perm, dead, bits, group, block, qweight, scale, zero,
                  g_idx, loss_row, Qdq, info, ws, stream=None, static_groups=False):
    """Quantize W with U (see include/gptq_b200.h); ``static_groups`` calls
    gptq_quantize_static (parameters fixed from the original weights)."""
    if W.dtype not in DTYPES:
        raise TypeError("W must be float32 or bfloat16")
    _need(W, "W", W.dtype)
    m, n = W.shape
    dev = W.device
    ng = -(-n // max(group, 1))           # the library rejects group < 1 itself
    nwords = -(-n * bits // 32)
    _need(U, "U", torch.float32, (n, n), dev)
    _need(perm, "perm", torch.int32, (n,), dev)
    _need(dead, "dead", torch.uint8, (n,), dev)
    _need(qweight, "qweight", torch.int32, (m, nwords), dev)
    _need(scale, "scale", torch.float32, (m, ng), dev)
    _need(zero, "zero", torch.uint8, (m, ng), dev)
    _need(g_idx, "g_idx", torch.int32, (n,), dev)
    if loss_row is not None:
        _need(loss_row, "loss_row", torch.float32, (m,), dev)
    if Qdq is not None:
        _need(Qdq, "Qdq", torch.float32, (m, n), dev)
    _need(info, "info", torch.int32, (2,), dev)
    _need(ws, "ws", torch.uint8, None, dev)
    fn = lib().gptq_quantize_static if static_groups else lib().gptq_quantize
    _raise(fn(_ptr(W), DTYPES[W.dtype], m, n, _ptr(U), _ptr(perm),
                               _ptr(dead), int(bits), int(group), int(block),
                               _ptr(qweight), _ptr(scale), _ptr(zero), _ptr(g_idx),
                               _ptr(loss_row), _ptr(Qdq), _ptr(info), _ptr(ws),
                               ws.numel(), _stream(stream, dev)))


def gptq_quantize_rowgroups(W, U, perm, dead, bits, gs, block, qweight, scale, zero,
                            loss_row, Qdq, info, ws, stream=None):
    """Quantize W with scales along the output channels (see include/gptq_b200.h)."""
    if W.dtype not in DTYPES:
        raise TypeError("W must be float32 or bfloat16")
    _need(W, "W", W.dtype)
    m, n = W.shape
    dev = W.device
    ngr = -(-m // gs)
    nwords = -(-n * bits // 32)
    _need(U, "U", torch.float32, (n, n), dev)
    _need(perm, "perm", torch.int32, (n,), dev)
    _need(dead, "dead", torch.uint8, (n,), dev)
    _need(qweight, "qweight", torch.int32, (m, nwords), dev)
    _need(scale, "scale", torch.float32, (ngr, n), dev)
    _need(zero, "zero", torch.uint8, (ngr, n), dev)
    if loss_row is not None:
        _need(loss_row, "loss_row", torch.float32, (m,), dev)
    if Qdq is not None:
        _need(Qdq, "Qdq", torch.float32, (m, n), dev)
    _need(info, "info", torch.int32, (2,), dev)
    _need(ws, "ws", torch.uint8, None, dev)
    _raise(lib().gptq_quantize_rowgroups(_ptr(W), DTYPES[W.dtype], m, n, _ptr(U), _ptr(perm),
                                         _ptr(dead), int(bits), int(gs), int(block),
                                         _ptr(qweight), _ptr(scale), _ptr(zero),
                                         _ptr(loss_row), _ptr(Qdq), _ptr(info), _ptr(ws),
                                         ws.numel(), _stream(stream, dev)))


def gptq_ssqr_workspace_bytes(m: int, n: int, block: int) -> int:
    return int(lib().gptq_ssqr_workspace_bytes(m, n, block))


def gptq_ssqr_quantize(W, U, perm, dead, bits, group, block, target, iters, alpha_lo,
                       alpha_hi, qweight, scale, zero, g_idx, row_ptr, col_idx, val, alpha,
                       trace_alpha, trace_count, loss_row, Qdq, info, ws, stream=None,
                       lookahead=1):
    """SSQR: GPTQ with kept outliers and a binary search on the scale factor
    (see include/gptq_b200.h)."""
    if W.dtype not in DTYPES:
        raise TypeError("W must be float32 or bfloat16")
    _need(W, "W", W.dtype)
    m, n = W.shape
    dev = W.device
    ng = -(-n // max(group, 1))           # the library rejects group < 1 itself
    nwords = -(-n * bits // 32)
    _need(U, "U", torch.float32, (n, n), dev)
    _need(perm, "perm", torch.int32, (n,), dev)
    _need(dead, "dead", torch.uint8, (n,), dev)
    _need(qweight, "qweight", torch.int32, (m, nwords), dev)
    _need(scale, "scale", torch.float32, (m, ng), dev)
    _need(zero, "zero", torch.uint8, (m, ng), dev)
    _need(g_idx, "g_idx", torch.int32, (n,), dev)
    _need(row_ptr, "row_ptr", torch.int64, (m + 1,), dev)
    cap = 0 if col_idx is None else col_idx.numel()
    if cap:
        _need(col_idx, "col_idx", torch.int32, (cap,), dev)
        _need(val, "val", torch.float32, (cap,), dev)
    _need(alpha, "alpha", torch.float32, (1,), dev)
    if trace_alpha is not None:
        _need(trace_alpha, "trace_alpha", torch.float32, (iters + 1,), dev)
        _need(trace_count, "trace_count", torch.int64, (iters + 1,), dev)
    if loss_row is not None:
        _need(loss_row, "loss_row", torch.float32, (m,), dev)
    if Qdq is not None:
        _need(Qdq, "Qdq", torch.float32, (m, n), dev)
    _need(info, "info", torch.int32, (2,), dev)
    _need(ws, "ws", torch.uint8, None, dev)
    _raise(lib().gptq_ssqr_quantize(
        _ptr(W), DTYPES[W.dtype], m, n, _ptr(U), _ptr(perm), _ptr(dead), int(bits),
        int(group), int(block), float(target), int(iters), float(alpha_lo), float(alpha_hi),
        int(bool(lookahead)), _ptr(qweight), _ptr(scale), _ptr(zero), _ptr(g_idx), _ptr(row_ptr),
        _ptr(col_idx) if cap else None, _ptr(val) if cap else None, cap, _ptr(alpha),
        _ptr(trace_alpha), _ptr(trace_count), _ptr(loss_row), _ptr(Qdq), _ptr(info),
        _ptr(ws), ws.numel(), _stream(stream, dev)))


HPTQ_SYMBOLS = 4096
HPTQ_SYMBOL_OFFSET = 2048


def gptq_hptq_workspace_bytes(m: int, n: int, block: int) -> int:
    return int(lib().gptq_hptq_workspace_bytes(m, n, block))


def gptq_hptq_quantize(W, U, perm, dead, bits, group, block, budget, iters, alpha_lo,
                       alpha_hi, codes, scale, g_idx, code_len, code_word, row_off,
                       stream_words, alpha, trace_alpha, trace_bits, loss_row, Qdq, info, ws,
                       stream=None, lookahead=1):
    """HPTQ: unclipped GPTQ codes, Huffman-coded to a bit budget (see
    include/gptq_b200.h)."""
    if W.dtype not in DTYPES:
        raise TypeError("W must be float32 or bfloat16")
    _need(W, "W", W.dtype)
    m, n = W.shape
    dev = W.device
    ng = -(-n // max(group, 1))           # the library rejects group < 1 itself
    _need(U, "U", torch.float32, (n, n), dev)
    _need(perm, "perm", torch.int32, (n,), dev)
    _need(dead, "dead", torch.uint8, (n,), dev)
    if codes is not None:
        _need(codes, "codes", torch.int16, (m, n), dev)
    _need(scale, "scale", torch.float32, (m, ng), dev)
    _need(g_idx, "g_idx", torch.int32, (n,), dev)
    _need(code_len, "code_len", torch.uint8, (HPTQ_SYMBOLS,), dev)
    if code_word is not None:
        _need(code_word, "code_word", torch.int64, (HPTQ_SYMBOLS,), dev)
    _need(row_off, "row_off", torch.int64, (m + 1,), dev)
    cap = 0 if stream_words is None else stream_words.numel()
    if cap:
        _need(stream_words, "stream_words", torch.int32, (cap,), dev)
    _need(alpha, "alpha", torch.float32, (1,), dev)
    if trace_alpha is not None:
        _need(trace_alpha, "trace_alpha", torch.float32, (iters + 1,), dev)
        _need(trace_bits, "trace_bits", torch.int64, (iters + 1,), dev)
    if loss_row is not None:
        _need(loss_row, "loss_row", torch.float32, (m,), dev)
    if Qdq is not None:
        _need(Qdq, "Qdq", torch.float32, (m, n), dev)
    _need(info, "info", torch.int32, (2,), dev)
    _need(ws, "ws", torch.uint8, None, dev)
    _raise(lib().gptq_hptq_quantize(
        _ptr(W), DTYPES[W.dtype], m, n, _ptr(U), _ptr(perm), _ptr(dead), int(bits),
        int(group), int(block), float(budget), int(iters), float(alpha_lo), float(alpha_hi),
        int(bool(lookahead)), _ptr(codes), _ptr(scale), _ptr(g_idx), _ptr(code_len), _ptr(code_word),
        _ptr(row_off), _ptr(stream_words) if cap else None, cap, _ptr(alpha),
        _ptr(trace_alpha), _ptr(trace_bits), _ptr(loss_row), _ptr(Qdq), _ptr(info), _ptr(ws),
        ws.numel(), _stream(stream, dev)))


def gptq_chmc_rank(o: int, i: int, bits: int = 4, gs: int = 128,
                   bpw_target: float = 4.2875) -> int:
    """The rank rule of the bit budget (see include/gptq_b200.h)."""
    return int(lib().gptq_chmc_rank(int(o), int(i), int(bits), int(gs), float(bpw_target)))


def gptq_chmc_workspace_bytes(o: int, i: int, r: int) -> int:
    return int(lib().gptq_chmc_workspace_bytes(int(o), int(i), int(r)))


def gptq_chmc_lowrank(W, H, tokens, lam, Omega, r, niter, Q, P, R, info, ws, stream=None):
    """Low-rank part and residual of W (see include/gptq_b200.h)."""
    if W.dtype not in DTYPES:
        raise TypeError("W must be float32 or bfloat16")
    _need(W, "W", W.dtype)
    o, i = W.shape
    dev = W.device
    if r > 0:
        _need(H, "H", torch.float32, (i, i), dev)
        _need(Omega, "Omega", torch.float32, (i, r), dev)
    if Q is not None:
        _need(Q, "Q", torch.float32, (o, r), dev)
    if P is not None:
        _need(P, "P", torch.float32, (r, i), dev)
    _need(R, "R", torch.float32, (o, i), dev)
    _need(info, "info", torch.int32, (2,), dev)
    _need(ws, "ws", torch.uint8, None, dev)
    _raise(lib().gptq_chmc_lowrank(_ptr(W), DTYPES[W.dtype], o, i, _ptr(H), int(tokens),
                                   float(lam), _ptr(Omega), int(r), int(niter), _ptr(Q),
                                   _ptr(P), _ptr(R), _ptr(info), _ptr(ws), ws.numel(),
                                   _stream(stream, dev)))


def gptq_check(info, stream=None) -> tuple[int, int]:
    """Synchronize the stream and return (status, index) from ``info``."""
    _need(info, "info", torch.int32, (2,))
    idx = C.c_int32(0)
    st = lib().gptq_check(_ptr(info), C.byref(idx), _stream(stream, info.device))
    if st == 6:
        _raise(st)
    return int(st), int(idx.value)


def gptq_peak_probe(kind: int, iters: int, info, sink, stream=None) -> float:
    """Launch one peak probe (0 float64, 1 TF32, 2 bf16) on ``stream``; returns
    the launch's floating-point operations (time it with CUDA events)."""
    _need(info, "info", torch.int32, (2,))
    _need(sink, "sink", torch.float64)
    flops = C.c_double(0.0)
    _raise(lib().gptq_peak_probe(int(kind), int(iters), C.byref(flops), _ptr(info), _ptr(sink),
                                 _stream(stream, info.device)))
    return float(flops.value)


def gptq_launch_count() -> int:
    return int(lib().gptq_launch_count())


def kernel_names() -> list[str]:
    L = lib()
    return [L.gptq_kernel_name(k).decode() for k in range(L.gptq_kernel_kinds())]


def gptq_profile_start(capacity: int = 1 << 16):
    _raise(lib().gptq_profile_start(int(capacity)))


def gptq_profile_stop() -> dict:
    """Stop timing; return {kernel name: (total ms, launches)}."""
    L = lib()
    _raise(L.gptq_profile_stop())
    out = {}
    for k, name in enumerate(kernel_names()):
        ms, cnt = C.c_double(0), C.c_int64(0)
        _raise(L.gptq_profile_get(k, C.byref(ms), C.byref(cnt)))
        out[name] = (ms.value, cnt.value)
    return out
