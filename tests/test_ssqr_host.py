"""Host-side checks of the SSQR entry point (no GPU needed).

Every argument error is found on the host and returned before anything is
enqueued, so these calls run here with host buffers standing in for device
pointers (none of them is dereferenced).
"""
import ctypes as C

import pytest

from oracle import ssqr as osq


def _lib():
    from post_weight_quantization_08_b200 import _binding as b
    return b.lib()


def _call(L, p, **kw):
    a = dict(W=p, dtype=0, m=64, n=64, U=p, perm=p, dead=p, bits=3, group=32, block=64,
             target=0.01, iters=8, lo=1.0 / 16, hi=1.0, la=1, qweight=p, scale=p, zero=p, g_idx=p,
             row_ptr=p, col_idx=p, val=p, cap=16, alpha=p, ta=None, tc=None, loss=None,
             qdq=None, info=p, ws=p, ws_bytes=1 << 30)
    a.update(kw)
    return L.gptq_ssqr_quantize(a["W"], a["dtype"], a["m"], a["n"], a["U"], a["perm"],
                                a["dead"], a["bits"], a["group"], a["block"], a["target"],
                                a["iters"], a["lo"], a["hi"], a["la"], a["qweight"], a["scale"],
                                a["zero"], a["g_idx"], a["row_ptr"], a["col_idx"], a["val"],
                                a["cap"], a["alpha"], a["ta"], a["tc"], a["loss"], a["qdq"],
                                a["info"], a["ws"], a["ws_bytes"], None)


@pytest.mark.parametrize("kw,status", [
    ({"W": None}, 1),                       # null pointer
    ({"row_ptr": None}, 1),
    ({"col_idx": None}, 1),                 # a capacity without arrays
    ({"bits": 8}, 4),                       # no room for the outlier flag
    ({"bits": 5}, 4),
    ({"target": 1.5}, 1),
    ({"target": -0.1}, 1),
    ({"target": float("nan")}, 1),
    ({"iters": -1}, 1),
    ({"iters": 65}, 1),
    ({"lo": 0.0}, 1),
    ({"lo": 0.5, "hi": 0.25}, 1),
    ({"hi": 17.0}, 1),
    ({"cap": -1}, 1),
    ({"group": 48}, 4),                     # the hot path's group rule
    ({"ws_bytes": 16}, 1),
])
def test_argument_errors_before_device_work(kw, status):
    L = _lib()
    buf = (C.c_uint8 * 4096)()
    p = C.cast(buf, C.c_void_p)
    # a 256-byte aligned stand-in for the workspace
    ws = C.c_void_p((p.value + 255) // 256 * 256)
    kw.setdefault("ws", ws)
    assert _call(L, p, **kw) == status


def test_workspace_adds_the_search_state_to_gptq():
    L = _lib()
    for m, n, b in [(576, 576, 128), (1, 40, 32), (4864, 896, 128)]:
        assert L.gptq_ssqr_workspace_bytes(m, n, b) > L.gptq_quantize_workspace_bytes(m, n, b)
    assert L.gptq_ssqr_workspace_bytes(0, 10, 32) == 0


def test_budget_rule_matches_the_oracle():
    """The library computes floor(target·m·n) in double on the host exactly
    as the oracle does; spot-check the oracle's values the GPU tests rely on."""
    assert osq.max_outliers(0.01, 576, 576) == 3317
    assert osq.max_outliers(0.005, 192, 576) == 552
    assert osq.max_outliers(0.02, 300, 260) == 1560
