"""Host-side checks of the HPTQ entry point (no GPU needed).

Every argument error is found on the host and returned before anything is
enqueued, so these calls run here with host buffers standing in for device
pointers (none of them is dereferenced).
"""
import ctypes as C

import pytest

from oracle import hptq as oh


def _lib():
    from post_weight_quantization_08_b200 import _binding as b
    return b.lib()


def _call(L, p, **kw):
    a = dict(W=p, dtype=0, m=64, n=64, U=p, perm=p, dead=p, bits=4, group=32, block=64,
             budget=3.125, iters=8, lo=1.0 / 16, hi=16.0, la=1, codes=None, scale=p,
             g_idx=p, code_len=p, code_word=None, row_off=p, stream=p, cap=64, alpha=p,
             ta=None, tb=None, loss=None, qdq=None, info=p, ws=p, ws_bytes=1 << 30)
    a.update(kw)
    return L.gptq_hptq_quantize(a["W"], a["dtype"], a["m"], a["n"], a["U"], a["perm"],
                                a["dead"], a["bits"], a["group"], a["block"], a["budget"],
                                a["iters"], a["lo"], a["hi"], a["la"], a["codes"], a["scale"],
                                a["g_idx"], a["code_len"], a["code_word"], a["row_off"],
                                a["stream"], a["cap"], a["alpha"], a["ta"], a["tb"], a["loss"],
                                a["qdq"], a["info"], a["ws"], a["ws_bytes"], None)


@pytest.mark.parametrize("kw,status", [
    ({"W": None}, 1),
    ({"code_len": None}, 1),
    ({"row_off": None}, 1),
    ({"stream": None}, 1),                  # a capacity without a stream
    ({"bits": 5}, 4),
    ({"budget": 0.0}, 1),
    ({"budget": 65.0}, 1),
    ({"budget": float("nan")}, 1),
    ({"iters": 65}, 1),
    ({"lo": 0.0}, 1),
    ({"lo": 2.0, "hi": 1.0}, 1),
    ({"hi": 300.0}, 1),
    ({"cap": -1}, 1),
    ({"group": 48}, 4),
    ({"ws_bytes": 16}, 1),
])
def test_argument_errors_before_device_work(kw, status):
    L = _lib()
    buf = (C.c_uint8 * 4096)()
    p = C.cast(buf, C.c_void_p)
    ws = C.c_void_p((p.value + 255) // 256 * 256)
    kw.setdefault("ws", ws)
    assert _call(L, p, **kw) == status


def test_workspace_adds_codes_and_tables_to_gptq():
    L = _lib()
    for m, n, b in [(576, 576, 128), (1, 40, 32), (4864, 896, 128)]:
        extra = L.gptq_hptq_workspace_bytes(m, n, b) - L.gptq_quantize_workspace_bytes(m, n, b)
        assert extra >= 2 * m * n + 8 * 4096 * 2 + 4096
    assert L.gptq_hptq_workspace_bytes(0, 10, 32) == 0


def test_budget_rule_matches_the_oracle():
    assert oh.max_bits(3.125, 576, 576) == 1036800
    assert oh.max_bits(2.5, 192, 576) == 276480
