"""Host-side checks of gptq_quantize_static (no GPU needed): argument errors
are returned before anything is enqueued."""
import ctypes as C

import pytest


def _lib():
    from post_weight_quantization_08_b200 import _binding as b
    return b.lib()


@pytest.mark.parametrize("kw,status", [
    ({"W": None}, 1), ({"g_idx": None}, 1), ({"group": 0}, 4), ({"block": 48}, 4),
    ({"block": 160}, 4), ({"bits": 5}, 4), ({"ws_bytes": 16}, 1),
])
def test_argument_errors_before_device_work(kw, status):
    L = _lib()
    buf = (C.c_uint8 * 4096)()
    p = C.cast(buf, C.c_void_p)
    ws = C.c_void_p((p.value + 255) // 256 * 256)
    a = dict(W=p, dtype=0, m=64, n=64, U=p, perm=p, dead=p, bits=4, group=40, block=64,
             qweight=p, scale=p, zero=p, g_idx=p, loss=None, qdq=None, info=p, ws=ws,
             ws_bytes=1 << 30)
    a.update(kw)
    assert L.gptq_quantize_static(a["W"], a["dtype"], a["m"], a["n"], a["U"], a["perm"],
                                  a["dead"], a["bits"], a["group"], a["block"], a["qweight"],
                                  a["scale"], a["zero"], a["g_idx"], a["loss"], a["qdq"],
                                  a["info"], a["ws"], a["ws_bytes"], None) == status
