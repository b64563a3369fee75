"""Host-side logic of the CHMC entry points (no GPU needed).

The rank rule is host arithmetic in the library; it must agree with the
oracle's brute-force-pinned rule.  Argument errors are raised before any
device work.
"""
import ctypes as C

import pytest

from oracle import chmc as oc


def _lib():
    from post_weight_quantization_08_b200 import _binding as b
    return b.lib()


@pytest.mark.parametrize("o,i,bits,gs,tgt", [
    (576, 576, 4, 128, 4.2875), (1536, 576, 4, 128, 4.2875), (576, 1536, 4, 128, 4.2875),
    (192, 576, 4, 128, 4.2875), (896, 4864, 4, 128, 4.2875), (4864, 896, 4, 128, 4.2875),
    (2048, 5632, 4, 128, 4.2875), (64, 64, 3, 32, 3.6), (128, 128, 4, 128, 4.0),
    (10, 10, 2, 4, 9.0)])
def test_rank_rule_matches_oracle(o, i, bits, gs, tgt):
    assert _lib().gptq_chmc_rank(o, i, bits, gs, tgt) == oc.chmc_rank(o, i, bits, gs, tgt)


def test_workspace_bytes():
    L = _lib()
    assert L.gptq_chmc_workspace_bytes(576, 576, 2) > 0
    assert L.gptq_chmc_workspace_bytes(576, 576, 33) == 0
    assert L.gptq_chmc_workspace_bytes(0, 576, 2) == 0
    assert L.gptq_chmc_workspace_bytes(576, 576, 0) > 0


def test_argument_errors_before_device_work():
    L = _lib()
    buf = (C.c_uint8 * 1024)()
    p = C.cast(buf, C.c_void_p)
    # null W
    assert L.gptq_chmc_lowrank(None, 0, 8, 8, p, 16, 0.05, p, 2, 5, None, None, p, p, p,
                               1024, None) == 1
    # rank above the limit
    assert L.gptq_chmc_lowrank(p, 0, 64, 64, p, 16, 0.05, p, 33, 5, None, None, p, p, p,
                               1024, None) == 4
    # rank above min(o, i)
    assert L.gptq_chmc_lowrank(p, 0, 8, 4, p, 16, 0.05, p, 5, 5, None, None, p, p, p,
                               1024, None) == 4
    # gs other than the CTA's rows
    assert L.gptq_quantize_rowgroups(p, 0, 8, 8, p, p, p, 4, 64, 64, p, p, p, None, None, p,
                                     p, 1 << 20, None) == 4
