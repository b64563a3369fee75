"""CPU checks of the C ABI: the library loads, exports every declared symbol,
and rejects bad arguments on the host before touching the GPU."""
import ctypes as C
import os
import re

import pytest

from post_weight_quantization_08_b200 import _binding
from post_weight_quantization_08_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(_binding.LIB_PATH):
        build()
    return _binding.lib()


def _declared():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            src = open(os.path.join(ROOT, "include", f)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(gptq_\w+)\s*\(", src))
    return names


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert {"gptq_hessian_accumulate", "gptq_prepare", "gptq_quantize", "gptq_check"} <= names
    for n in names:
        assert hasattr(lib, n), n
    assert names == set(_binding.exported_symbols())


def test_status_strings(lib):
    assert lib.gptq_status_string(0) == b"GPTQ_OK"
    assert lib.gptq_status_string(4) == b"GPTQ_ERR_UNSUPPORTED"
    assert lib.gptq_kernel_kinds() >= 10
    assert lib.gptq_kernel_name(0) == b"hessian"


def test_workspace_sizes(lib):
    assert lib.gptq_prepare_workspace_bytes(0) == 0
    b = lib.gptq_prepare_workspace_bytes(576)
    assert b >= 2 * 576 * 576 * 8 and b % 256 == 0
    q = lib.gptq_quantize_workspace_bytes(100, 576, 128)
    assert q >= 100 * 576 * 5 + 100 * 128 * 4 and q % 256 == 0


FAKE = C.c_void_p(0x100000)   # never dereferenced: validation returns first


def test_host_validation_without_gpu(lib):
    # null pointers
    assert lib.gptq_hessian_accumulate(None, 10, 10, None, None, None) == 1
    assert lib.gptq_hessian_accumulate(FAKE, -1, 10, FAKE, None, None) == 1
    assert lib.gptq_prepare(None, 10, 0.01, 0, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 30, None) == 1
    assert lib.gptq_prepare(FAKE, 10, -1.0, 0, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 30, None) == 1
    assert lib.gptq_prepare(FAKE, 10, 0.01, 9, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 30, None) == 1
    assert lib.gptq_prepare(FAKE, 10, 0.01, 0, FAKE, FAKE, FAKE, FAKE, FAKE, 8, None) == 1

    def q(bits=4, group=128, block=128, ws_bytes=1 << 30, m=16, n=256, dtype=1):
        return lib.gptq_quantize(FAKE, dtype, m, n, FAKE, FAKE, FAKE, bits, group, block,
                                 FAKE, FAKE, FAKE, FAKE, None, None, FAKE, FAKE,
                                 ws_bytes, None)
    assert q(bits=5) == 4 and q(bits=1) == 4
    assert q(group=48, block=96) == 4
    assert q(group=64, block=32) == 4
    assert q(block=256) == 4
    assert q(ws_bytes=16) == 1
    assert q(dtype=7) == 1
    assert q(m=0) == 1
    assert b"bits" in lib.gptq_last_error() or b"m=" in lib.gptq_last_error()
    assert lib.gptq_check(None, None, None) == 1
