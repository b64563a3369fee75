"""gptq_prepare_noalloc: the prepare step for callers that cannot pass device
memory to the library (it uses a fixed scratch array inside the library).

Called through the C ABI and compared with gptq_prepare on the same inputs,
twice in a row with different problems, so that leftovers of the first call
in the shared scratch would show up in the second.  The second pair runs at the
size limit itself, where the scratch is used to its last byte, with the
min-pivot order first (it reuses the scratch's two float64 arrays for a
factorisation of its own before the regular one overwrites them).  Collected last (file
name) so that a run stopping at the first failure has run everything else.
"""
import ctypes as C

import numpy as np
import pytest
import torch

from workloads import cone_activations

from . import parity as P

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _noalloc(H, damp, order):
    from post_weight_quantization_08_b200 import _binding as b
    n = H.shape[0]
    perm = torch.empty(n, dtype=torch.int32, device=DEV)
    U = torch.empty(n, n, dtype=torch.float32, device=DEV)
    dead = torch.empty(n, dtype=torch.uint8, device=DEV)
    info = torch.zeros(2, dtype=torch.int32, device=DEV)
    stream = torch.cuda.current_stream(DEV).cuda_stream
    st = b.lib().gptq_prepare_noalloc(H.data_ptr(), n, float(damp), b.ORDERS[order],
                                      perm.data_ptr(), U.data_ptr(), dead.data_ptr(),
                                      info.data_ptr(), stream)
    assert st == 0, b.lib().gptq_last_error()
    idx = C.c_int32(0)
    assert b.lib().gptq_check(info.data_ptr(), C.byref(idx), stream) == 0
    return {"U": U.cpu().numpy(), "perm": perm.cpu().numpy().astype(np.int64),
            "dead": dead.cpu().numpy().astype(bool)}


def _with_workspace(H, damp, order):
    import post_weight_quantization_08_b200 as g
    p = g.prepare(H, damp, order)
    return {"U": p["U"].cpu().numpy(), "perm": p["perm"].cpu().numpy().astype(np.int64),
            "dead": p["dead"].cpu().numpy().astype(bool)}


def _hessian(T, n, seed):
    import post_weight_quantization_08_b200 as g
    X = cone_activations(T, n, seed).to(torch.bfloat16).to(DEV)
    return g.hessian(X)


@pytest.mark.parametrize("first,second", [((576, "act", 1), (320, "natural", 2)),
                                          ((1024, "minpivot", 3), (1024, "reverse", 4))])
def test_noalloc_matches_prepare_twice(first, second):
    for n, order, seed in (first, second):
        H = _hessian(1024, n, seed)
        got = _noalloc(H, 0.01, order)
        ref = _with_workspace(H, 0.01, order)
        assert np.array_equal(got["perm"], ref["perm"])
        assert np.array_equal(got["dead"], ref["dead"])
        # same kernels on the same data: equal within the U tolerance of the
        # other tests (in practice bit for bit)
        Hh = H.cpu().numpy()
        got.update(H=Hh)
        P.check_prepare(Hh, got, 0.01, order)
        assert np.array_equal(got["U"], ref["U"])


def test_noalloc_rejects_sizes_beyond_its_scratch():
    from post_weight_quantization_08_b200 import _binding as b
    n = 1025
    st = b.lib().gptq_prepare_noalloc(None, n, 0.01, 0, None, None, None, None, None)
    assert st == 1
    assert b"fixed scratch" in b.lib().gptq_last_error()
