"""The device time-out path of the dataflow factorisation.

gptq_prepare's Cholesky is one launch whose CTAs wait on each other's tiles
through flags; every wait is bounded.  With the poll limit lowered to one
poll, a worker that finds its input tile not yet final gives up at once: the
launch reports GPTQ_ERR_TIMEOUT through `info`, raises its abort flag, every
CTA returns, and the context stays usable.  Nothing here can wait forever:
the failing waits are the bounded ones, and the limit is restored before the
normal call that follows, which must pass parity.
"""
import ctypes as C

import numpy as np
import pytest
import torch

from workloads import cone_activations

from . import parity as P

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
GPTQ_ERR_TIMEOUT = 5


def _prepare_raw(H, order=0):
    import post_weight_quantization_08_b200 as g
    from post_weight_quantization_08_b200 import _binding as b
    n = H.shape[0]
    perm = torch.empty(n, dtype=torch.int32, device=DEV)
    U = torch.empty(n, n, dtype=torch.float32, device=DEV)
    dead = torch.empty(n, dtype=torch.uint8, device=DEV)
    info = torch.zeros(2, dtype=torch.int32, device=DEV)
    ws = g.workspace(b.lib().gptq_prepare_workspace_bytes(n), torch.device(DEV))
    stream = torch.cuda.current_stream(DEV).cuda_stream
    st = b.lib().gptq_prepare(H.data_ptr(), n, 0.01, order, perm.data_ptr(), U.data_ptr(),
                              dead.data_ptr(), info.data_ptr(), ws.data_ptr(), ws.numel(),
                              stream)
    assert st == 0, b.lib().gptq_last_error()
    idx = C.c_int32(0)
    st = b.lib().gptq_check(info.data_ptr(), C.byref(idx), stream)
    return st, idx.value, {"U": U, "perm": perm, "dead": dead}


def test_wait_time_out_is_reported_and_the_context_survives():
    import post_weight_quantization_08_b200 as g
    from post_weight_quantization_08_b200 import _binding as b
    n = 2048            # 32×32 tiles: workers start long before the chain's first tile is final
    X = cone_activations(2048, n, 77).to(torch.bfloat16).to(DEV)
    H = g.hessian(X)
    try:
        b.lib().gptq_set_wait_limit(1)
        st, idx, _ = _prepare_raw(H)
    finally:
        b.lib().gptq_set_wait_limit(0)
    assert st == GPTQ_ERR_TIMEOUT, (st, b.lib().gptq_status_string(st))
    assert idx >= 1                      # the awaited flag value + 1
    torch.cuda.synchronize()
    # the same call with the default limit succeeds and matches the oracle
    st, _, out = _prepare_raw(H)
    assert st == 0, b.lib().gptq_status_string(st)
    Hh = H.cpu().numpy()
    res = {"U": out["U"].cpu().numpy(), "perm": out["perm"].cpu().numpy().astype(np.int64),
           "dead": out["dead"].cpu().numpy().astype(bool)}
    P.check_prepare(Hh, res, 0.01, "natural")
