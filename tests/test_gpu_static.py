"""GPU parity of static-group GPTQ against the float64 oracle.

Static groups fix each group's scale and zero from the original weights of
consecutive original columns before the sweep; act-order then changes only
the order of the columns.  The GPU gets the oracle's own preparation.  The
parameters come from the original weights alone, so they must agree bit for
bit; the codes are checked in follow mode with the hot path's tolerances.
"""
import numpy as np
import pytest
import torch

from oracle import gptq as og
from oracle import static as ost
from workloads import cone_activations, gaussian_weights

from . import parity as P

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.mark.parametrize("m,n,bits,group,block,order,wdtype", [
    (300, 320, 4, 64, 128, "act", torch.float32),
    (128, 576, 3, 128, 128, "act", torch.bfloat16),
    (257, 96, 2, 32, 32, "natural", torch.float32),
    (50, 130, 4, 40, 64, "act", torch.float32),        # groups of 40 across blocks; SIMT trailing
    (64, 200, 8, 100, 96, "reverse", torch.float32),
    (576, 1536, 4, 128, 128, "act", torch.bfloat16),   # the SmolLM-135M down projection
])
def test_static_groups_match_oracle(m, n, bits, group, block, order, wdtype):
    import post_weight_quantization_08_b200 as g
    X = cone_activations(2048, n, 71).to(torch.bfloat16)
    W = gaussian_weights(m, n, 72).to(wdtype)
    H = og.hessian(X.to(torch.float64).numpy())
    prep = og.prepare(H, 0.01, order)
    U32 = prep["U"].astype(np.float32)
    gp = {"U": torch.from_numpy(U32).to(DEV),
          "perm": torch.from_numpy(prep["perm"].astype(np.int32)).to(DEV),
          "dead": torch.from_numpy(prep["dead"].astype(np.uint8)).to(DEV)}
    q = g.quantize(W.to(DEV), gp, bits, group, block, want_loss=True, want_qdq=True,
                   static_groups=True)
    torch.cuda.synchronize()
    Wz = W.to(torch.float64).numpy().copy()
    Wz[:, prep["dead"]] = 0.0
    scale_or, zero_or = ost.static_params(Wz, bits, group)
    scale = q["scale"].cpu().numpy()
    zero = q["zero"].cpu().numpy().astype(np.float32)
    assert np.array_equal(scale, scale_or) and np.array_equal(zero, zero_or)
    assert np.array_equal(q["g_idx"].cpu().numpy(), np.arange(n) // group)
    codes = P.unpack_rows(q["qweight"].cpu().numpy(), bits, n)
    perm = prep["perm"]
    f = ost.follow_static(Wz[:, perm], U32.astype(np.float64), bits, perm // group, scale,
                          zero, block, codes[:, perm])
    assert f["n_bad"] == 0 and f["n_diff"] <= P.CODE_FRAC * m * n, f
    loss_or = float(np.sum(f["err"] ** 2))
    loss_gpu = float(q["loss_row"].cpu().to(torch.float64).sum())
    assert abs(loss_gpu - loss_or) <= P.LOSS_RTOL * loss_or
    gi = np.arange(n) // group
    want = scale[:, gi] * (codes.astype(np.float32) - zero[:, gi])
    assert np.allclose(q["Qdq"].cpu().numpy(), want, rtol=0, atol=1e-7 * np.abs(want).max())


def test_identity_hessian_is_rtn_in_act_order():
    """H = I on the GPU: act-order permutes the columns, static groups keep
    the round-to-nearest of the original groups, bit for bit."""
    import post_weight_quantization_08_b200 as g
    from oracle import lattice as ol
    m, n = 40, 300
    W = gaussian_weights(m, n, 73)
    d = torch.linspace(2.0, 0.5, n)[torch.randperm(n, generator=torch.Generator().manual_seed(1))]
    prep = g.prepare(torch.diag(d).to(DEV), 0.01, "act")
    q = g.quantize(W.to(DEV), prep, 4, 64, 128, static_groups=True)
    torch.cuda.synchronize()
    codes, scale, zero, _ = ol.rtn(W.to(torch.float64).numpy(), 4, 64)
    assert np.array_equal(P.unpack_rows(q["qweight"].cpu().numpy(), 4, n), codes)
    assert np.array_equal(q["scale"].cpu().numpy(), scale)


def test_argument_errors():
    import post_weight_quantization_08_b200 as g
    W = gaussian_weights(64, 64, 74).to(DEV)
    prep = g.prepare(torch.eye(64, device=DEV) * 2.0)
    with pytest.raises(g.GptqError):
        g.quantize(W, prep, 4, 0, 64, static_groups=True)
    with pytest.raises(g.GptqError):
        g.quantize(W, prep, 4, 32, 48, static_groups=True)
