"""GPU parity of the CHMC frontend against the float64 oracle.

Page: "Warum Geometrie Gewichte nicht komprimiert", "Methodik. Was ist CHMC".
Every input handed to the GPU here is computed on the host (the oracle's
Hessian and inverse-Cholesky factor, rounded to float32 where the library takes
float32), so the oracle never sees a value that came from the CUDA path.

Tolerances (from the arithmetic of each side):
  * low-rank stage: both sides run the same float64 iteration from the same Ω;
    R differs by its float32 rounding (2⁻²³·|R|) plus 1e-9·max|W|.
  * residual quantization: the hot path's criterion (codes within 1e-4 code
    units of a rounding boundary, at most 0.1 %; scales 1e-5 relative; loss
    1e-3 relative).
"""
import numpy as np
import pytest
import torch

from oracle import chmc as oc
from oracle import gptq as og
from workloads import cone_activations, gaussian_weights, normal_matrix, spectral_weights

from . import parity as P

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _g():
    import post_weight_quantization_08_b200 as g
    return g


@pytest.mark.parametrize("o,i,r,wdtype", [
    (300, 200, 5, torch.float32),      # ragged 128-row chunks
    (576, 576, 2, torch.bfloat16),     # a SmolLM-135M attention projection, rank from the rule
    (130, 260, 32, torch.float32),     # the largest rank
    (1536, 576, 4, torch.bfloat16),    # gate/up shape, rank from the rule
])
def test_lowrank_matches_oracle(o, i, r, wdtype):
    g = _g()
    T = 512
    X = cone_activations(T, i, 11).to(torch.bfloat16)
    W = spectral_weights(o, i, 12).to(wdtype)
    H = torch.from_numpy(og.hessian(X.to(torch.float64).numpy())).to(torch.float32)
    Om = normal_matrix(i, r, 13)
    out = g.chmc_lowrank(W.to(DEV), H.to(DEV), T, Om.to(DEV), r, lam=0.05, niter=5)
    torch.cuda.synchronize()
    Wf = W.to(torch.float64).numpy()
    c = oc.activation_energy_from_hessian(H.to(torch.float64).numpy(), T, 0.05)
    lr = oc.weighted_lowrank(Wf, c, Om.to(torch.float64).numpy(), 5)
    R_or = Wf - lr["Wlr"]
    R = out["R"].cpu().to(torch.float64).numpy()
    tol = 2.0 ** -23 * np.abs(R_or) + 1e-9 * np.abs(Wf).max()
    assert np.all(np.abs(R - R_or) <= tol), float(np.max(np.abs(R - R_or) / tol))
    Q = out["Q"].cpu().to(torch.float64).numpy()
    Pm = out["P"].cpu().to(torch.float64).numpy()
    assert np.allclose(Q.T @ Q, np.eye(r), atol=1e-5)
    assert np.abs(Q @ Pm - lr["Wlr"]).max() <= 1e-6 * np.abs(Wf).max()


def test_lowrank_rank_zero_copies_w():
    g = _g()
    W = gaussian_weights(70, 90, 3)
    out = g.chmc_lowrank(W.to(DEV), None, 16, None, 0)
    assert torch.equal(out["R"].cpu(), W)


def test_lowrank_of_an_exactly_low_rank_matrix_leaves_no_residual():
    """rank(W) = 3 < r = 6: the sketch reaches the whole range; the Cholesky
    step drops the directions it cannot reach, and R vanishes."""
    g = _g()
    A = normal_matrix(200, 3, 21).to(torch.float64)
    B = normal_matrix(3, 150, 22).to(torch.float64)
    W = (0.01 * A @ B).to(torch.float32)
    X = cone_activations(256, 150, 23).to(torch.bfloat16)
    H = torch.from_numpy(og.hessian(X.to(torch.float64).numpy())).to(torch.float32)
    out = g.chmc_lowrank(W.to(DEV), H.to(DEV), 256, normal_matrix(150, 6, 24).to(DEV), 6)
    assert float(out["R"].abs().max()) <= 1e-6 * float(W.abs().max())


@pytest.mark.parametrize("m,n,bits,block,order", [
    (300, 320, 4, 128, "act"),       # 3 row groups (the last partial), 2½ blocks
    (128, 576, 4, 128, "act"),       # one row group, 4½ blocks
    (257, 96, 3, 32, "natural"),     # a group of one row at the end
    (64, 200, 2, 64, "reverse"),
    (1, 40, 8, 32, "natural"),       # one row
])
def test_quantize_rowgroups_matches_oracle(m, n, bits, block, order):
    g = _g()
    T = 256
    X = cone_activations(T, n, 31).to(torch.bfloat16)
    W = gaussian_weights(m, n, 32)
    H = og.hessian(X.to(torch.float64).numpy())
    prep = og.prepare(H, 0.01, order)
    U32 = prep["U"].astype(np.float32)
    gp = {"U": torch.from_numpy(U32).to(DEV),
          "perm": torch.from_numpy(prep["perm"].astype(np.int32)).to(DEV),
          "dead": torch.from_numpy(prep["dead"].astype(np.uint8)).to(DEV)}
    q = g.quantize_rowgroups(W.to(DEV), gp, bits, 128, block, want_loss=True, want_qdq=True)
    torch.cuda.synchronize()
    codes = P.unpack_rows(q["qweight"].cpu().numpy(), bits, n)
    scale = q["scale"].cpu().numpy()
    zero = q["zero"].cpu().numpy().astype(np.float32)
    perm = prep["perm"]
    Wz = W.to(torch.float64).numpy().copy()
    Wz[:, prep["dead"]] = 0.0
    f = oc.follow_rowgroups(Wz[:, perm], U32.astype(np.float64), bits, 128, block,
                            codes[:, perm], scale[:, perm], zero[:, perm])
    assert f["n_bad"] == 0 and f["z_bad"] == 0, f
    assert f["n_diff"] <= P.CODE_FRAC * m * n, f
    assert f["z_diff"] <= P.ZERO_FRAC * zero.size, f
    assert f["max_scale_rel"] <= P.SCALE_RTOL, f
    loss_or = float(np.sum(f["err"] ** 2))
    loss_gpu = float(q["loss_row"].cpu().to(torch.float64).sum())
    # relative, with a floor for layers quantized almost exactly (one row:
    # every value sits on its own grid's endpoint, the loss is rounding noise)
    assert abs(loss_gpu - loss_or) <= P.LOSS_RTOL * loss_or + 1e-10 * float(np.sum(Wz ** 2))
    # the dequantized copy is s·(q − z) of the library's own outputs
    rows = np.arange(m) // 128
    want = scale[rows, :] * (codes.astype(np.float32) - zero[rows, :])
    assert np.allclose(q["Qdq"].cpu().numpy(), want, rtol=0, atol=1e-7 * np.abs(want).max())


def test_chmc_layer_end_to_end():
    """X → Hessian → low-rank part → inverse-Cholesky → residual GPTQ on the
    GPU against the oracle's chmc_layer from X alone: layer loss to 1e-3."""
    g = _g()
    T, o, i = 2048, 576, 576
    X = cone_activations(T, i, 41).to(torch.bfloat16)
    W = spectral_weights(o, i, 42)
    r = g.gptq_chmc_rank(o, i, 4, 128, 4.2875)
    assert r == oc.chmc_rank(o, i, 4, 128, 4.2875)
    Om = normal_matrix(i, r, 43)
    H = g.hessian(X.to(DEV))
    out = g.chmc_layer(W.to(DEV), H, T, Om.to(DEV), r=r, damp=0.05)
    torch.cuda.synchronize()
    Wc = (out["Q"].double() @ out["P"].double() + out["Qdq"].double()).cpu().numpy()
    Hx = og.hessian(X.to(torch.float64).numpy())
    ref = oc.chmc_layer(W.to(torch.float64).numpy(), Hx, T, Om.to(torch.float64).numpy(),
                        rank=r, damp=0.05)
    loss_gpu = og.layer_loss(W.to(torch.float64).numpy(), Wc, Hx)
    assert abs(loss_gpu - ref["loss"]) <= P.LOSS_RTOL * ref["loss"], (loss_gpu, ref["loss"])


def test_errors():
    g = _g()
    W = gaussian_weights(64, 64, 5).to(DEV)
    with pytest.raises(g.GptqError):
        g.chmc_lowrank(W, torch.zeros(64, 64, device=DEV), 16, torch.zeros(64, 40, device=DEV), 40)
    prep = g.prepare(torch.eye(64, device=DEV) * 2.0)
    with pytest.raises(g.GptqError):
        g.quantize_rowgroups(W, prep, 4, 64, 64)
