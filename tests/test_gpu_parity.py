"""GPU parity: every stage of the CUDA path against the float64 oracle.

Sizes span several tiles and a ragged tail (n = 576 is 4½ groups of 128;
m = 300 is not a multiple of the 64-row CTA) and stay small enough for the
oracle to finish in seconds.  Edge cases: n = 1 / 8 / 64, m = 1 / 7, every bit
width, groups of 32/64/128, every order (min-pivot included), dead columns,
and the error paths.
"""
import numpy as np
import pytest
import torch

from oracle import gptq as og
from oracle import lattice as ol
from workloads import cone_activations, gaussian_weights, problems_for

from . import parity as P

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _layer(T, n, m, seed, wdtype=torch.bfloat16):
    X = cone_activations(T, n, seed).to(torch.bfloat16)
    W = gaussian_weights(m, n, seed + 1).to(wdtype)
    return X, W


def _full_check(X, W, bits, group, block, order="natural", damp=0.01, perm=None):
    out = P.run_gpu(X, W, bits, group, block, damp, order, perm, DEV)
    stats = P.check_hessian(X, out["H"])
    _, s2 = P.check_prepare(out["H"], out, damp, order, perm)
    stats.update(s2)
    stats.update(P.check_quantize(W, out, None, bits, group, block))
    stats.update(P.check_layer_loss(X, W, out, bits, group, block, damp, order, perm))
    Xf = X.to(torch.bfloat16).to(torch.float64).numpy()
    stats.update(P.check_rtn_dominance(W, out, og.hessian(Xf), bits, group))
    return out, stats


def test_single_layer_576():
    """The single-layer workload: 576×576 float32 W, 2048 cone tokens."""
    p = problems_for(0)[0]
    out, st = _full_check(p.X, p.W, 4, 128, 128)
    assert st["code_diff"] <= 1e-3 * st["codes"]


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_bits(bits):
    X, W = _layer(1024, 576, 300, 100 + bits)
    _full_check(X, W, bits, 128, 128)


@pytest.mark.parametrize("group,block", [(32, 32), (32, 128), (64, 64), (64, 128), (128, 128)])
def test_group_block(group, block):
    X, W = _layer(512, 320, 130, 7)
    _full_check(X, W, 4, group, block)


@pytest.mark.parametrize("order", ["natural", "act", "reverse", "minpivot"])
def test_orders(order):
    X, W = _layer(768, 448, 96, 11)
    _full_check(X, W, 4, 64, 128, order)


def _assert_min_pivot_sequence(Hd, perm, rtol=1e-10):
    """Along the elimination order (perm reversed) every step takes a smallest
    Schur-complement diagonal (float64, recomputed here), ties to the larger
    column."""
    S = np.array(Hd, dtype=np.float64, copy=True)
    n = len(perm)
    alive = np.ones(n, dtype=bool)
    assert sorted(perm.tolist()) == list(range(n))
    for t, j in enumerate(perm[::-1]):
        d = np.where(alive, np.diag(S), np.inf)
        assert alive[j] and d[j] <= d.min() + rtol * abs(d.min()), (t, j)
        alive[j] = False
        c = S[:, j].copy()
        S -= np.outer(c, c) / c[j]


@pytest.mark.parametrize("T,n,m", [(512, 40, 30), (768, 130, 50), (1024, 300, 64), (2048, 576, 96)])
def test_min_pivot_order(T, n, m):
    """The GPU's min-pivot order is a valid min-pivot sequence, equals the
    oracle's, and the rest of the path follows it to parity."""
    X, W = _layer(T, n, m, 21 + n)
    out = P.run_gpu(X, W, 4, 64, 128, 0.01, "minpivot", None, DEV)
    Hd, _, _ = og.damp_and_fix(out["H"].astype(np.float64), 0.01)
    _assert_min_pivot_sequence(Hd, out["perm"])
    _, st = P.check_prepare(out["H"], out, 0.01, "minpivot")
    st.update(P.check_quantize(W, out, None, 4, 64, 128))
    st.update(P.check_layer_loss(X, W, out, 4, 64, 128, 0.01, "minpivot"))


def test_min_pivot_identity_and_diagonal():
    """H = I gives the natural order; a diagonal H (ties included) gives act-order."""
    import post_weight_quantization_08_b200 as g
    n = 150
    p = g.prepare(torch.eye(n, device=DEV), 0.01, "minpivot")
    assert np.array_equal(p["perm"].cpu().numpy(), np.arange(n))
    d = torch.tensor(np.random.default_rng(5).choice([0.5, 1.0, 2.0, 4.0], size=n),
                     dtype=torch.float32)
    H = torch.diag(d).to(DEV)
    a = g.prepare(H, 0.01, "act")["perm"].cpu().numpy()
    b = g.prepare(H, 0.01, "minpivot")["perm"].cpu().numpy()
    assert np.array_equal(a, b)


@pytest.mark.parametrize("n", [1500, 3000])
def test_min_pivot_block_diagonal(n):
    """A block-diagonal H (blocks of 1–3 columns): every step of the GPU's order
    takes a smallest Schur diagonal, checked along the order with the blocks'
    own Schur complements (exact, cheap at any n).  n = 3000 runs the panel
    with its factor columns in global memory (they no longer fit in shared
    memory), n = 1500 with them in shared memory."""
    import post_weight_quantization_08_b200 as g
    rng = np.random.default_rng(n)
    sizes = []
    while sum(sizes) < n:
        sizes.append(int(min(rng.integers(1, 4), n - sum(sizes))))
    H = np.zeros((n, n))
    blocks, owner = [], np.empty(n, dtype=np.int64)
    c0 = 0
    for b, sz in enumerate(sizes):
        A = rng.standard_normal((sz, sz))
        B = A @ A.T + np.diag(rng.uniform(0.5, 2.0, sz))
        H[c0:c0 + sz, c0:c0 + sz] = B
        blocks.append([list(range(c0, c0 + sz)), B.copy()])
        owner[c0:c0 + sz] = b
        c0 += sz
    Ht = torch.tensor(H.astype(np.float32), device=DEV)
    perm = g.prepare(Ht, 0.0, "minpivot")["perm"].cpu().numpy()
    assert sorted(perm.tolist()) == list(range(n))
    # the float32 H the GPU saw, in float64, block by block
    H32 = H.astype(np.float32).astype(np.float64)
    for blk in blocks:
        cols = blk[0]
        blk[1] = H32[np.ix_(cols, cols)].copy()
    d = np.diag(H32).copy()
    alive = np.ones(n, dtype=bool)
    for t, j in enumerate(perm[::-1]):
        dm = np.where(alive, d, np.inf).min()
        assert alive[j] and d[j] <= dm + 1e-10 * abs(dm), (t, j, d[j], dm)
        cols, S = blocks[owner[j]]
        a = cols.index(j)
        c = S[:, a].copy()
        S -= np.outer(c, c) / c[a]
        alive[j] = False
        for q, col in enumerate(cols):
            if alive[col]:
                d[col] = S[q, q]


def test_min_pivot_not_positive_definite():
    """A negative pivot is met at the first elimination step: processed last."""
    import post_weight_quantization_08_b200 as g
    n = 90
    H = torch.eye(n, device=DEV)
    H[5, 5] = -1.0
    out = g.prepare(H, 0.0, "minpivot", check=False)
    st, idx = g.gptq_check(out["info"])
    assert st == 2 and idx == n


def test_custom_order():
    X, W = _layer(512, 200, 40, 12)
    perm = np.random.default_rng(0).permutation(200)
    _full_check(X, W, 3, 32, 64, "custom", perm=perm)


@pytest.mark.parametrize("m,n", [(1, 1), (7, 8), (1, 64), (7, 130), (65, 33)])
def test_small_and_ragged(m, n):
    X, W = _layer(256, n, m, 13 + m + n)
    _full_check(X, W, 4, 32, 64)


def test_float32_weights():
    X, W = _layer(512, 256, 70, 14, torch.float32)
    _full_check(X, W, 4, 128, 128)


def test_identity_hessian_is_rtn():
    """H = I (prepare fed directly): codes, scales and zeros equal RTN bit for bit."""
    import post_weight_quantization_08_b200 as g
    n, m = 300, 50
    W = gaussian_weights(m, n, 15)
    H = torch.eye(n, dtype=torch.float32, device=DEV)
    prep = g.prepare(H, 0.01, "natural")
    q = g.quantize(W.to(DEV), prep, 4, 64, 128)
    codes = P.unpack_rows(q["qweight"].cpu().numpy(), 4, n)
    c, s, z, _ = ol.rtn(W.double().numpy(), 4, 64)
    assert np.array_equal(codes, c)
    assert np.array_equal(q["scale"].cpu().numpy(), s)
    assert np.array_equal(q["zero"].cpu().numpy().astype(np.float32), z)


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_identity_hessian_is_rtn_streamed(bits):
    """The streamed ingest and pack (identity order, n a multiple of 32, no
    dequantized copy): with H = I, codes, scales and zeros equal RTN bit for bit."""
    import post_weight_quantization_08_b200 as g
    n, m = 512, 70
    W = gaussian_weights(m, n, 150 + bits)
    H = torch.eye(n, dtype=torch.float32, device=DEV)
    prep = g.prepare(H, 0.01, "natural")
    q = g.quantize(W.to(DEV), prep, bits, 128, 128, want_qdq=False)
    codes = P.unpack_rows(q["qweight"].cpu().numpy(), bits, n)
    c, s, z, _ = ol.rtn(W.double().numpy(), bits, 128)
    assert np.array_equal(codes, c)
    assert np.array_equal(q["scale"].cpu().numpy(), s)
    assert np.array_equal(q["zero"].cpu().numpy().astype(np.float32), z)


@pytest.mark.parametrize("order", ["natural", "act"])
@pytest.mark.parametrize("bits", [3, 4])
def test_pack_paths_agree(order, bits):
    """Asking for the dequantized copy switches the packer (and, for the
    natural order, nothing else) to its gathering path: the words agree."""
    import post_weight_quantization_08_b200 as g
    X, W = _layer(512, 576, 130, 30 + bits)
    H = g.hessian(X.to(DEV))
    prep = g.prepare(H, 0.01, order)
    a = g.quantize(W.to(DEV), prep, bits, 128, 128, want_qdq=False)
    b = g.quantize(W.to(DEV), prep, bits, 128, 128, want_qdq=True)
    for k in ("qweight", "scale", "zero", "g_idx", "loss_row"):
        assert torch.equal(a[k], b[k]), k


def test_dead_columns():
    X, W = _layer(300, 100, 20, 16)
    X[:, [3, 50]] = 0
    out, _ = _full_check(X, W, 4, 32, 64, "act")
    assert out["dead"][3] and out["dead"][50] and out["dead"].sum() == 2


def test_hessian_accumulates_across_calls():
    import post_weight_quantization_08_b200 as g
    X = cone_activations(1000, 200, 17).to(torch.bfloat16).to(DEV)
    H1 = g.hessian(X)
    H2 = g.hessian(X[:400].contiguous())
    g.hessian(X[400:].contiguous(), H2)
    torch.cuda.synchronize()
    ref = og.hessian(X.cpu().double().numpy())
    S = 2.0 * np.abs(X.cpu().double().numpy()).T @ np.abs(X.cpu().double().numpy())
    for H in (H1, H2):
        assert np.all(np.abs(H.cpu().double().numpy() - ref) <= 2 * 1000 * 2 ** -24 * S + 1e-30)
    # T = 0 is a no-op
    g.hessian(X[:0], H1)
    torch.cuda.synchronize()


def test_repeatable():
    X, W = _layer(512, 256, 64, 18)
    a = P.run_gpu(X, W, 4, 128, 128)
    b = P.run_gpu(X, W, 4, 128, 128)
    for k in ("H", "U", "qweight", "scale", "zero"):
        assert np.array_equal(a[k], b[k]), k


# ---------------------------------------------------------------- error paths

def test_not_positive_definite():
    import post_weight_quantization_08_b200 as g
    n = 70
    H = torch.eye(n, device=DEV)
    H[5, 5] = -4.0
    with pytest.raises(g.GptqError) as e:
        g.prepare(H, 0.0)
    assert e.value.status == 2


@pytest.mark.parametrize("n,col", [(70, 5), (200, 3), (200, 190), (130, 64)])
def test_not_positive_definite_index(n, col):
    """The reported index is the processing position of the first bad pivot.

    The factorisation runs on the reversed matrix, so the first pivot it meets
    is the last processed column; with natural order a single negative
    diagonal entry at `col` (and an identity elsewhere) is bad exactly there.
    """
    import post_weight_quantization_08_b200 as g
    H = torch.eye(n, device=DEV)
    H[col, col] = -1.0
    out = g.prepare(H, 0.0, "natural", check=False)
    st, idx = g.gptq_check(out["info"])
    assert st == 2 and idx == col + 1


def test_singular_block_is_not_positive_definite():
    """Two identical columns with no damping: the second pivot is exactly 0."""
    import post_weight_quantization_08_b200 as g
    n = 96
    H = torch.eye(n, device=DEV)
    H[10, 10] = H[11, 11] = H[10, 11] = H[11, 10] = 2.0
    out = g.prepare(H, 0.0, "natural", check=False)
    st, idx = g.gptq_check(out["info"])
    assert st == 2 and idx == 10 + 1


def test_nonfinite_inputs():
    import post_weight_quantization_08_b200 as g
    n = 40
    H = torch.eye(n, device=DEV)
    H[2, 7] = float("nan")
    with pytest.raises(g.GptqError) as e:
        g.prepare(H, 0.01)
    assert e.value.status == 3
    prep = g.prepare(torch.eye(n, device=DEV), 0.01)
    W = torch.zeros(4, n, device=DEV)
    W[1, 3] = float("inf")
    with pytest.raises(g.GptqError) as e:
        g.quantize(W, prep, 4, 32, 32)
    assert e.value.status == 3


def test_bad_custom_order():
    import post_weight_quantization_08_b200 as g
    n = 10
    perm = torch.arange(n, dtype=torch.int32, device=DEV)
    perm[3] = 4            # duplicate
    with pytest.raises(g.GptqError) as e:
        g.prepare(torch.eye(n, device=DEV), 0.01, "custom", perm=perm)
    assert e.value.status == 1


def test_host_side_argument_errors():
    import post_weight_quantization_08_b200 as g
    n = 64
    prep = g.prepare(torch.eye(n, device=DEV), 0.01)
    W = torch.randn(8, n, device=DEV)
    for bits, group, block in ((5, 32, 32), (4, 48, 96), (4, 64, 32), (4, 64, 256)):
        with pytest.raises(g.GptqError) as e:
            g.quantize(W, prep, bits, group, block)
        assert e.value.status == 4
    small = torch.empty(256, dtype=torch.uint8, device=DEV)
    with pytest.raises(g.GptqError) as e:
        g.quantize(W, prep, 4, 32, 32, ws=small)
    assert e.value.status == 1
