"""SSQR and HPTQ on the SmolLM-135M layer, in the launch configuration
bench.py times (its constants, its per-matrix lookahead), against the oracle.

Page: "The Geometry of LLM Quantization: GPTQ as Babai's Nearest Plane
Algorithm", §3.  Every matrix of the layer is quantized on the GPU from the
oracle's own preparation of its Hessian; the oracle then follows the GPU's
decisions at the α the GPU chose, row for row, with the tolerances of the
other SSQR/HPTQ tests, and checks the budget, the coded size and the CSR or
code table.  The search's own trace is compared step by step at smaller
sizes (test_gpu_ssqr.py, test_gpu_hptq.py); here its end point is checked:
within budget, and reproduced by the last pass.
"""
import numpy as np
import pytest
import torch

import bench
from oracle import gptq as og
from oracle import hptq as oh
from oracle import ssqr as osq
from workloads import problems_for

from . import parity as P

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _layer(bits):
    probs = problems_for(1, layer=0, bits=bits, order="act")
    most = max(-(-p.n // p.block) for p in probs)
    for p in probs:
        H = og.hessian(p.X.to(torch.float64).numpy())
        prep = og.prepare(H, p.damp, "act")
        U32 = prep["U"].astype(np.float32)
        gp = {"U": torch.from_numpy(U32).to(DEV),
              "perm": torch.from_numpy(prep["perm"].astype(np.int32)).to(DEV),
              "dead": torch.from_numpy(prep["dead"].astype(np.uint8)).to(DEV)}
        row0 = 0
        for name, rows in p.parts:
            W = p.W[row0:row0 + rows]
            row0 += rows
            Wz = W.to(torch.float64).numpy().copy()
            Wz[:, prep["dead"]] = 0.0
            yield name, p, W, prep, U32, gp, Wz, -(-p.n // p.block) == most


def test_ssqr_layer_in_the_bench_configuration():
    import post_weight_quantization_08_b200 as g
    for name, p, W, prep, U32, gp, Wz, look in _layer(bench.SSQR_BITS):
        m, n = W.shape
        q = g.ssqr_quantize(W.to(DEV), gp, bench.SSQR_BITS, p.group, p.block,
                            target=bench.SSQR_TARGET, iters=bench.SSQR_ITERS,
                            alpha_lo=bench.SSQR_LO, alpha_hi=bench.SSQR_HI, want_trace=True,
                            lookahead=look)
        torch.cuda.synchronize()
        alpha = np.float32(float(q["alpha"].cpu()[0]))
        nnz = int(q["row_ptr"][-1])
        assert nnz <= osq.max_outliers(bench.SSQR_TARGET, m, n), name
        tc = q["trace_count"].cpu().numpy()
        ta = q["trace_alpha"].cpu().numpy()
        assert [int(c) for a, c in zip(ta, tc) if c >= 0 and a == alpha][-1] == nnz, name
        codes = P.unpack_rows(q["qweight"].cpu().numpy(), bench.SSQR_BITS, n)
        mask = np.zeros((m, n), bool)
        vals = np.zeros((m, n))
        rp = q["row_ptr"].cpu().numpy()
        rows = np.repeat(np.arange(m), np.diff(rp))
        mask[rows, q["col_idx"].cpu().numpy()] = True
        vals[rows, q["col_idx"].cpu().numpy()] = q["val"].cpu().numpy()
        pm = prep["perm"]
        f = osq.follow_ssqr(Wz[:, pm], U32.astype(np.float64), bench.SSQR_BITS, p.group, p.block,
                            alpha, codes[:, pm], mask[:, pm], vals[:, pm],
                            q["scale"].cpu().numpy(), q["zero"].cpu().numpy().astype(np.float32))
        assert f["n_bad"] == 0 and f["z_bad"] == 0, (name, f)
        assert f["n_diff"] <= P.CODE_FRAC * m * n, (name, f)
        assert f["max_scale_rel"] <= P.SCALE_RTOL and f["max_val_rel"] <= 1e-5, (name, f)
        loss_or = float(np.sum(f["err"] ** 2))
        loss_gpu = float(q["loss_row"].cpu().to(torch.float64).sum())
        assert abs(loss_gpu - loss_or) <= P.LOSS_RTOL * loss_or, name


def test_hptq_layer_in_the_bench_configuration():
    import post_weight_quantization_08_b200 as g
    for name, p, W, prep, U32, gp, Wz, look in _layer(bench.HPTQ_BITS):
        m, n = W.shape
        q = g.hptq_quantize(W.to(DEV), gp, bench.HPTQ_BITS, p.group, p.block,
                            budget=bench.HPTQ_BUDGET, iters=bench.HPTQ_ITERS,
                            alpha_lo=bench.HPTQ_LO, alpha_hi=bench.HPTQ_HI, want_trace=True,
                            lookahead=look)
        torch.cuda.synchronize()
        alpha = np.float32(float(q["alpha"].cpu()[0]))
        nbits = int(q["row_off"][-1])
        assert nbits <= oh.max_bits(bench.HPTQ_BUDGET, m, n), name
        tb = q["trace_bits"].cpu().numpy()
        ta = q["trace_alpha"].cpu().numpy()
        assert [int(b) for a, b in zip(ta, tb) if b >= 0 and a == alpha][-1] == nbits, name
        codes = q["codes"].cpu().numpy().astype(np.int64)
        pm = prep["perm"]
        f = oh.follow_hptq(Wz[:, pm], U32.astype(np.float64), bench.HPTQ_BITS, p.group, p.block,
                           alpha, codes[:, pm], q["scale"].cpu().numpy())
        assert f["n_bad"] == 0 and f["n_diff"] <= P.CODE_FRAC * m * n, (name, f)
        assert f["max_scale_rel"] <= P.SCALE_RTOL, (name, f)
        loss_or = float(np.sum(f["err"] ** 2))
        loss_gpu = float(q["loss_row"].cpu().to(torch.float64).sum())
        assert abs(loss_gpu - loss_or) <= P.LOSS_RTOL * loss_or, name
        # the code is optimal for the GPU's histogram, and the stream is its encoding
        lens_all = q["code_len"].cpu().numpy().astype(np.int64)
        lens = {s - 2048: int(lens_all[s]) for s in np.nonzero(lens_all)[0]}
        hist = oh.histogram(codes)
        assert oh.cost(hist, lens) == oh.cost(hist, oh.huffman_lengths(hist)) == nbits, name
        ro_or, st_or = oh.encode(codes[:16], lens)
        st = q["stream"].cpu().numpy().view(np.uint32)
        assert np.array_equal(q["row_off"].cpu().numpy()[:17], ro_or)
        assert np.array_equal(st[:ro_or[-1] // 32], st_or[:ro_or[-1] // 32])
