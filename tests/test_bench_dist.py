"""Host logic of the multi-GPU bench on CPU: world-size-2 gloo ranks.

Every rank quantizes its own layer (seed block = rank); the device times are
combined as a max over ranks and the parameter counts as a sum.  No data-path
collective exists, so these helpers are the whole multi-process surface.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from workloads import problems_for


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, w, lr = bench.dist_env()
        assert (r, w, lr) == (rank, world, rank)
        layer = bench.layer_for_rank(r)
        t = bench.max_over_ranks(10.0 + rank, w)
        p = bench.sum_over_ranks(100.0 * (rank + 1), w)
        probs = problems_for(0, layer=layer)
        first = float(probs[0].W[0, 0])
        out[rank] = (layer, t, p, first)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    port = _free_port()
    with mp.Manager() as man:
        out = man.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == 0 and res[1][0] == 1            # own layers
    assert res[0][1] == res[1][1] == 11.0                # max over ranks
    assert res[0][2] == res[1][2] == 300.0               # sum over ranks
    assert res[0][3] != res[1][3]                        # different seeded weights


def test_single_rank_helpers_are_identity():
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.sum_over_ranks(2.0, 1) == 2.0


def test_kernel_work_accounting():
    probs = problems_for(1)
    work = bench.kernel_work(probs, 128)
    T = probs[0].T
    n0, n1 = probs[0].n, probs[1].n
    assert work["hessian"][1] == T * n0 * (n0 + 1) + T * n1 * (n1 + 1)
    # float64 tile work approaches 2n³/3 from above (tiles are 64 wide)
    tiles = work["cholesky"][1]
    assert 0.9 * (2 * (n0 ** 3 + n1 ** 3) / 3) < tiles < 1.6 * (2 * (n0 ** 3 + n1 ** 3) / 3)
    assert work["sweep"][0] == "GB/s"


def test_workload_name_names_sizes():
    name = bench.workload_name(1, 4)
    assert "4608x576" in name and "576x1536" in name and "T=2048" in name
