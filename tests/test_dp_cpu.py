"""Token data parallelism of the layer on CPU ranks (gloo, world size 2).

Each rank takes its own token rows (workloads.rank_rows, as bench.py does), computes
its coefficient gradient with the oracle, and the ranks sum them with all_reduce: the
result must equal the gradient over all tokens at once (dc is a sum over tokens), and
dX/Y of each rank must equal the rows of the single-process result."""

import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

D_IN, D_OUT, N, T_RANK, P = 64, 48, 32, 6, 48 * 5


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _layer():
    from workloads import random_pattern, rng_for

    g = rng_for(40, "dp")
    rp, ci, cf = random_pattern(D_OUT, D_IN, p=P, rng=g)
    X = g.standard_normal((2 * T_RANK, D_IN))
    dY = g.standard_normal((2 * T_RANK, D_OUT))
    return rp, ci, cf, X, dY


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import oracle
    from workloads import rank_rows

    oracle.set_threads(1)
    rp, ci, cf, X, dY = _layer()
    rows = rank_rows(rank, T_RANK)
    dc = oracle.adapter_bwd_dc(X[rows], dY[rows], oracle.csr_rows(rp), ci, N)
    t = torch.from_numpy(dc)
    dist.all_reduce(t)
    dX = oracle.adapter_bwd_dx(rp, ci, cf, dY[rows], D_IN, N)
    out[rank] = (t.numpy().copy(), dX)
    dist.barrier()
    dist.destroy_process_group()


def test_dp_allreduce_of_dc_matches_single_process():
    import oracle

    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
    rp, ci, cf, X, dY = _layer()
    dc_all = oracle.adapter_bwd_dc(X, dY, oracle.csr_rows(rp), ci, N)
    dX_all = oracle.adapter_bwd_dx(rp, ci, cf, dY, D_IN, N)
    for r in range(2):
        dc_r, dX_r = out[r]
        assert np.allclose(dc_r, dc_all, rtol=1e-12, atol=1e-12)
        assert np.allclose(dX_r, dX_all[r * T_RANK:(r + 1) * T_RANK], rtol=1e-12, atol=1e-12)
