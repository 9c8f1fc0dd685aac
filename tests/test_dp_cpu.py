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


# --------------------------------------------------------------------------- sharded AdaAlloc

SH_DOUT, SH_DIN, SH_N, SH_P = 97, 128, 64, 97 * 11 + 5  # odd d_out: uneven shards


def _sharded_weights():
    from workloads import rng_for

    g = rng_for(41, "sharded-init")
    w = (g.standard_normal((SH_DOUT, SH_DIN)) * 0.01).astype(np.float32)
    w[5] *= np.float32(300.0)  # a row that hits the cap d_in
    w[::9] = np.float32(0.0)  # empty-error rows
    return w


def _oracle_steps():
    """The three AdaAlloc steps of the oracle, on CPU torch tensors (what the library's steps are on the GPU)."""
    import oracle

    def norms(w):
        return torch.from_numpy(oracle.init_norms(w.numpy()))

    def budgets(e, d_in, p, min_per_row, mode):
        b, rp = oracle.init_budgets(e.numpy(), d_in, p, min_per_row, mode)
        return torch.from_numpy(b), torch.from_numpy(rp)

    def select(w, n, b, rp):
        ci, c = oracle.init_select(w.numpy(), n, b.numpy(), rp.numpy())
        return torch.from_numpy(ci), torch.from_numpy(c)

    return norms, budgets, select


def _sharded_worker(rank, world, port, mode, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import oracle
    from walsh_hadamard_sparse_b200.api import init_alloc_sharded, shard_rows

    oracle.set_threads(1)
    w = _sharded_weights()
    r0, r1 = shard_rows(SH_DOUT, rank, world)
    got = init_alloc_sharded(torch.from_numpy(w[r0:r1].copy()), SH_DOUT, SH_P, SH_N, 2, mode, steps=_oracle_steps())
    out[rank] = {k: v.numpy().copy() for k, v in got.items()}
    dist.barrier()
    dist.destroy_process_group()


def test_sharded_init_matches_single_process():
    """AdaAlloc sharded by output rows over 2 and 3 gloo ranks (norms exchanged in fp64, budgets computed on
    every rank, CSR slices gathered) gives every rank bit for bit the single-process result."""
    import oracle

    w = _sharded_weights()
    for world, mode in ((2, "fewest"), (3, "largest")):
        ref = oracle.init_alloc(w, SH_P, SH_N, 2, mode)
        assert ref["budgets"].max() == SH_DIN  # the cap is exercised
        port = _free_port()
        mgr = mp.Manager()
        out = mgr.dict()
        mp.spawn(_sharded_worker, args=(world, port, mode, out), nprocs=world, join=True)
        for r in range(world):
            got = out[r]
            for k in ("budgets", "row_ptr", "col_idx"):
                assert np.array_equal(got[k], ref[k]), (world, r, k)
            assert np.array_equal(got["coef"].view(np.uint32), ref["coef"].view(np.uint32)), (world, r)
