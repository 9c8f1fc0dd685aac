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


# --------------------------------------------------------------------------- the package's data-parallel step


def _oracle_layer_steps(log):
    """adapter_fwd / adapter_bwd of the oracle on CPU tensors, with the signatures of the package's functions; every
    call is appended to `log` so that the test can check the order of the step's parts."""
    import oracle

    rp, ci, cf, _, _ = _layer()

    def fwd(a, X, alpha, wq, Z_out=None, Y=None, ws=None):
        log.append("fwd")
        Zr, Yr = oracle.adapter_fwd(rp, ci, cf, X.numpy(), D_OUT, N, alpha)
        return torch.from_numpy(Zr), torch.from_numpy(Yr)

    def bwd(a, dY, Z, alpha, wq, dc=None, dX=None, want_dx=True, ws=None, want_dc=True):
        log.append(("bwd", want_dc, want_dx))
        out_dc = out_dx = None
        if want_dc:
            # the oracle's dc takes X; Z = X H and H is its own inverse, so X = Z H
            X = oracle.fwht(Z.numpy(), N)
            out_dc = torch.from_numpy(oracle.adapter_bwd_dc(X, dY.numpy(), oracle.csr_rows(rp), ci, N, alpha))
        if want_dx:
            out_dx = torch.from_numpy(oracle.adapter_bwd_dx(rp, ci, cf, dY.numpy(), D_IN, N, alpha))
        return out_dc, out_dx

    return fwd, bwd


def _dp_step_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import oracle
    from walsh_hadamard_sparse_b200.api import dp_step
    from workloads import rank_rows

    oracle.set_threads(1)
    _, _, _, X, dY = _layer()
    rows = rank_rows(rank, T_RANK)
    log = []
    fwd, bwd = _oracle_layer_steps(log)
    Z, Y, dc, dX = dp_step(None, torch.from_numpy(X[rows]), torch.from_numpy(dY[rows]), 0.7, fwd=fwd, bwd=bwd)
    out[rank] = (Y.numpy().copy(), dc.numpy().copy(), dX.numpy().copy(), log)
    dist.barrier()
    dist.destroy_process_group()


def test_dp_step_of_the_package_on_two_ranks():
    """walsh_hadamard_sparse_b200.dp_step on 2 gloo ranks, the oracle's forward and backward injected: every rank
    ends with the dc of all tokens (one all-reduce) and the Y and dX rows of its own tokens, and the step runs the
    forward, then dc alone, then dX alone (dc's all-reduce is in flight while dX is computed)."""
    import oracle

    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_dp_step_worker, args=(2, port, out), nprocs=2, join=True)
    rp, ci, cf, X, dY = _layer()
    _, Y_all = oracle.adapter_fwd(rp, ci, cf, X, D_OUT, N, 0.7)
    dc_all = oracle.adapter_bwd_dc(X, dY, oracle.csr_rows(rp), ci, N, 0.7)
    dX_all = oracle.adapter_bwd_dx(rp, ci, cf, dY, D_IN, N, 0.7)
    for r in range(2):
        Y_r, dc_r, dX_r, log = out[r]
        rows = slice(r * T_RANK, (r + 1) * T_RANK)
        assert log == ["fwd", ("bwd", True, False), ("bwd", False, True)], log
        assert np.allclose(dc_r, dc_all, rtol=1e-12, atol=1e-12)
        assert np.allclose(Y_r, Y_all[rows], rtol=1e-12, atol=1e-12)
        assert np.allclose(dX_r, dX_all[rows], rtol=1e-12, atol=1e-12)


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
