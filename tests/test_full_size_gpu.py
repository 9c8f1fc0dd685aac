"""Parity at the full workload sizes, in the launch configuration bench.py times.

The whole layer runs on the GPU; the oracle checks seeded samples it can
compute one by one: 32-64 token rows of Y and dX, and a few dozen entries of dc
(each needs the full token sum). E and c come from the oracle's own AdaAlloc
(the GPU AdaAlloc is checked against it bit for bit separately), so no oracle
input comes from the CUDA path."""

import numpy as np
import pytest

import oracle
from _util import TOL_BF16, bf16_dev, host, rel_fro
from workloads import CONFIGS, layer_inputs, pack_codes, rng_for

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def _device_layer(spec, workload, seed=0):
    import torch
    import walsh_hadamard_sparse_b200 as W

    d = layer_inputs(spec, seed, workload)
    ref = oracle.init_alloc(d["dWq"], spec.p, spec.had_block, spec.min_per_row, spec.remainder)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()  # noqa: E731
    wq = W.QWeight(spec.bits, spec.group, dev(d["qweight"]), dev(d["scales"]), dev(d["zeros"]))
    X, dY = bf16_dev(d["X_bits"]), bf16_dev(d["dY_bits"])
    return d, ref, wq, X, dY


def _check_layer(spec, workload, algos=("dense", "sparse"), rows_n=48, dc_n=48):
    import torch
    import walsh_hadamard_sparse_b200 as W

    d, ref, wq, X, dY = _device_layer(spec, workload)
    rp, ci, cf = ref["row_ptr"], ref["col_idx"], ref["coef"]
    g = rng_for(60, "full", workload, spec.name)
    rows = np.sort(g.choice(spec.T, rows_n, replace=False))
    sel = np.sort(g.choice(spec.p, dc_n, replace=False))
    Wq = oracle.dequant(d["qweight"], d["scales"], d["zeros"], spec.bits, spec.group, spec.d_out, spec.d_in)
    _, Yr = oracle.adapter_fwd(rp, ci, cf, d["X"][rows], spec.d_out, spec.had_block, 1.0, Wq, want_z=False)
    dXr = oracle.adapter_bwd_dx(rp, ci, cf, d["dY"][rows], spec.d_in, spec.had_block, 1.0, Wq)
    dcr = oracle.adapter_bwd_dc(d["X"], d["dY"], oracle.csr_rows(rp)[sel], ci[sel], spec.had_block, 1.0)
    dv = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()  # noqa: E731
    ri = torch.as_tensor(rows).cuda()
    for algo in algos:
        a = W.Adapter(spec.d_in, spec.d_out, spec.had_block, spec.p, dv(rp), dv(ci), dv(cf), algo=algo)
        W.plan_build(a)
        if algo == "dense":
            a.weff = torch.empty((spec.d_out, spec.d_in), dtype=torch.bfloat16, device="cuda")
        Z, Y = W.adapter_fwd(a, X, 1.0, wq)
        dc, dX = W.adapter_bwd(a, dY, Z, 1.0, wq)
        torch.cuda.synchronize()
        errs = {"Y": rel_fro(host(Y[ri]), Yr), "dX": rel_fro(host(dX[ri]), dXr),
                "dc": rel_fro(dc.cpu().numpy()[sel], dcr)}
        assert all(v <= TOL_BF16 for v in errs.values()), (algo, errs)
        assert bool(torch.isfinite(dc).all()) and bool(torch.isfinite(Y.float()).all())
        del a, Z, Y, dc, dX


def _zero_base(spec, d):
    """A base weight of the layer's format whose codes all equal their group's zero point, so W_Q = 0 exactly:
    the dense algorithm then runs its full-size kernels (W_eff from packed codes, the GEMMs with the fused
    transform) while Y and dX hold the adapter term alone."""
    import torch
    import walsh_hadamard_sparse_b200 as W

    codes = np.repeat(d["zeros"], spec.group, axis=1)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()  # noqa: E731
    return W.QWeight(spec.bits, spec.group, dev(pack_codes(codes, spec.bits)), dev(d["scales"]), dev(d["zeros"]))


def _check_adapter_alone(spec, workload, rows_n=32):
    """The adapter term alone at full size, where the base term cannot hide an error in it: Z, Y and dX on sampled
    token rows against the oracle's adapter-only forward and backward (papernotes.org "QWHA", 整体框架: Y_ad =
    alpha X (F H^-1)^T, with E and c from AdaAlloc of the layer's real quantization error). Sparse algorithm without
    a base weight; dense algorithm with an all-zero base weight of the layer's bit width."""
    import torch
    import walsh_hadamard_sparse_b200 as W

    d, ref, _, X, dY = _device_layer(spec, workload)
    rp, ci, cf = ref["row_ptr"], ref["col_idx"], ref["coef"]
    g = rng_for(61, "full-adapter", workload, spec.name)
    rows = np.sort(g.choice(spec.T, rows_n, replace=False))
    rows[0], rows[-1] = 0, spec.T - 1  # the first and the last token tile
    Zr, Yr = oracle.adapter_fwd(rp, ci, cf, d["X"][rows], spec.d_out, spec.had_block, 1.0)
    dXr = oracle.adapter_bwd_dx(rp, ci, cf, d["dY"][rows], spec.d_in, spec.had_block, 1.0)
    assert np.linalg.norm(Yr) > 0 and np.linalg.norm(dXr) > 0
    wq0 = _zero_base(spec, d)
    dv = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()  # noqa: E731
    ri = torch.as_tensor(rows).cuda()
    for algo, wq in (("sparse", None), ("dense", wq0)):
        a = W.Adapter(spec.d_in, spec.d_out, spec.had_block, spec.p, dv(rp), dv(ci), dv(cf), algo=algo)
        W.plan_build(a)
        if algo == "dense":
            a.weff = torch.empty((spec.d_out, spec.d_in), dtype=torch.bfloat16, device="cuda")
        Z, Y = W.adapter_fwd(a, X, 1.0, wq)
        _, dX = W.adapter_bwd(a, dY, Z, 1.0, wq, want_dc=False)
        torch.cuda.synchronize()
        errs = {"Z": rel_fro(host(Z[ri]), Zr), "Y": rel_fro(host(Y[ri]), Yr), "dX": rel_fro(host(dX[ri]), dXr)}
        assert all(v <= TOL_BF16 for v in errs.values()), (algo, errs)
        del a, Z, Y, dX


def test_q_proj_full_size():
    """LLaMA-7B q_proj: 4096 x 4096, 8192 tokens, 4-bit g128, p = 524288."""
    _check_layer(CONFIGS["q_proj"][0], "q_proj")


@pytest.mark.parametrize("name", ["gate", "down"])
def test_llama3_mlp_full_size(name):
    """LLaMA-3-8B MLP, 16384 tokens, 3-bit g128, r = 64: gate 4096 -> 14336, and
    down 14336 -> 4096 whose H is block-diagonal with seven 2048-point blocks."""
    spec = next(s for s in CONFIGS["mlp"] if s.name == name)
    _check_layer(spec, "mlp", rows_n=32, dc_n=24)


def test_q_proj_adapter_alone_full_size():
    """The q_proj layer's adapter term alone (no base term to dominate it), both algorithms."""
    _check_adapter_alone(CONFIGS["q_proj"][0], "q_proj")


@pytest.mark.parametrize("name", ["gate", "down"])
def test_llama3_mlp_adapter_alone_full_size(name):
    """The MLP layers' adapter term alone at 16384 tokens: gate (4096 -> 14336) and down (14336 -> 4096, seven
    2048-point Hadamard blocks), both algorithms."""
    spec = next(s for s in CONFIGS["mlp"] if s.name == name)
    _check_adapter_alone(spec, "mlp", rows_n=24)


def test_init_sweep_full_size_bitexact():
    """AdaAlloc on all seven LLaMA-3-8B linear shapes, 2-bit g64, r in {16, 64, 128}:
    budgets, E and c bit for bit against the oracle."""
    import torch
    import walsh_hadamard_sparse_b200 as W

    cache = {}
    for spec in sorted(CONFIGS["init_sweep"], key=lambda s: s.w_stream):  # the three r of a shape share dW_Q
        if spec.w_stream not in cache:
            cache.clear()
            cache[spec.w_stream] = layer_inputs(spec, 0, "init_sweep", parts=("W",))["dWq"]
        w = cache[spec.w_stream]
        got = W.init_alloc(torch.from_numpy(w).cuda(), spec.p, spec.had_block, spec.min_per_row, spec.remainder)
        ref = oracle.init_alloc(w, spec.p, spec.had_block, spec.min_per_row, spec.remainder)
        for k in ("budgets", "row_ptr", "col_idx"):
            assert np.array_equal(got[k].cpu().numpy(), ref[k]), (spec.name, k)
        assert np.array_equal(got["coef"].cpu().numpy().view(np.uint32), ref["coef"].view(np.uint32)), spec.name


@pytest.mark.parametrize("sel", ["magnitude", "random"])
def test_select_global_full_size_bitexact(sel):
    """The pages' alternatives to AdaAlloc on the q_proj layer (4096 x 4096, p = 524288): whole-matrix magnitude
    top-p and seeded random E, budgets, E and c bit for bit against the oracle."""
    import torch
    import walsh_hadamard_sparse_b200 as W

    spec = CONFIGS["q_proj"][0]
    w = layer_inputs(spec, 0, "q_proj", parts=("W",))["dWq"]
    got = W.init_select_global(torch.from_numpy(w).cuda(), spec.p, spec.had_block, sel, 2024)
    ref = oracle.init_select_global(w, spec.p, spec.had_block, sel, 2024)
    for k in ("budgets", "row_ptr", "col_idx"):
        assert np.array_equal(got[k].cpu().numpy(), ref[k]), (sel, k)
    assert np.array_equal(got["coef"].cpu().numpy().view(np.uint32), ref["coef"].view(np.uint32)), sel
