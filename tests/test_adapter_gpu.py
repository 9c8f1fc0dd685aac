"""Forward, backward, plan and AdaAlloc through the C ABI, against the oracle."""

import numpy as np
import pytest

import oracle
from _util import TOL_BF16, TOL_F32, bf16_dev, host, rel_fro, to_dev
from workloads import (
    CONFIGS,
    bf16_bits_to_f32,
    f32_to_bf16_bits,
    layer_inputs,
    pack_codes,
    quantize_rtn,
    random_pattern,
    rng_for,
)

pytestmark = pytest.mark.gpu

# edge of the tile view's blocks (QWHA_TILE in include/qwha.h)
TILE = int(next(l.split()[2] for l in open(__import__("_util").HEADER) if l.startswith("#define QWHA_TILE")))


def _W():
    import walsh_hadamard_sparse_b200 as W

    return W


def device_adapter(d_in, d_out, n, rp, ci, cf, plan=True, algo="sparse"):
    import torch

    W = _W()
    a = W.Adapter(d_in, d_out, n, int(ci.size), to_dev(rp), to_dev(ci) if ci.size else torch.zeros(1, dtype=torch.int32, device="cuda"),
                  to_dev(cf) if cf.size else torch.zeros(1, device="cuda"), algo=algo)
    if plan:
        W.plan_build(a)
    return a


def synth_layer(seed, d_in, d_out, n, T, p, dtype, bits=4, group=64, pattern="init"):
    """Seeded layer: activations, gradients, a quantized weight, and E/c from the oracle's AdaAlloc
    (or a random pattern for edge cases)."""
    g = rng_for(seed, "adapter-test", d_in, d_out, n, T, p)
    group = group if d_in % group == 0 else 32
    w0 = (g.standard_normal((d_out, d_in)).astype(np.float32) * np.float32(0.02))
    w0[g.random((d_out, d_in)) < 0.002] *= np.float32(15.0)
    q, s, z, wq, dwq = quantize_rtn(w0, bits, group)
    X = g.standard_normal((T, d_in)).astype(np.float32)
    X[:, g.choice(d_in, max(1, d_in // 100), replace=False)] *= np.float32(20.0)
    dY = g.standard_normal((T, d_out)).astype(np.float32)
    if dtype == "bf16":
        X = bf16_bits_to_f32(f32_to_bf16_bits(X))
        dY = bf16_bits_to_f32(f32_to_bf16_bits(dY))
    if pattern == "init":
        e = oracle.init_alloc(dwq, p, n, 2, "fewest")
        rp, ci, cf = e["row_ptr"], e["col_idx"], e["coef"]
    else:
        rp, ci, cf = random_pattern(d_out, d_in, p=p, rng=g)
    return dict(X=X, dY=dY, rp=rp, ci=ci, cf=cf, qweight=pack_codes(q, bits), scales=s, zeros=z, Wq=wq,
                dWq=dwq, bits=bits, group=group)


def dev_act(a, dtype):
    if dtype == "bf16":
        return bf16_dev(f32_to_bf16_bits(a))
    return to_dev(a)


def dev_qweight(L):
    W = _W()
    return W.QWeight(L["bits"], L["group"], to_dev(L["qweight"]), to_dev(L["scales"]), to_dev(L["zeros"]))


# --------------------------------------------------------------------------- plan


def expected_tiles(rp, ci, d_out, d_in):
    cp, ri, pm = oracle.plan_build(rp, ci, d_in)
    E = TILE
    n_rb = -(-d_out // E)
    n_kb = -(-d_in // E)
    cols = np.repeat(np.arange(d_in), np.diff(cp))
    tile = (cols // E) * n_rb + ri // E
    order = np.argsort(tile, kind="stable")
    tile_ptr = np.zeros(n_rb * n_kb + 1, dtype=np.int64)
    tile_ptr[1:] = np.cumsum(np.bincount(tile, minlength=n_rb * n_kb))
    rk = ((ri % E) << 16) | (cols % E)
    return cp, ri, pm, tile_ptr, pm[order], rk[order]


@pytest.mark.parametrize(
    "d_out,d_in,counts",
    [
        (64, 256, "random"),
        (1200, 1104, "random"),  # several row and column blocks, ragged edges
        (40, 96, "edge"),  # empty rows, full rows
        (8, 8, "full"),
        (16, 32, "empty"),
    ],
)
def test_plan_build_matches_oracle(d_out, d_in, counts):
    import torch

    W = _W()
    g = rng_for(30, "plan", d_out, d_in)
    if counts == "random":
        rp, ci, cf = random_pattern(d_out, d_in, p=min(d_out * d_in, 40 * d_out), rng=g)
    elif counts == "edge":
        c = g.integers(0, 12, d_out)
        c[::7] = 0
        c[3] = d_in
        rp, ci, cf = random_pattern(d_out, d_in, counts=c, rng=g)
    elif counts == "full":
        rp, ci, cf = random_pattern(d_out, d_in, counts=np.full(d_out, d_in), rng=g)
    else:
        rp, ci, cf = random_pattern(d_out, d_in, counts=np.zeros(d_out, dtype=np.int64), rng=g)
    a = device_adapter(d_in, d_out, 8, rp, ci, cf)
    torch.cuda.synchronize()
    cp, ri, pm, tp, tpos, trk = expected_tiles(rp, ci, d_out, d_in)
    p = ci.size
    assert np.array_equal(a.col_ptr.cpu().numpy(), cp)
    assert np.array_equal(a.row_idx.cpu().numpy()[:p], ri)
    assert np.array_equal(a.perm.cpu().numpy()[:p], pm)
    assert np.array_equal(a.tile_ptr.cpu().numpy(), tp)
    assert np.array_equal(a.tile_pos.cpu().numpy()[:p], tpos)
    assert np.array_equal(a.tile_rk.cpu().numpy()[:p], trk)
    W.validate_plan(a)


def test_validate_plan_rejects_bad_patterns():
    import torch

    W = _W()
    rp, ci, cf = random_pattern(32, 64, p=200, rng=rng_for(31, "bad"))
    a = device_adapter(64, 32, 64, rp, ci, cf)
    W.validate_plan(a)
    bad = ci.copy()
    r = 5
    bad[rp[r]], bad[rp[r] + 1] = bad[rp[r] + 1], bad[rp[r]]  # unsorted inside row 5
    a.col_idx = to_dev(bad)
    with pytest.raises(W.QwhaError, match="increasing"):
        W.validate_plan(a)
    bad2 = ci.copy()
    bad2[7] = 64  # out of range
    a.col_idx = to_dev(bad2)
    with pytest.raises(W.QwhaError, match="out of"):
        W.validate_plan(a)
    a.col_idx = to_dev(ci)
    a.perm = torch.flip(a.perm[: ci.size], [0]).contiguous()
    with pytest.raises(W.QwhaError):
        W.validate_plan(a)


# --------------------------------------------------------------------------- init


@pytest.mark.parametrize("mode", ["fewest", "largest"])
def test_init_tiny_workload_bitexact(mode):
    W = _W()
    spec = CONFIGS["tiny"][0]
    d = layer_inputs(spec, 0, "tiny", parts=("W",))
    got = W.init_alloc(to_dev(d["dWq"]), spec.p, spec.had_block, 2, mode)
    ref = oracle.init_alloc(d["dWq"], spec.p, spec.had_block, 2, mode)
    for k in ("budgets", "row_ptr", "col_idx"):
        assert np.array_equal(got[k].cpu().numpy(), ref[k]), k
    assert np.array_equal(got["coef"].cpu().numpy().view(np.uint32), ref["coef"].view(np.uint32))


@pytest.mark.parametrize(
    "d_out,d_in,n,p,mode,kind",
    [
        (96, 128, 128, 96 * 9 + 5, "fewest", "normal"),
        (80, 3 * 64, 64, 80 * 5 + 33, "largest", "normal"),  # block-diagonal transform
        (1000, 1024, 1024, 1000 * 40 + 123, "fewest", "normal"),  # several budget threads per row
        (64, 64, 64, 64 * 6, "fewest", "cap"),  # a few rows hit the cap d_in
        (64, 64, 64, 64 * 6, "largest", "cap"),
        (48, 32, 32, 48 * 3 + 7, "fewest", "ties"),  # zero rows and integer data: many equal |V|
        (16, 16, 16, 16 * 16, "fewest", "normal"),  # p = d_in * d_out
        (24, 2048, 2048, 24 * 3, "largest", "normal"),  # p = 3 per row, long rows
        # rows of 4096 entries take the register-resident selection kernel
        (40, 4096, 4096, 40 * 50 + 7, "fewest", "normal"),
        (33, 4096, 1024, 33 * 20 + 5, "largest", "normal"),  # block-diagonal: stages above 1024 skipped
        (17, 4096, 64, 17 * 9 + 3, "fewest", "normal"),  # 64-point blocks: two of three register phases
        (20, 4096, 4096, 20 * 700, "fewest", "cap"),  # capped rows take all 4096 entries
        (24, 4096, 4096, 24 * 30 + 11, "largest", "ties"),  # zero rows (all keys equal), many ties
        (12, 4096, 4096, 12 * 2, "fewest", "normal"),  # the minimum: 2 entries per row
    ],
)
def test_init_bitexact(d_out, d_in, n, p, mode, kind):
    W = _W()
    g = rng_for(32, "init", d_out, d_in, n, p, kind)
    w = g.standard_normal((d_out, d_in)).astype(np.float32) * np.float32(0.01)
    if kind == "cap":
        w[:3] *= np.float32(1000.0)
    if kind == "ties":
        w = g.integers(-2, 3, size=(d_out, d_in)).astype(np.float32)
        w[::5] = 0.0
    got = W.init_alloc(to_dev(w), p, n, 2, mode)
    ref = oracle.init_alloc(w, p, n, 2, mode)
    if kind == "cap":
        assert ref["budgets"].max() == d_in
    for k in ("budgets", "row_ptr", "col_idx"):
        assert np.array_equal(got[k].cpu().numpy(), ref[k]), k
    assert np.array_equal(got["coef"].cpu().numpy().view(np.uint32), ref["coef"].view(np.uint32))


@pytest.mark.parametrize("shards,mode,d_in", [(1, "fewest", 1024), (3, "largest", 1024), (2, "fewest", 4096)])
def test_init_split_steps_bitexact(shards, mode, d_in):
    """qwha_init_norms / _budgets / _select over row shards (as the ranks of a sharded AdaAlloc run them)
    reproduce qwha_init_alloc and the oracle bit for bit; the shards' row_ptr slices do not start at 0."""
    import torch

    from walsh_hadamard_sparse_b200.api import shard_rows

    W = _W()
    d_out, n = 301, 512
    p = d_out * 17 + 9
    g = rng_for(34, "init-split", shards, mode) if d_in == 1024 else rng_for(34, "init-split", shards, mode, d_in)
    w = g.standard_normal((d_out, d_in)).astype(np.float32) * np.float32(0.01)
    w[7] *= np.float32(500.0 if d_in == 1024 else 5000.0)  # capped row
    dw = to_dev(w)
    whole = W.init_alloc(dw, p, n, 2, mode)
    bounds = [shard_rows(d_out, r, shards) for r in range(shards)]
    e = torch.cat([W.init_norms(dw[r0:r1]) for r0, r1 in bounds])
    b, rp = W.init_budgets(e, d_in, p, 2, mode)
    sel = [W.init_select(dw[r0:r1], n, b[r0:r1], rp[r0:r1 + 1]) for r0, r1 in bounds]  # slices at any offset
    ci = torch.cat([s[0] for s in sel]).cpu().numpy()
    cf = torch.cat([s[1] for s in sel]).cpu().numpy()
    ref = oracle.init_alloc(w, p, n, 2, mode)
    assert ref["budgets"].max() == d_in
    for got in ({"budgets": b.cpu().numpy(), "row_ptr": rp.cpu().numpy(), "col_idx": ci, "coef": cf},
                {k: v.cpu().numpy() for k, v in whole.items()}):
        for k in ("budgets", "row_ptr", "col_idx"):
            assert np.array_equal(got[k], ref[k]), k
        assert np.array_equal(got["coef"].view(np.uint32), ref["coef"].view(np.uint32))


@pytest.mark.parametrize(
    "d_out,d_in,n,p,sel,kind",
    [
        (96, 128, 128, 96 * 9 + 5, "magnitude", "normal"),
        (80, 3 * 64, 64, 700, "magnitude", "normal"),  # block-diagonal transform
        (48, 32, 32, 300, "magnitude", "ties"),  # integer data: many equal |V|, decided by the flat index
        (300, 512, 512, 300 * 20, "random", "normal"),
        (64, 64, 64, 64 * 64, "random", "normal"),  # p = all entries
        (64, 64, 64, 1, "magnitude", "normal"),
        (64, 64, 64, 0, "random", "normal"),
    ],
)
def test_select_global_bitexact(d_out, d_in, n, p, sel, kind):
    """Whole-matrix selection (magnitude top-p, seeded random E) bit for bit against the oracle."""
    W = _W()
    g = rng_for(36, "select-global", d_out, d_in, p, sel, kind)
    if kind == "ties":
        w = g.integers(-1, 2, size=(d_out, d_in)).astype(np.float32)
    else:
        w = g.standard_normal((d_out, d_in)).astype(np.float32) * np.float32(0.01)
    seed = 0x5EED0000 + p
    got = W.init_select_global(to_dev(w), p, n, sel, seed)
    ref = oracle.init_select_global(w, p, n, sel, seed)
    for k in ("budgets", "row_ptr", "col_idx"):
        assert np.array_equal(got[k].cpu().numpy(), ref[k]), k
    assert np.array_equal(got["coef"].cpu().numpy().view(np.uint32), ref["coef"].view(np.uint32))


# --------------------------------------------------------------------------- forward / backward


CASES = [
    # d_in, d_out, n, T, p, dtype, pattern
    (256, 256, 256, 64, 1024, "f32", "init"),
    (512, 384, 128, 77, 384 * 20, "f32", "init"),
    (1024, 768, 1024, 300, 768 * 24, "bf16", "init"),
    (768, 512, 256, 33, 512 * 30, "bf16", "random"),  # block-diagonal transform
    (96, 40, 32, 5, 300, "bf16", "random"),
    (1024, 1024, 1024, 600, 1024 * 20, "bf16", "init"),  # dense: dc GEMM split in two along tokens
]


ALGO_CASES = [c + ("sparse",) for c in CASES] + [c + ("dense",) for c in CASES if c[5] == "bf16"]


@pytest.mark.parametrize("d_in,d_out,n,T,p,dtype,pattern,algo", ALGO_CASES)
def test_adapter_forward_backward(d_in, d_out, n, T, p, dtype, pattern, algo):
    import torch

    W = _W()
    L = synth_layer(33, d_in, d_out, n, T, p, dtype, pattern=pattern)
    a = device_adapter(d_in, d_out, n, L["rp"], L["ci"], L["cf"], algo=algo)
    alpha = 0.8
    Xd, dYd = dev_act(L["X"], dtype), dev_act(L["dY"], dtype)
    Z, Y = W.adapter_fwd(a, Xd, alpha)
    dc, dX = W.adapter_bwd(a, dYd, Z, alpha)
    torch.cuda.synchronize()
    Zr, Yr = oracle.adapter_fwd(L["rp"], L["ci"], L["cf"], L["X"], d_out, n, alpha)
    dXr = oracle.adapter_bwd_dx(L["rp"], L["ci"], L["cf"], L["dY"], d_in, n, alpha)
    rows = oracle.csr_rows(L["rp"])
    sel = np.arange(L["ci"].size)
    if sel.size > 3000:
        sel = np.sort(rng_for(34, "dcsel").choice(sel.size, 3000, replace=False))
    dcr = oracle.adapter_bwd_dc(L["X"], L["dY"], rows[sel], L["ci"][sel], n, alpha)
    tol = TOL_F32 if dtype == "f32" else TOL_BF16
    errs = dict(Z=rel_fro(host(Z), Zr), Y=rel_fro(host(Y), Yr), dX=rel_fro(host(dX), dXr),
                dc=rel_fro(dc.cpu().numpy()[sel], dcr))
    assert all(v <= tol for v in errs.values()), errs
    # fixed-order reduction: a second backward is bitwise identical
    dc2, _ = W.adapter_bwd(a, dYd, Z, alpha)
    assert torch.equal(dc, dc2)
    if algo == "dense":
        # W_eff saved by the forward and reused by the backward gives the same bits
        a.weff = torch.empty((d_out, d_in), dtype=torch.bfloat16, device="cuda")
        Z3, Y3 = W.adapter_fwd(a, Xd, alpha)
        dc3, dX3 = W.adapter_bwd(a, dYd, Z3, alpha)
        assert torch.equal(Y3, Y) and torch.equal(dc3, dc) and torch.equal(dX3, dX)


def edge_pattern(kind, d_out, d_in, g):
    """Sparsity patterns with the degenerate rows and columns a real E can have: "rows" mixes empty and full rows
    into rows of ordinary length; "cols" leaves two thirds of the columns (two of every three 256-column tiles, and
    a ragged run at the end) without any nonzero."""
    if kind == "rows":
        c = g.integers(1, 24, d_out)
        c[::5] = 0
        c[1::9] = d_in
        c[-1] = 0
        return random_pattern(d_out, d_in, counts=c, rng=g)
    live = np.array([k for k in range(d_in) if (k // 256) % 3 == 1 and k < d_in - 40])
    rp, ci, cf = random_pattern(d_out, live.size, p=d_out * 12, rng=g)
    return rp, live[ci].astype(np.int32), cf


EDGE_CASES = [
    # d_in, d_out, n, T, dtype, pattern
    (1024, 768, 1024, 1, "bf16", "init"),
    (1024, 768, 1024, 3, "bf16", "init"),
    (1024, 768, 1024, 127, "bf16", "init"),
    (256, 256, 256, 1, "f32", "init"),
    (256, 256, 256, 3, "f32", "init"),
    (512, 384, 512, 100, "bf16", "rows"),
    (512, 384, 256, 100, "f32", "rows"),
    (1536, 520, 512, 70, "bf16", "cols"),
]


@pytest.mark.parametrize("algo", ["sparse", "dense"])
@pytest.mark.parametrize("d_in,d_out,n,T,dtype,pattern", EDGE_CASES)
def test_adapter_edge_cases(d_in, d_out, n, T, dtype, pattern, algo):
    """Token counts of 1, 3 and 127 (a single token, a few, one short of a 128-row tile) and patterns with empty rows,
    full rows and empty columns: Z, Y, dX and every dc against the oracle, the adapter alone and with a base weight."""
    import torch

    if algo == "dense" and dtype != "bf16":
        pytest.skip("the dense algorithm is bf16 only")
    W = _W()
    if pattern == "init":
        L = synth_layer(42, d_in, d_out, n, T, d_out * 16, dtype)
    else:
        L = synth_layer(42, d_in, d_out, n, T, d_out * 4, dtype, pattern="random")
        L["rp"], L["ci"], L["cf"] = edge_pattern(pattern, d_out, d_in, rng_for(43, "edge", pattern, d_in))
    rp, ci, cf = L["rp"], L["ci"], L["cf"]
    if pattern == "rows":
        cnt = np.diff(rp)
        assert (cnt == 0).any() and (cnt == d_in).any()
    if pattern == "cols":
        assert np.bincount(ci, minlength=d_in)[d_in - 40:].sum() == 0
    a = device_adapter(d_in, d_out, n, rp, ci, cf, algo=algo)
    alpha = 0.75
    Xd, dYd = dev_act(L["X"], dtype), dev_act(L["dY"], dtype)
    tol = TOL_F32 if dtype == "f32" else TOL_BF16
    Zr, Yr = oracle.adapter_fwd(rp, ci, cf, L["X"], d_out, n, alpha)
    dXr = oracle.adapter_bwd_dx(rp, ci, cf, L["dY"], d_in, n, alpha)
    dcr = oracle.adapter_bwd_dc(L["X"], L["dY"], oracle.csr_rows(rp), ci, n, alpha)
    Z, Y = W.adapter_fwd(a, Xd, alpha)
    dc, dX = W.adapter_bwd(a, dYd, Z, alpha)
    torch.cuda.synchronize()
    errs = dict(Z=rel_fro(host(Z), Zr), Y=rel_fro(host(Y), Yr), dX=rel_fro(host(dX), dXr), dc=rel_fro(dc.cpu().numpy(), dcr))
    assert all(v <= tol for v in errs.values()), errs
    if dtype != "bf16":
        return
    wq = dev_qweight(L)
    Wq = oracle.dequant(L["qweight"], L["scales"], L["zeros"], L["bits"], L["group"], d_out, d_in)
    _, Yr = oracle.adapter_fwd(rp, ci, cf, L["X"], d_out, n, alpha, Wq, want_z=False)
    dXr = oracle.adapter_bwd_dx(rp, ci, cf, L["dY"], d_in, n, alpha, Wq)
    Z, Y = W.adapter_fwd(a, Xd, alpha, wq=wq)
    dc, dX = W.adapter_bwd(a, dYd, Z, alpha, wq=wq)
    torch.cuda.synchronize()
    errs = dict(Y=rel_fro(host(Y), Yr), dX=rel_fro(host(dX), dXr), dc=rel_fro(dc.cpu().numpy(), dcr))
    assert all(v <= tol for v in errs.values()), errs


GEMM_CASES = [
    (512, 256, 512, 200, 4, 64),  # ragged token tile (200 = 128 + 72)
    (1024, 768, 1024, 300, 3, 128),  # int3 bit stream
    (640, 1280, 128, 129, 2, 64),  # int2, ragged token tile, K of 10 ring blocks
    (256, 264, 256, 7, 4, 64),  # N = 264: partial 32-column epilogue chunk
]


@pytest.mark.parametrize("algo", ["sparse", "dense"])
@pytest.mark.parametrize("d_in,d_out,n,T,bits,group", GEMM_CASES)
def test_base_gemm_forward_backward(d_in, d_out, n, T, bits, group, algo):
    import torch

    W = _W()
    p = d_out * 8
    L = synth_layer(35, d_in, d_out, n, T, p, "bf16", bits=bits, group=group)
    a = device_adapter(d_in, d_out, n, L["rp"], L["ci"], L["cf"], algo=algo)
    wq = dev_qweight(L)
    alpha = 1.0
    Xd, dYd = dev_act(L["X"], "bf16"), dev_act(L["dY"], "bf16")
    Z, Y = W.adapter_fwd(a, Xd, alpha, wq=wq)
    dc, dX = W.adapter_bwd(a, dYd, Z, alpha, wq=wq)
    torch.cuda.synchronize()
    Wq = oracle.dequant(L["qweight"], L["scales"], L["zeros"], bits, group, d_out, d_in)
    _, Yr = oracle.adapter_fwd(L["rp"], L["ci"], L["cf"], L["X"], d_out, n, alpha, Wq, want_z=False)
    dXr = oracle.adapter_bwd_dx(L["rp"], L["ci"], L["cf"], L["dY"], d_in, n, alpha, Wq)
    sel = np.sort(rng_for(37, "dcsel", d_out).choice(L["ci"].size, min(1500, L["ci"].size), replace=False))
    dcr = oracle.adapter_bwd_dc(L["X"], L["dY"], oracle.csr_rows(L["rp"])[sel], L["ci"][sel], n, alpha)
    errs = dict(Y=rel_fro(host(Y), Yr), dX=rel_fro(host(dX), dXr), dc=rel_fro(dc.cpu().numpy()[sel], dcr))
    assert all(v <= TOL_BF16 for v in errs.values()), errs
    # the base term alone (empty adapter) against the oracle's X W_Q^T
    e = device_adapter(d_in, d_out, n, np.zeros(d_out + 1, np.int32), np.zeros(0, np.int32), np.zeros(0, np.float32),
                       algo=algo)
    _, Yb = W.adapter_fwd(e, Xd, alpha, wq=wq)
    torch.cuda.synchronize()
    assert rel_fro(host(Yb), L["X"].astype(np.float64) @ Wq.T) <= TOL_BF16


@pytest.mark.parametrize("algo", ["sparse", "dense"])
def test_backward_in_two_calls_bitwise(algo):
    """dc alone (dX NULL), then dX alone (dc NULL), as a data-parallel step issues them around the all-reduce of dc:
    bit for bit the outputs of one call."""
    import torch

    W = _W()
    d_in, d_out, n, T = 1024, 768, 1024, 300
    L = synth_layer(38, d_in, d_out, n, T, d_out * 8, "bf16", bits=4, group=128)
    a = device_adapter(d_in, d_out, n, L["rp"], L["ci"], L["cf"], algo=algo)
    if algo == "dense":
        a.weff = torch.empty((d_out, d_in), dtype=torch.bfloat16, device="cuda")
    wq = dev_qweight(L)
    Z, _ = W.adapter_fwd(a, dev_act(L["X"], "bf16"), 0.8, wq=wq)
    dYd = dev_act(L["dY"], "bf16")
    dc1, dX1 = W.adapter_bwd(a, dYd, Z, 0.8, wq=wq)
    dc2, none_dx = W.adapter_bwd(a, dYd, Z, 0.8, wq=wq, want_dx=False)
    none_dc, dX2 = W.adapter_bwd(a, dYd, Z, 0.8, wq=wq, want_dc=False)
    torch.cuda.synchronize()
    assert none_dx is None and none_dc is None
    assert torch.equal(dc1.view(torch.int32), dc2.view(torch.int32))
    assert torch.equal(dX1.view(torch.int16), dX2.view(torch.int16))


@pytest.mark.parametrize("algo", ["sparse", "dense"])
def test_dp_backward_world_size_one_bitwise(algo):
    """The package's data-parallel backward (dc, its NCCL all-reduce started asynchronously, dX meanwhile) in a
    one-rank NCCL process group: bit for bit the single call's dc and dX."""
    import torch
    import torch.distributed as dist

    W = _W()
    d_in, d_out, n, T = 1024, 768, 1024, 300
    L = synth_layer(44, d_in, d_out, n, T, d_out * 8, "bf16", bits=4, group=128)
    a = device_adapter(d_in, d_out, n, L["rp"], L["ci"], L["cf"], algo=algo)
    if algo == "dense":
        a.weff = torch.empty((d_out, d_in), dtype=torch.bfloat16, device="cuda")
    wq = dev_qweight(L)
    Xd, dYd = dev_act(L["X"], "bf16"), dev_act(L["dY"], "bf16")
    Z, _ = W.adapter_fwd(a, Xd, 0.8, wq=wq)
    dc1, dX1 = W.adapter_bwd(a, dYd, Z, 0.8, wq=wq)
    dist.init_process_group("nccl", store=dist.HashStore(), rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        dc2, dX2 = W.dp_backward(a, dYd, Z, 0.8, wq=wq)
        _, Y3, dc3, dX3 = W.dp_step(a, Xd, dYd, 0.8, wq=wq)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    for dc in (dc2, dc3):
        assert torch.equal(dc1.view(torch.int32), dc.view(torch.int32))
    for dX in (dX2, dX3):
        assert torch.equal(dX1.view(torch.int16), dX.view(torch.int16))


@pytest.mark.parametrize("d_in,d_out,n,T", [(4096, 512, 4096, 300), (3 * 2048, 384, 2048, 129), (4096, 256, 4096, 8)])
def test_dense_forward_fused_transform(d_in, d_out, n, T):
    """The dense forward with Hadamard blocks of 2048 / 4096 writes Z from extra warps of the GEMM launch: Z bit for
    bit what the standalone transform gives, Y and dX against the oracle (ragged token counts, several blocks)."""
    import torch

    W = _W()
    L = synth_layer(41, d_in, d_out, n, T, d_out * 24, "bf16", bits=4, group=128, pattern="random")
    a = device_adapter(d_in, d_out, n, L["rp"], L["ci"], L["cf"], algo="dense")
    wq = dev_qweight(L)
    Xd, dYd = dev_act(L["X"], "bf16"), dev_act(L["dY"], "bf16")
    Z, Y = W.adapter_fwd(a, Xd, 0.9, wq=wq)
    dc, dX = W.adapter_bwd(a, dYd, Z, 0.9, wq=wq)
    Zs = W.fwht(Xd, n)
    torch.cuda.synchronize()
    assert torch.equal(Z, Zs)
    Wq = oracle.dequant(L["qweight"], L["scales"], L["zeros"], 4, 128, d_out, d_in)
    _, Yr = oracle.adapter_fwd(L["rp"], L["ci"], L["cf"], L["X"], d_out, n, 0.9, Wq, want_z=False)
    dXr = oracle.adapter_bwd_dx(L["rp"], L["ci"], L["cf"], L["dY"], d_in, n, 0.9, Wq)
    errs = dict(Y=rel_fro(host(Y), Yr), dX=rel_fro(host(dX), dXr))
    assert all(v <= TOL_BF16 for v in errs.values()), errs


def test_dense_long_rows_with_base():
    """W_eff for rows with more nonzeros than the transform stages per row block
    (700 per row; the rest is read straight from the CSR arrays), 4-bit g128."""
    import torch

    W = _W()
    d_in, d_out, n, T = 4096, 96, 4096, 40
    L = synth_layer(39, d_in, d_out, n, T, d_out * 700, "bf16", bits=4, group=128, pattern="random")
    a = device_adapter(d_in, d_out, n, L["rp"], L["ci"], L["cf"], algo="dense")
    wq = dev_qweight(L)
    Xd, dYd = dev_act(L["X"], "bf16"), dev_act(L["dY"], "bf16")
    Z, Y = W.adapter_fwd(a, Xd, 0.7, wq=wq)
    dc, dX = W.adapter_bwd(a, dYd, Z, 0.7, wq=wq)
    torch.cuda.synchronize()
    Wq = oracle.dequant(L["qweight"], L["scales"], L["zeros"], 4, 128, d_out, d_in)
    _, Yr = oracle.adapter_fwd(L["rp"], L["ci"], L["cf"], L["X"], d_out, n, 0.7, Wq, want_z=False)
    dXr = oracle.adapter_bwd_dx(L["rp"], L["ci"], L["cf"], L["dY"], d_in, n, 0.7, Wq)
    assert np.diff(L["rp"]).min() > 512
    errs = dict(Y=rel_fro(host(Y), Yr), dX=rel_fro(host(dX), dXr))
    assert all(v <= TOL_BF16 for v in errs.values()), errs


def test_workspace_and_dtype_errors():
    import torch

    W = _W()
    L = synth_layer(36, 256, 256, 256, 16, 512, "bf16", pattern="random")
    a = device_adapter(256, 256, 256, L["rp"], L["ci"], L["cf"])
    Xd = dev_act(L["X"], "bf16")
    with pytest.raises(W.QwhaError) as ei:
        W.adapter_fwd(a, Xd, 1.0, wq=dev_qweight(L), ws=torch.empty(256, dtype=torch.uint8, device="cuda"))
    assert ei.value.status == 4
    with pytest.raises(W.QwhaError) as ei:
        W.adapter_fwd(a, to_dev(L["X"]), 1.0, wq=dev_qweight(L))  # base GEMM needs bf16
    assert ei.value.status == 3


def test_dense_rejects_fp32():
    W = _W()
    L = synth_layer(38, 256, 256, 256, 16, 512, "f32", pattern="random")
    a = device_adapter(256, 256, 256, L["rp"], L["ci"], L["cf"], algo="dense")
    with pytest.raises(W.QwhaError) as ei:
        W.adapter_fwd(a, to_dev(L["X"]), 1.0)
    assert ei.value.status == 3


@pytest.mark.parametrize("algo", ["sparse", "dense"])
def test_token_shards_give_the_same_rows_bitwise(algo):
    """Token data parallelism hands each rank a slice of the step's tokens. The per-token outputs of a slice (Z, Y, dX)
    are bit for bit the same rows of the whole call, also for slices that start inside a token tile: the sparse
    products' entry order depends on E alone and every token is summed in the same order wherever it sits in a tile.
    Only dc, a sum over tokens, is split across ranks."""
    import torch

    W = _W()
    d_in, d_out, n, T = 1024, 768, 1024, 300
    L = synth_layer(39, d_in, d_out, n, T, d_out * 8, "bf16", bits=4, group=128)
    a = device_adapter(d_in, d_out, n, L["rp"], L["ci"], L["cf"], algo=algo)
    wq = dev_qweight(L)
    Xd, dYd = dev_act(L["X"], "bf16"), dev_act(L["dY"], "bf16")
    Z, Y = W.adapter_fwd(a, Xd, 0.8, wq=wq)
    _, dX = W.adapter_bwd(a, dYd, Z, 0.8, wq=wq, want_dc=False)
    for lo, hi in ((0, 129), (129, 300)):
        Zs, Ys = W.adapter_fwd(a, Xd[lo:hi].contiguous(), 0.8, wq=wq)
        _, dXs = W.adapter_bwd(a, dYd[lo:hi].contiguous(), Zs, 0.8, wq=wq, want_dc=False)
        torch.cuda.synchronize()
        for name, part, whole in (("Z", Zs, Z), ("Y", Ys, Y), ("dX", dXs, dX)):
            assert torch.equal(part.view(torch.int16), whole[lo:hi].view(torch.int16)), (name, lo, hi)


# Shapes for the sliced SpMM's layouts (sparse algorithm): the 8-token tile (rows too wide for 16
# tokens: 8192 bf16 or 4096 fp32 columns) and output windows whose last one is partial (the kernel
# ranks segments within windows of 1024 or 2048 output columns, 32- or 16-segment groups).
SLICED_CASES = [
    # d_in, d_out, n, T, p per row, dtype
    (8192, 2600, 4096, 50, 20, "bf16"),  # forward: 8-token tile, windows 2048 + 552; gather: 4 windows
    (4096, 4616, 4096, 40, 24, "bf16"),  # forward: 16-token tile, windows 4 x 1024 + 520
    (4096, 3000, 2048, 30, 16, "f32"),  # fp32 forward: 8-token tile, windows 2048 + 952
]


@pytest.mark.parametrize("d_in,d_out,n,T,per_row,dtype", SLICED_CASES)
def test_sliced_spmm_tiles_and_windows(d_in, d_out, n, T, per_row, dtype):
    """Y, dX (the SpMM and the CSC gather) and dc of the sparse algorithm against the oracle at shapes that reach
    the 8-token tile and partial output windows, with rows of uneven length (so that the length ranking and
    the group padding matter) and a few empty and full rows."""
    import torch

    W = _W()
    g = rng_for(37, "sliced", d_in, d_out, T, dtype)
    counts = g.integers(per_row // 4, 2 * per_row, d_out)
    counts[::97] = 0
    counts[5] = d_in
    rp, ci, cf = random_pattern(d_out, d_in, counts=counts, rng=g)
    X = g.standard_normal((T, d_in)).astype(np.float32)
    dY = g.standard_normal((T, d_out)).astype(np.float32)
    if dtype == "bf16":
        X, dY = bf16_bits_to_f32(f32_to_bf16_bits(X)), bf16_bits_to_f32(f32_to_bf16_bits(dY))
    a = device_adapter(d_in, d_out, n, rp, ci, cf)
    alpha = 0.7
    Xd, dYd = dev_act(X, dtype), dev_act(dY, dtype)
    Z, Y = W.adapter_fwd(a, Xd, alpha)
    dc, dX = W.adapter_bwd(a, dYd, Z, alpha)
    torch.cuda.synchronize()
    _, Yr = oracle.adapter_fwd(rp, ci, cf, X, d_out, n, alpha, want_z=False)
    dXr = oracle.adapter_bwd_dx(rp, ci, cf, dY, d_in, n, alpha)
    rows = oracle.csr_rows(rp)
    sel = np.sort(rng_for(38, "sliced-dc").choice(ci.size, min(ci.size, 3000), replace=False))
    dcr = oracle.adapter_bwd_dc(X, dY, rows[sel], ci[sel], n, alpha)
    tol = TOL_F32 if dtype == "f32" else TOL_BF16
    errs = dict(Y=rel_fro(host(Y), Yr), dX=rel_fro(host(dX), dXr), dc=rel_fro(dc.cpu().numpy()[sel], dcr))
    assert all(v <= tol for v in errs.values()), errs
    # every output column, the empty rows' zeros included, against the oracle column by column
    Yh = host(Y)
    assert np.abs(Yh[:, counts == 0]).max() == 0.0
    col_err = np.abs(Yh - Yr).max(axis=0) / (np.abs(Yr).max() + 1e-30)
    assert col_err.max() <= (1e-5 if dtype == "f32" else 4e-2), (int(col_err.argmax()), float(col_err.max()))
