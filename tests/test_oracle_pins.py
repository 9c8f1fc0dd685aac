"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each test ties one oracle function to something independent of it: a
hand-written golden fixture, a textbook construction from a library
(scipy.linalg.hadamard, scipy.sparse), a closed form, an identity of the
mathematics (orthonormality, adjointness, linearity), finite differences, or
brute force over every subset on tiny shapes. A plausible slip in the oracle
(a wrong sign, index, stage order, scale, transposed operand, dropped term)
fails at least one of them.
"""

import itertools
import json
import os

import numpy as np
import pytest
import scipy.linalg
import scipy.sparse

import oracle
from workloads import CONFIGS, layer_inputs, pack_codes, quantize_rtn, random_pattern, rng_for

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def H_ref(n):
    return scipy.linalg.hadamard(n).astype(np.float64) / np.sqrt(n)


def H_block(d, n):
    return scipy.linalg.block_diag(*([H_ref(n)] * (d // n)))


def F_dense(row_ptr, col_idx, coef, d_out, d_in):
    F = np.zeros((d_out, d_in))
    for r in range(d_out):
        for j in range(row_ptr[r], row_ptr[r + 1]):
            F[r, col_idx[j]] += coef[j]
    return F


def rel(a, b):
    return np.linalg.norm(np.asarray(a) - np.asarray(b)) / max(np.linalg.norm(b), 1e-300)


# ---------------------------------------------------------------- Hadamard


def test_hadamard_golden_h4():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "hadamard_4.txt")) if not l.startswith("#")]
    g = np.array(rows, dtype=np.float64)
    assert np.array_equal(oracle.hadamard(4) * 2.0, g)


@pytest.mark.parametrize("n", [1, 2, 4, 8, 16, 64, 256, 1024])
def test_hadamard_is_sylvester(n):
    assert np.array_equal(oracle.hadamard(n) * np.sqrt(n), scipy.linalg.hadamard(n).astype(np.float64))


@pytest.mark.parametrize("n", [2, 32, 512])
def test_hadamard_orthonormal_symmetric_involutory(n):
    H = oracle.hadamard(n)
    assert np.array_equal(H, H.T)
    assert np.abs(H @ H - np.eye(n)).max() < 1e-13


@pytest.mark.parametrize("n", [2, 8, 128, 2048])
def test_fwht_of_unit_vectors_is_h(n):
    # row e_k through the transform gives row k of H, exactly
    I = np.eye(n)
    assert np.array_equal(oracle.fwht(I, n), oracle.hadamard(n))


@pytest.mark.parametrize("d,n", [(256, 256), (448, 64), (7 * 32, 32), (16, 2), (4096, 4096)])
def test_fwht_and_dense_transform_match_library_hadamard(d, n):
    X = rng_for(1, "fwht", d, n).standard_normal((5, d))
    ref = X @ H_block(d, n)
    assert rel(oracle.fwht(X, n), ref) < 1e-13
    if d <= 512:
        assert rel(oracle.transform_dense(X, n), ref) < 1e-13


def test_fwht_unnormalised_integer_exact():
    X = rng_for(2, "fwht_int").integers(-50, 50, size=(9, 64)).astype(np.float64)
    assert np.array_equal(oracle.fwht(X, 64, normalize=False), X @ scipy.linalg.hadamard(64))


def test_fwht_parseval_involution_constant():
    n = 1024
    X = rng_for(3, "parseval").standard_normal((4, n))
    Z = oracle.fwht(X, n)
    assert np.allclose(np.linalg.norm(Z, axis=1), np.linalg.norm(X, axis=1), rtol=1e-13)
    assert rel(oracle.fwht(Z, n), X) < 1e-13
    c = oracle.fwht(np.ones((1, n)), n)[0]
    assert c[0] == pytest.approx(np.sqrt(n), rel=1e-15) and np.all(c[1:] == 0.0)


def test_fwht_textbook_stage_order():
    # The ranking transform must sum in the textbook order h = 1, 2, ...: for n = 4,
    # output 0 is (x0 + x1) + (x2 + x3), not (x0 + x2) + (x1 + x3). The values are
    # chosen so that the two orders round to different doubles (2^-53 vs 2^-52).
    x = np.array([[1.0, 2.0**-53, -1.0, 2.0**-53]])
    v = oracle.fwht(x, 4, normalize=False)[0, 0]
    textbook = (1.0 + 2.0**-53) + (-1.0 + 2.0**-53)
    other = (1.0 + -1.0) + (2.0**-53 + 2.0**-53)
    assert textbook != other
    assert v == textbook


# ---------------------------------------------------------------- base weight


def test_packing_and_dequant_golden():
    g = json.load(open(os.path.join(GOLDEN, "packing.json")))
    for c in g["cases"]:
        codes = np.array([c["codes"]], dtype=np.uint8)
        assert list(pack_codes(codes, c["bits"])[0]) == c["bytes"]
        # oracle unpacking of the hand-packed bytes with s = 1, z = 0 returns the codes
        n = len(c["codes"])
        W = oracle.dequant(np.array([c["bytes"]], np.uint8), np.ones((1, 1), np.float32),
                           np.zeros((1, 1), np.uint8), c["bits"], n, 1, n)
        assert list(W[0]) == [float(v) for v in c["codes"]]
    d = g["dequant"]
    qb = pack_codes(np.array([d["codes"]], np.uint8), d["bits"])
    W = oracle.dequant(qb, np.array([[d["scale"]]], np.float32), np.array([[d["zero"]]], np.uint8),
                       d["bits"], d["group"], 1, len(d["codes"]))
    assert list(W[0]) == d["values"]


@pytest.mark.parametrize("bits,group", [(2, 64), (3, 128), (4, 64), (4, 128)])
def test_dequant_matches_quantizer_and_error_bound(bits, group):
    w = rng_for(4, "q", bits).standard_normal((16, 512)).astype(np.float32) * np.float32(0.02)
    w[3, 7] = 0.9  # an outlier inflates its group's step
    q, s, z, wq, dwq = quantize_rtn(w, bits, group)
    W = oracle.dequant(pack_codes(q, bits), s, z, bits, group, 16, 512)
    assert np.array_equal(W, wq.astype(np.float64))
    assert q.max() <= 2**bits - 1
    step = np.repeat(s, group, axis=1)
    inside = (q > 0) & (q < 2**bits - 1)
    assert np.all(np.abs(dwq[inside]) <= step[inside] * 0.5 * (1 + 1e-6))
    assert np.array_equal(dwq, (w - wq).astype(np.float32))


# ---------------------------------------------------------------- forward


def _layer(seed, d_out, d_in, n, p, T, with_wq=True):
    g = rng_for(seed, "layer", d_out, d_in, n, p, T)
    rp, ci, cf = random_pattern(d_out, d_in, p=p, rng=g)
    X = g.standard_normal((T, d_in))
    dY = g.standard_normal((T, d_out))
    Wq = g.standard_normal((d_out, d_in)) * 0.02 if with_wq else None
    return rp, ci, cf, X, dY, Wq


@pytest.mark.parametrize("d_out,d_in,n,p,T", [(24, 64, 64, 150, 7), (40, 96, 32, 300, 5), (8, 16, 16, 128, 3)])
def test_forward_matches_numpy_definition(d_out, d_in, n, p, T):
    rp, ci, cf, X, _, Wq = _layer(5, d_out, d_in, n, p, T)
    alpha = 0.75
    Z, Y = oracle.adapter_fwd(rp, ci, cf, X, d_out, n, alpha, Wq)
    H = H_block(d_in, n)
    dW = F_dense(rp, ci, cf, d_out, d_in) @ H
    assert rel(Z, X @ H) < 1e-13
    assert rel(Y, X @ Wq.T + alpha * X @ dW.T) < 1e-12
    assert rel(oracle.delta_w(rp, ci, cf, d_out, d_in, n), dW) < 1e-13
    Ys = oracle.adapter_fwd_sparse(rp, ci, cf, X, d_out, n, alpha)
    assert rel(Ys, alpha * (X @ H) @ F_dense(rp, ci, cf, d_out, d_in).T) < 1e-12


def test_single_nonzero_closed_form():
    # F = c e_r e_k^T  ->  dW[r, :] = c H[k, :], entries +-c/sqrt(n), other rows 0
    n, r, k, c = 16, 2, 5, 3.0
    rp = np.array([0, 0, 0, 1, 1], np.int32)
    dW = oracle.delta_w(rp, np.array([k], np.int32), np.array([c]), 4, n, n)
    sign = np.array([(-1) ** bin(k & i).count("1") for i in range(n)], dtype=np.float64)
    assert np.array_equal(dW[r], c * sign / 4.0)
    assert np.all(dW[[0, 1, 3]] == 0)


# ---------------------------------------------------------------- backward


def test_dc_by_finite_differences_and_identity():
    d_out, d_in, n, p, T = 12, 32, 32, 60, 6
    rp, ci, cf, X, dY, Wq = _layer(6, d_out, d_in, n, p, T)
    alpha = 1.3
    rows = oracle.csr_rows(rp)
    dc = oracle.adapter_bwd_dc(X, dY, rows, ci, n, alpha)

    def L(c):
        return float(np.sum(oracle.adapter_fwd(rp, ci, c, X, d_out, n, alpha, Wq, want_z=False)[1] * dY))

    for j in [0, 7, 31, 59]:
        e = np.zeros(p)
        e[j] = 1.0
        fd = (L(cf + e) - L(cf - e)) / 2.0  # L is linear in c: the central difference is exact
        assert fd == pytest.approx(dc[j], rel=1e-9, abs=1e-9)
    # sum_j c_j dc_j = <Y_adapter, dY>
    Yad = oracle.adapter_fwd(rp, ci, cf, X, d_out, n, alpha, None, want_z=False)[1]
    assert float(np.dot(cf, dc)) == pytest.approx(float(np.sum(Yad * dY)), rel=1e-11)


def test_dx_adjoint_and_finite_differences():
    d_out, d_in, n, p, T = 20, 64, 16, 200, 4
    rp, ci, cf, X, dY, Wq = _layer(7, d_out, d_in, n, p, T)
    alpha = 0.6
    dX = oracle.adapter_bwd_dx(rp, ci, cf, dY, d_in, n, alpha, Wq)
    Y = oracle.adapter_fwd(rp, ci, cf, X, d_out, n, alpha, Wq, want_z=False)[1]
    # Y is linear in X: <Y(X), dY> = <X, dX>
    assert float(np.sum(Y * dY)) == pytest.approx(float(np.sum(X * dX)), rel=1e-11)
    for t, k in [(0, 0), (2, 33), (3, 63)]:
        E = np.zeros_like(X)
        E[t, k] = 1.0
        Lp = np.sum(oracle.adapter_fwd(rp, ci, cf, X + E, d_out, n, alpha, Wq, want_z=False)[1] * dY)
        Lm = np.sum(oracle.adapter_fwd(rp, ci, cf, X - E, d_out, n, alpha, Wq, want_z=False)[1] * dY)
        assert (Lp - Lm) / 2.0 == pytest.approx(dX[t, k], rel=1e-9, abs=1e-9)


# ---------------------------------------------------------------- AdaAlloc


@pytest.mark.parametrize("mode", ["fewest", "largest"])
def test_init_golden_tiny(mode):
    g = json.load(open(os.path.join(GOLDEN, "adaalloc_tiny.json")))
    w = np.array(g["dWq"], dtype=np.float32)
    out = oracle.init_alloc(w, g["p"], g["n"], g["min_per_row"], mode)
    exp = g[mode]
    assert list(out["budgets"]) == exp["budgets"]
    rp = out["row_ptr"]
    for i in range(w.shape[0]):
        assert list(out["col_idx"][rp[i] : rp[i + 1]]) == exp["col_idx"][i]
        want = np.float32(np.array(exp["coef_times_sqrt8"][i], dtype=np.float64) / np.sqrt(8.0))
        assert np.array_equal(out["coef"][rp[i] : rp[i + 1]], want)


def test_init_brute_force_subsets():
    # For orthonormal H, ||w - x H_S||^2 is minimised over |S| = b by the b largest
    # |(w H)_k|, with x the least-squares values. Check against every subset.
    d_out, d_in, n = 6, 8, 8
    w = rng_for(8, "brute").standard_normal((d_out, d_in)).astype(np.float32)
    out = oracle.init_alloc(w, 20, n, 2, "fewest")
    H = H_ref(n)
    rp, ci, cf = out["row_ptr"], out["col_idx"], out["coef"]
    for i in range(d_out):
        b = int(out["budgets"][i])
        wi = w[i].astype(np.float64)
        best, best_S = np.inf, None
        for S in itertools.combinations(range(d_in), b):
            A = H[list(S), :]
            x, *_ = np.linalg.lstsq(A.T, wi, rcond=None)
            err = float(np.sum((wi - x @ A) ** 2))
            if err < best - 1e-12:
                best, best_S = err, S
        assert tuple(ci[rp[i] : rp[i + 1]]) == best_S
        x, *_ = np.linalg.lstsq(H[list(best_S), :].T, wi, rcond=None)
        assert np.allclose(cf[rp[i] : rp[i + 1]], x, rtol=1e-6, atol=1e-7)


@pytest.mark.parametrize("mode", ["fewest", "largest"])
def test_init_tiny_workload_invariants(mode):
    spec = CONFIGS["tiny"][0]
    d = layer_inputs(spec, 0, "tiny", parts=("W",))
    w = d["dWq"]
    out = oracle.init_alloc(w, spec.p, spec.had_block, 2, mode)
    b, rp, ci, cf = out["budgets"], out["row_ptr"], out["col_idx"], out["coef"]
    assert b.sum() == spec.p and b.min() >= 2 and b.max() <= spec.d_in
    assert rp[0] == 0 and np.array_equal(np.diff(rp), b)
    # budgets follow the error norms: the floor share plus at most one remainder unit
    e = np.linalg.norm(w.astype(np.float64), axis=1)
    assert np.allclose(out["err_norm"], e, rtol=1e-14)
    share = 2 + (spec.p - 2 * spec.d_out) * e / e.sum()
    assert np.all(b >= np.floor(share) - 1e-9) and np.all(b <= np.floor(share) + 1)
    # selection equals a numpy ranking of the library transform (no ties in this data)
    V = w.astype(np.float64) @ scipy.linalg.hadamard(spec.had_block)
    for i in range(spec.d_out):
        order = np.lexsort((np.arange(spec.d_in), -np.abs(V[i])))
        assert np.array_equal(ci[rp[i] : rp[i + 1]], np.sort(order[: b[i]]))
    # ||dW_Q - F H||^2 = ||dW_Q||^2 - sum c^2 (orthonormal H, dense-solution values)
    F = F_dense(rp, ci, cf.astype(np.float64), spec.d_out, spec.d_in)
    resid = np.sum((w.astype(np.float64) - F @ H_ref(spec.had_block)) ** 2)
    assert resid == pytest.approx(np.sum(w.astype(np.float64) ** 2) - np.sum(cf.astype(np.float64) ** 2), rel=1e-6)


def test_init_block_diagonal_and_all_zero():
    # d_in = 3 blocks of 8: the transform is per block
    w = rng_for(9, "blk").standard_normal((5, 24)).astype(np.float32)
    out = oracle.init_alloc(w, 40, 8, 2, "largest")
    V = w.astype(np.float64) @ scipy.linalg.block_diag(*[scipy.linalg.hadamard(8)] * 3)
    rp = out["row_ptr"]
    for i in range(5):
        order = np.lexsort((np.arange(24), -np.abs(V[i])))
        assert np.array_equal(out["col_idx"][rp[i] : rp[i + 1]], np.sort(order[: out["budgets"][i]]))
    z = oracle.init_alloc(np.zeros((4, 16), np.float32), 13, 16, 2, "fewest")
    assert list(z["budgets"]) == [4, 3, 3, 3]  # pool 5 shared equally: 1 each, remainder 1 to row 0
    assert np.all(z["coef"] == 0)
    assert list(z["col_idx"][:4]) == [0, 1, 2, 3]


def test_init_rejects_bad_budgets():
    w = np.zeros((4, 8), np.float32)
    with pytest.raises(ValueError):
        oracle.init_alloc(w, 7, 8, 2)  # below 2 per row
    with pytest.raises(ValueError):
        oracle.init_alloc(w, 33, 8, 2)  # above d_in * d_out
    with pytest.raises(ValueError):
        oracle.init_alloc(np.zeros((4, 12), np.float32), 10, 8, 2)  # 12 not a multiple of 8


# ---------------------------------------------------------------- plan


def test_plan_build_matches_scipy_csc():
    d_out, d_in = 37, 53
    rp, ci, _ = random_pattern(d_out, d_in, p=400, rng=rng_for(10, "plan"))
    cp, ri, pm = oracle.plan_build(rp, ci, d_in)
    M = scipy.sparse.csr_matrix((np.arange(1, 401, dtype=np.float64), ci, rp), shape=(d_out, d_in)).tocsc()
    M.sort_indices()
    assert np.array_equal(cp, M.indptr) and np.array_equal(ri, M.indices)
    assert np.array_equal(pm, M.data.astype(np.int64) - 1)


# --------------------------------------------------------------------------- selection over the whole matrix

MASK64 = (1 << 64) - 1


def splitmix64(seed, n):
    """Output n (n >= 1) of SplitMix64 seeded with `seed`, from the generator's published definition."""
    z = (seed + n * 0x9E3779B97F4A7C15) & MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
    return z ^ (z >> 31)


def test_splitmix64_published_outputs():
    # the first outputs of the reference generator for seed 0, and the first for seed 1234567
    assert [splitmix64(0, n) for n in (1, 2, 3)] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]
    assert splitmix64(1234567, 1) == 6457827717110365317


def _expected_global(w, n, p, keys_lex):
    """CSR of the p flat positions first in np.lexsort order of keys_lex (last key primary)."""
    d_out, d_in = w.shape
    order = np.lexsort(keys_lex)
    pick = np.sort(order[:p])
    rows, cols = pick // d_in, pick % d_in
    budgets = np.bincount(rows, minlength=d_out).astype(np.int32)
    rp = np.concatenate([[0], np.cumsum(budgets)]).astype(np.int32)
    V = w.astype(np.float64) @ scipy.linalg.block_diag(*[scipy.linalg.hadamard(n)] * (d_in // n)).astype(np.float64)
    coef = (V.reshape(-1)[pick] * (1.0 / np.sqrt(n))).astype(np.float32)  # c = float(V * (1/sqrt(n)))
    return budgets, rp, cols.astype(np.int32), coef


@pytest.mark.parametrize("kind", ["normal", "ties"])
def test_select_global_magnitude_matches_sort(kind):
    g = rng_for(70, "global-mag", kind)
    d_out, d_in, n, p = 24, 64, 32, 150
    if kind == "ties":  # small integers: many equal |V|, the tie rule decides
        w = g.integers(-1, 2, size=(d_out, d_in)).astype(np.float32)
    else:
        w = g.standard_normal((d_out, d_in)).astype(np.float32)
    V = w.astype(np.float64) @ scipy.linalg.block_diag(*[scipy.linalg.hadamard(n)] * (d_in // n))
    flat = np.arange(d_out * d_in)
    b, rp, ci, cf = _expected_global(w, n, p, (flat, -np.abs(V.reshape(-1))))
    got = oracle.init_select_global(w, p, n, "magnitude")
    assert np.array_equal(got["budgets"], b) and np.array_equal(got["row_ptr"], rp)
    assert np.array_equal(got["col_idx"], ci)
    assert np.array_equal(got["coef"].view(np.uint32), cf.view(np.uint32))


def test_select_global_random_matches_generator():
    g = rng_for(71, "global-rand")
    d_out, d_in, n, p, seed = 20, 32, 32, 97, 0xDEADBEEF12345
    w = g.standard_normal((d_out, d_in)).astype(np.float32)
    flat = np.arange(d_out * d_in)
    u = np.array([splitmix64(seed, int(j) + 1) for j in flat], dtype=np.uint64)
    b, rp, ci, cf = _expected_global(w, n, p, (flat, u))
    got = oracle.init_select_global(w, p, n, "random", seed)
    assert np.array_equal(got["budgets"], b) and np.array_equal(got["row_ptr"], rp)
    assert np.array_equal(got["col_idx"], ci)
    assert np.array_equal(got["coef"].view(np.uint32), cf.view(np.uint32))
    # a uniform p-subset: another seed gives another one, with the same count
    other = oracle.init_select_global(w, p, n, "random", seed + 1)
    assert other["row_ptr"][-1] == p and not np.array_equal(other["col_idx"], got["col_idx"])


# --------------------------------------------------------------------------- value refinement


def _refine_case(seed, d_out=20, d_in=64, n=32, per=7, T=300):
    g = rng_for(seed, "refine")
    w = (g.standard_normal((d_out, d_in)) * 0.01).astype(np.float32)
    e = oracle.init_alloc(w, d_out * per, n, 2, "fewest")
    X = g.standard_normal((T, d_in))
    X[:, g.choice(d_in, 3, replace=False)] *= 20.0  # outlier input channels, as in the workloads
    return w, e, X.T @ X


def test_refine_identity_hessian_is_dense_solution():
    # the page: with R proportional to I the refinement changes nothing (x* = x0), for any scale of S
    w, e, _ = _refine_case(80)
    d_in = w.shape[1]
    for scale in (1.0, 7.5):
        c = oracle.refine_values(w, scale * np.eye(d_in), e["row_ptr"], e["col_idx"], 32)
        assert np.array_equal(c.view(np.uint32), e["coef"].view(np.uint32))


def test_refine_matches_least_squares_on_the_page_formulation():
    """x* from an independent route: R = U Sigma^(1/2) from an eigendecomposition of the (damped) Hessian,
    v = dW_Q[i,:] R, B = H^-1 R with H from scipy, and numpy's least squares over the selected rows of B."""
    w, e, S = _refine_case(81)
    d_out, d_in = w.shape
    damp = 0.01
    Sd = S + damp * np.trace(S) / d_in * np.eye(d_in)
    lam, U = np.linalg.eigh(Sd)
    R = U * np.sqrt(lam)
    Hinv = H_block(d_in, 32)  # orthonormal, its own inverse
    B = Hinv @ R
    got = oracle.refine_values(w, S, e["row_ptr"], e["col_idx"], 32, damp)
    rp, ci = e["row_ptr"], e["col_idx"]
    for i in range(d_out):
        sel = ci[rp[i]:rp[i + 1]]
        v = w[i].astype(np.float64) @ R
        x, *_ = np.linalg.lstsq(B[sel].T, v, rcond=None)
        assert np.allclose(got[rp[i]:rp[i + 1]], x, rtol=1e-5, atol=1e-9), i


def test_refine_never_worse_than_dense_solution():
    # the refined values minimise the per-channel output error, so they never do worse than x0 on it
    w, e, S = _refine_case(82)
    d_out, d_in = w.shape
    H = H_block(d_in, 32)
    got = oracle.refine_values(w, S, e["row_ptr"], e["col_idx"], 32)
    rp, ci = e["row_ptr"], e["col_idx"]
    for i in range(d_out):
        sel = ci[rp[i]:rp[i + 1]]
        def err(x):
            r = w[i].astype(np.float64) - x @ H[sel]  # dW_Q[i,:] - (F H^-1)[i,:]
            return r @ S @ r  # || r X^T ||^2
        assert err(got[rp[i]:rp[i + 1]].astype(np.float64)) <= err(e["coef"][rp[i]:rp[i + 1]].astype(np.float64)) + 1e-12


# --------------------------------------------------------------------------- selection diagnostics


def _csr_from_rows(rows):
    rp = np.zeros(len(rows) + 1, dtype=np.int32)
    rp[1:] = np.cumsum([len(r) for r in rows])
    ci = np.array([k for r in rows for k in r], dtype=np.int32)
    return rp, ci


def test_pattern_stats_golden():
    """Row and column counts, empty rows and columns, the rank bound and the half-mass row count of a hand-worked
    pattern; the numerical rank of F with generic coefficients reaches the bound."""
    g = json.load(open(os.path.join(GOLDEN, "pattern_stats.json")))
    rp, ci = _csr_from_rows(g["rows"])
    got = oracle.pattern_stats(rp, ci, g["d_in"])
    assert list(got["col_counts"]) == g["col_counts"]
    assert {k: got[k] for k in g["stats"]} == g["stats"]
    coef = rng_for(80, "pattern-golden").uniform(0.5, 2.0, ci.size)
    assert oracle.numerical_rank(rp, ci, coef, g["d_in"]) == g["generic_rank"]


def test_numerical_rank_of_constructed_patterns():
    """rank(F) on patterns whose rank is known by construction: a full diagonal, all entries in two rows, two rows
    with proportional coefficients on the same columns, and a full block with outer-product values (rank 1)."""
    g = rng_for(81, "rank")
    d = 12
    rp, ci = _csr_from_rows([[i] for i in range(d)])
    assert oracle.numerical_rank(rp, ci, g.uniform(1, 2, d), d) == d
    rows = [list(range(0, 14, 1)) if i in (2, 7) else [] for i in range(9)]
    rp, ci = _csr_from_rows(rows)
    assert oracle.numerical_rank(rp, ci, g.standard_normal(ci.size), 14) == 2
    base = g.standard_normal(5)
    rows = [[1, 3, 4, 8, 9], [], [1, 3, 4, 8, 9]]
    rp, ci = _csr_from_rows(rows)
    assert oracle.numerical_rank(rp, ci, np.concatenate([base, -2.5 * base]), 10) == 1
    u, v = g.uniform(1, 2, 4), g.uniform(1, 2, 6)
    rows = [list(range(6))] * 4
    rp, ci = _csr_from_rows(rows)
    assert oracle.numerical_rank(rp, ci, np.outer(u, v).ravel(), 6) == 1
    # a wide pattern (rows fewer than columns): a transposed scatter would not fit
    rp, ci = _csr_from_rows([[0, 5], [1, 6], [2, 7]])
    assert oracle.numerical_rank(rp, ci, np.ones(6), 8) == 3


def _spike_rows(d_in, n):
    """dW_Q whose rows hold one spike each (values 8, 2, 0.5, 0; powers of two, exact in fp32): row r of
    V = dW_Q H_unnormalised is s_r times a row of the n-point Hadamard block it falls in, so n magnitudes equal |s_r|
    and the other d_in - n are zero."""
    w = np.zeros((4, d_in), dtype=np.float32)
    for r, (s, k) in enumerate(((8.0, 3), (2.0, 10), (0.5, 6), (0.0, 0))):
        w[r, k] = s
    return w


def test_energy_stats_closed_form():
    """Hill exponent and cumulative energy where the order statistics are known exactly (spike rows), for the
    full transform and for a block-diagonal one: eta = k / sum_{i<=k} ln(a_(i)/a_(k+1)), energy = sum of the k
    largest a^2 over all, NaN for eta when a_(k+1) = 0."""
    ln4, ln16 = np.log(4.0), np.log(16.0)
    w = _spike_rows(16, 16)  # magnitudes: 16 x 8, 16 x 2, 16 x 0.5, 16 x 0; total 16 * 68.25 = 1092
    cases = {
        16: (1.0 / ln4, 1024.0 / 1092, 2.0),
        20: (20.0 / (16 * ln4), 1040.0 / 1092, 2.0),
        40: (40.0 / (16 * ln16 + 16 * ln4), 1090.0 / 1092, 0.5),
        50: (np.nan, 1092.0 / 1092, 0.0),
    }
    for k, (eta, energy, thr) in cases.items():
        got = oracle.energy_stats(w, k, 16)
        assert got["threshold"] == thr and got["total"] == 1092.0, k
        assert np.isclose(got["energy"], energy, rtol=1e-14), k
        assert (np.isnan(got["eta"]) and np.isnan(eta)) or np.isclose(got["eta"], eta, rtol=1e-14), k
    # two blocks of 8: each spike fills only its own block (8 magnitudes |s_r|, the other 8 of the row zero)
    got = oracle.energy_stats(_spike_rows(16, 8), 8, 8)
    assert got["threshold"] == 2.0 and got["total"] == 8 * 68.25
    assert np.isclose(got["eta"], 1.0 / ln4, rtol=1e-14) and np.isclose(got["energy"], 64.0 / 68.25, rtol=1e-14)


def test_energy_stats_recovers_a_pareto_tail_index():
    """Coefficients drawn from a Pareto law of tail index 1.5 (random signs), mapped back to dW_Q through the
    library-independent Hadamard matrix: the Hill exponent over the 2000 largest of 65536 is within a few standard
    errors (1.5 / sqrt(2000) = 0.034) of 1.5. A reciprocal or a log-base mistake lands far away. The total
    energy obeys Parseval: sum (dW_Q H_unnormalised)^2 = n ||dW_Q||^2."""
    from scipy.linalg import hadamard

    n, d_out, alpha = 256, 256, 1.5
    g = rng_for(82, "pareto")
    V = (1.0 + g.pareto(alpha, (d_out, n))) * g.choice([-1.0, 1.0], (d_out, n))
    w = (V @ hadamard(n).astype(np.float64) / n).astype(np.float32)  # V = w H_unnormalised (up to fp32 rounding)
    got = oracle.energy_stats(w, 2000, n)
    assert abs(got["eta"] - alpha) < 0.15, got
    assert np.isclose(got["total"], n * np.sum(w.astype(np.float64) ** 2), rtol=1e-12)
    assert 0.0 < got["energy"] < 1.0
