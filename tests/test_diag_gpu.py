"""Selection diagnostics on the GPU against the oracle: the row and column counts of E with the rank bound they
give (bit for bit), and the Hill exponent and cumulative energy of the transform coefficients of dW_Q (the
threshold bit for bit, the sums to 1e-9 relative). E comes from the oracle's AdaAlloc, whole-matrix magnitude
and seeded random selections, the pages' three rules (papernotes.org "QWHA", 关键设计 1 and 2)."""

import json
import os

import numpy as np
import pytest

import oracle
from _util import to_dev
from workloads import CONFIGS, layer_inputs, random_pattern, rng_for

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
NAMES = ("empty_rows", "empty_cols", "min_row", "max_row", "min_col", "max_col", "rank_bound", "half_rows")


def _check_pattern(rp, ci, d_in):
    import walsh_hadamard_sparse_b200 as W

    st, cc = W.pattern_stats(to_dev(rp), to_dev(ci) if ci.size else to_dev(np.zeros(1, np.int32))[:0], d_in)
    got = dict(zip(NAMES, st.cpu().numpy().tolist()))
    ref = oracle.pattern_stats(rp, ci, d_in)
    assert got == {k: ref[k] for k in NAMES}
    assert np.array_equal(cc.cpu().numpy(), ref["col_counts"])
    return got


def _layer_dwq(d_out, d_in, seed):
    g = rng_for(seed, "diag-layer", d_out, d_in)
    w = g.standard_normal((d_out, d_in)).astype(np.float32) * np.float32(0.02)
    w[g.random((d_out, d_in)) < 0.001] *= np.float32(20.0)  # outliers, as in the workloads
    from workloads import quantize_rtn

    return quantize_rtn(w, 4, 128)[4]


def test_pattern_stats_golden_and_edge_patterns():
    g = json.load(open(os.path.join(GOLDEN, "pattern_stats.json")))
    rows = g["rows"]
    rp = np.zeros(len(rows) + 1, np.int32)
    rp[1:] = np.cumsum([len(r) for r in rows])
    ci = np.array([k for r in rows for k in r], np.int32)
    assert _check_pattern(rp, ci, g["d_in"]) == g["stats"]
    rng = rng_for(90, "diag-edge")
    c = rng.integers(0, 9, 300)
    c[::7] = 0
    c[5] = 700
    _check_pattern(*random_pattern(300, 700, counts=c, rng=rng)[:2], 700)  # empty and full rows
    _check_pattern(*random_pattern(40, 5000, p=120, rng=rng)[:2], 5000)  # most columns empty
    _check_pattern(np.zeros(17, np.int32), np.zeros(0, np.int32), 33)  # no entries at all


@pytest.mark.parametrize("d_out,d_in,n", [(512, 1024, 1024), (384, 768, 256)])
def test_pattern_stats_of_the_three_selections(d_out, d_in, n):
    """AdaAlloc, whole-matrix magnitude and random E of one layer: counts bit for bit, and the GPU's rank bound
    holds the oracle's numerical rank of F."""
    w = _layer_dwq(d_out, d_in, 91)
    p = 16 * (d_in + d_out)
    sels = {"adaalloc": oracle.init_alloc(w, p, n, 2, "fewest"),
            "magnitude": oracle.init_select_global(w, p, n, "magnitude"),
            "random": oracle.init_select_global(w, p, n, "random", 7)}
    for name, e in sels.items():
        got = _check_pattern(e["row_ptr"], e["col_idx"], d_in)
        assert oracle.numerical_rank(e["row_ptr"], e["col_idx"], e["coef"], d_in) <= got["rank_bound"], name
        if name == "adaalloc":
            assert got["empty_rows"] == 0 and got["min_row"] >= 2  # the per-channel floor


def _check_energy(w, k, n):
    import torch
    import walsh_hadamard_sparse_b200 as W

    got = W.energy_stats(torch.from_numpy(np.ascontiguousarray(w)).cuda(), k, n).cpu().numpy()
    ref = oracle.energy_stats(w, k, n)
    assert got[2] == ref["threshold"]
    for i, key in ((3, "total"), (1, "energy"), (0, "eta")):
        if np.isnan(ref[key]):
            assert np.isnan(got[i]), key
        else:
            assert abs(got[i] - ref[key]) <= 1e-9 * abs(ref[key]), (key, got[i], ref[key])
    return got


def test_energy_stats_small_cases():
    w = np.zeros((4, 16), np.float32)
    for r, (s, k) in enumerate(((8.0, 3), (2.0, 10), (0.5, 6), (0.0, 0))):
        w[r, k] = s
    for k in (16, 20, 40, 50):  # the closed-form spike rows, ties at the threshold, a zero threshold
        _check_energy(w, k, 16)
    _check_energy(w, 8, 8)  # block-diagonal
    ties = rng_for(92, "energy-ties").integers(-2, 3, (96, 128)).astype(np.float32)
    for k in (1, 500, 5000):
        _check_energy(ties, k, 128)
    w = _layer_dwq(512, 1024, 93)
    for k, n in ((16 * 1536, 1024), (1, 1024), (512 * 1024 - 1, 256)):
        _check_energy(w, k, n)


@pytest.mark.slow
def test_diagnostics_full_size_q_proj():
    """The q_proj layer (4096 x 4096, 4-bit g128, p = 524288): eta and the energy of the p largest coefficients,
    and the counts of E under the three rules."""
    spec = CONFIGS["q_proj"][0]
    w = layer_inputs(spec, 0, "q_proj", parts=("W",))["dWq"]
    _check_energy(w, spec.p, spec.had_block)
    for e in (oracle.init_alloc(w, spec.p, spec.had_block, 2, spec.remainder),
              oracle.init_select_global(w, spec.p, spec.had_block, "magnitude")):
        _check_pattern(e["row_ptr"], e["col_idx"], spec.d_in)
