"""Value Refinement on the GPU (qwha_calib_hessian, qwha_refine_values) against the oracle.

The oracle gets the Hessian S = X^T X in fp64 from the same bf16 calibration rows
(a numpy product), the GPU forms it in fp32 on the tensor cores. The values are
compared by relative Frobenius norm: see REFINE_TOL."""

import numpy as np
import pytest

import oracle
from _util import bf16_dev, rel_fro, to_dev
from workloads import CONFIGS, bf16_bits_to_f32, f32_to_bf16_bits, layer_inputs, rng_for

pytestmark = pytest.mark.gpu

# The solve amplifies the input errors (S from fp32 accumulation of exact bf16 products, ~1e-6 relative; the
# dW_Q S product from three split-bf16 tensor-core passes, ~1e-5; the fp32 transforms, ~1e-6) by the
# conditioning of G[E, E]. Measured errors on these layers are 3e-6 .. 8e-6 (the full q_proj layer included);
# the bound leaves a margin of about 12x.
REFINE_TOL = 1e-4


def _layer(seed, d_out, d_in, n, T, per):
    g = rng_for(seed, "refine-gpu", d_out, d_in, n, T)
    w = (g.standard_normal((d_out, d_in)) * 0.01).astype(np.float32)
    X = g.standard_normal((T, d_in)).astype(np.float32)
    X[:, g.choice(d_in, max(1, d_in // 100), replace=False)] *= np.float32(20.0)
    Xb = f32_to_bf16_bits(X)
    e = oracle.init_alloc(w, d_out * per, n, 2, "fewest")
    return w, Xb, bf16_bits_to_f32(Xb).astype(np.float64), e


@pytest.mark.parametrize(
    "d_out,d_in,n,T,per,damp",
    [
        (96, 256, 256, 1024, 12, 0.01),
        (200, 512, 128, 700, 40, 0.01),  # block-diagonal H, rows with more than 32 entries (several blocks)
        (64, 128, 128, 512, 90, 0.0),  # undamped, T > d_in
    ],
)
def test_refine_matches_oracle(d_out, d_in, n, T, per, damp):
    import torch
    import walsh_hadamard_sparse_b200 as W

    w, Xb, X, e = _layer(90, d_out, d_in, n, T, per)
    S = W.calib_hessian(bf16_dev(Xb))
    c = W.refine_values(to_dev(w), S, to_dev(e["row_ptr"]), to_dev(e["col_idx"]), n, damp)
    torch.cuda.synchronize()
    Sr = X.T @ X
    ref = oracle.refine_values(w, Sr, e["row_ptr"], e["col_idx"], n, damp)
    assert rel_fro(S.cpu().numpy().astype(np.float64), Sr) < 1e-5
    err = rel_fro(c.cpu().numpy().astype(np.float64), ref.astype(np.float64))
    print("refine rel err", err)
    assert np.isfinite(c.cpu().numpy()).all() and err <= REFINE_TOL, err


def test_refine_identity_hessian_gives_dense_solution():
    import torch
    import walsh_hadamard_sparse_b200 as W

    d_out, d_in, n = 80, 256, 256
    w, _, _, e = _layer(91, d_out, d_in, n, 8, 20)
    S = torch.eye(d_in, dtype=torch.float32, device="cuda")
    c = W.refine_values(to_dev(w), S, to_dev(e["row_ptr"]), to_dev(e["col_idx"]), n, 0.0)
    torch.cuda.synchronize()
    assert rel_fro(c.cpu().numpy().astype(np.float64), e["coef"].astype(np.float64)) < 1e-5


@pytest.mark.slow
def test_refine_full_size_q_proj():
    """q_proj (4096 x 4096, p = 524288 from AdaAlloc) refined with its 8192 workload tokens as calibration rows;
    the oracle solves 16 sampled channels."""
    import torch
    import walsh_hadamard_sparse_b200 as W

    spec = CONFIGS["q_proj"][0]
    d = layer_inputs(spec, 0, "q_proj", parts=("W", "X"))
    e = oracle.init_alloc(d["dWq"], spec.p, spec.had_block, spec.min_per_row, spec.remainder)
    S = W.calib_hessian(bf16_dev(d["X_bits"]))
    c = W.refine_values(torch.from_numpy(d["dWq"]).cuda(), S, to_dev(e["row_ptr"]), to_dev(e["col_idx"]),
                        spec.had_block, 0.01)
    torch.cuda.synchronize()
    X = d["X"].astype(np.float64)
    rows = np.sort(rng_for(92, "refine-full").choice(spec.d_out, 16, replace=False)).astype(np.int32)
    ref = oracle.refine_values(d["dWq"], X.T @ X, e["row_ptr"], e["col_idx"], spec.had_block, 0.01, rows=rows)
    m = np.isfinite(ref)
    got = c.cpu().numpy()
    err = rel_fro(got[m].astype(np.float64), ref[m].astype(np.float64))
    print("full-size refine rel err", err, "entries", int(m.sum()))
    assert np.isfinite(got).all() and err <= REFINE_TOL, err
