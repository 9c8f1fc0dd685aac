"""Parity on the whole decoder-block workload: the seven LLaMA-3-8B-shaped linears
(q, k, v, o, gate, up, down) at 32768 tokens (8 x 4096), 4-bit g128 base weights,
p = 64 (d_in + d_out) per layer.

Layers that read the same input share its transform Z = X H (same X, same H):
q computes it and k, v read it (`z_given`), gate computes it and up reads it.
Every layer runs forward + backward on the GPU with both algorithms; the oracle
checks sampled token rows of Y and dX and sampled entries of dc (each needs the
full token sum), E and c coming from the oracle's own AdaAlloc."""

import numpy as np
import pytest

import oracle
from _util import TOL_BF16, bf16_dev, host, rel_fro
from workloads import CONFIGS, layer_inputs, rng_for

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def _dc_reference(spec, X, dY, rp, ci, sel):
    """Oracle dc at the CSR positions `sel`. For a block-diagonal H only the
    columns of X in the entries' Hadamard block matter, so the positions are
    drawn from one block and only its columns are handed over; likewise only
    the entries' columns of dY."""
    n = spec.had_block
    rows = oracle.csr_rows(rp)[sel]
    cols = ci[sel]
    b = int(cols[0]) // n
    assert np.all(cols // n == b)
    used = np.unique(rows)
    return oracle.adapter_bwd_dc(X[:, b * n:(b + 1) * n], dY[:, used], np.searchsorted(used, rows), cols - b * n, n,
                                 1.0)


def _pick_dc(spec, ci, g, count):
    n = spec.had_block
    blk = int(g.integers(0, spec.d_in // n))
    cand = np.nonzero(ci // n == blk)[0]
    return np.sort(g.choice(cand, min(count, cand.size), replace=False))


def test_decoder_block_with_shared_transform():
    import torch
    import walsh_hadamard_sparse_b200 as W

    specs = CONFIGS["block"]
    T = specs[0].T
    g = rng_for(61, "block-test")
    rows = np.sort(g.choice(T, 32, replace=False))
    ri = torch.as_tensor(rows).cuda()
    dv = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()  # noqa: E731
    x_stream, x_host, x_dev = None, None, None
    z_dev = {}  # x_stream -> device Z = X H, written by the first layer of that stream
    for spec in specs:
        if spec.x_stream != x_stream:
            x_stream = spec.x_stream
            x_host = x_dev = None
            xi = layer_inputs(spec, 0, "block", parts=("X",))
            x_host, x_dev = xi["X"], bf16_dev(xi["X_bits"])
            del xi
        d = layer_inputs(spec, 0, "block", parts=("W", "dY"))
        ref = oracle.init_alloc(d["dWq"], spec.p, spec.had_block, spec.min_per_row, spec.remainder)
        rp, ci, cf = ref["row_ptr"], ref["col_idx"], ref["coef"]
        sel = _pick_dc(spec, ci, g, 24)
        Wq = oracle.dequant(d["qweight"], d["scales"], d["zeros"], spec.bits, spec.group, spec.d_out, spec.d_in)
        _, Yr = oracle.adapter_fwd(rp, ci, cf, x_host[rows], spec.d_out, spec.had_block, 1.0, Wq, want_z=False)
        dXr = oracle.adapter_bwd_dx(rp, ci, cf, d["dY"][rows], spec.d_in, spec.had_block, 1.0, Wq)
        dcr = _dc_reference(spec, x_host, d["dY"], rp, ci, sel)
        wq = W.QWeight(spec.bits, spec.group, dv(d["qweight"]), dv(d["scales"]), dv(d["zeros"]))
        dY = bf16_dev(d["dY_bits"])
        for algo in ("dense", "sparse"):
            a = W.Adapter(spec.d_in, spec.d_out, spec.had_block, spec.p, dv(rp), dv(ci), dv(cf), algo=algo)
            W.plan_build(a)
            shared = x_stream in z_dev
            Z = z_dev[x_stream] if shared else torch.empty_like(x_dev)
            Z, Y = W.adapter_fwd(a, x_dev, 1.0, wq, Z_out=Z, z_given=shared)
            z_dev[x_stream] = Z
            dc, dX = W.adapter_bwd(a, dY, Z, 1.0, wq)
            torch.cuda.synchronize()
            errs = {"Y": rel_fro(host(Y[ri]), Yr), "dX": rel_fro(host(dX[ri]), dXr),
                    "dc": rel_fro(dc.cpu().numpy()[sel], dcr)}
            assert all(v <= TOL_BF16 for v in errs.values()), (spec.name, algo, errs)
            if shared and spec.name == "k" and algo == "dense":
                # reading the shared transform gives bit for bit what computing it gives
                Z2, Y2 = W.adapter_fwd(a, x_dev, 1.0, wq)
                torch.cuda.synchronize()
                assert torch.equal(Z2, Z) and torch.equal(Y2, Y)
            del a, Y, dc, dX
        del d, dY, wq
