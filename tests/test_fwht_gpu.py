"""qwha_fwht against the oracle's transform, element by element."""

import numpy as np
import pytest

import oracle
from _util import TOL_BF16, TOL_F32, bf16_dev, host, rel_fro, to_dev
from workloads import CONFIGS, bf16_bits_to_f32, f32_to_bf16_bits, layer_inputs, rng_for

pytestmark = pytest.mark.gpu

# (rows, n, had_block): every kernel path (n <= 64, 128..4096, >= 8192), odd and
# even log2, block-diagonal rows, ragged row counts.
SHAPES = [
    (5, 2, 2), (33, 16, 16), (7, 64, 64), (3, 64, 8), (129, 128, 128), (37, 256, 256), (64, 256, 256),
    (11, 512, 512), (65, 1024, 1024), (9, 2048, 2048), (31, 4096, 4096), (3, 4096, 1024),
    (5, 7 * 2048, 2048), (2, 8192, 8192), (3, 32768, 32768), (4, 3 * 256, 256),
]


@pytest.mark.parametrize("rows,n,hb", SHAPES)
@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_fwht_matches_oracle(rows, n, hb, dt):
    import torch
    import walsh_hadamard_sparse_b200 as W

    x = rng_for(20, "fwht", rows, n, hb).standard_normal((rows, n)).astype(np.float32)
    if dt == "bf16":
        bits = f32_to_bf16_bits(x)
        x = bf16_bits_to_f32(bits)
        xd = bf16_dev(bits)
    else:
        xd = to_dev(x)
    z = W.fwht(xd, hb)
    torch.cuda.synchronize()
    ref = oracle.fwht(x.astype(np.float64), hb)
    err = rel_fro(host(z), ref)
    assert err <= (TOL_F32 if dt == "f32" else TOL_BF16), err
    if dt == "f32":
        assert err < 2e-6


def test_fwht_unit_rows_exact_signs():
    import torch
    import walsh_hadamard_sparse_b200 as W

    n = 1024
    z = host(W.fwht(torch.eye(n, device="cuda"), n))
    H = oracle.hadamard(n)
    assert np.array_equal(np.sign(z), np.sign(H))
    assert np.abs(np.abs(z) - 1 / 32).max() == 0.0


def test_fwht_rejects_overlap():
    import torch
    import walsh_hadamard_sparse_b200 as W

    x = torch.zeros(4, 256, device="cuda")
    with pytest.raises(W.QwhaError):
        W.fwht(x, 256, out=x)


@pytest.mark.slow
def test_fwht_full_q_proj_sampled_rows():
    """The q_proj workload's X (8192 x 4096 bf16): every row through the kernel,
    64 seeded rows checked against the oracle."""
    import torch
    import walsh_hadamard_sparse_b200 as W

    spec = CONFIGS["q_proj"][0]
    d = layer_inputs(spec, 0, "q_proj", parts=("X",))
    z = W.fwht(bf16_dev(d["X_bits"]), spec.had_block)
    torch.cuda.synchronize()
    rows = np.sort(rng_for(21, "rows").choice(spec.T, 64, replace=False))
    ref = oracle.fwht(d["X"][rows].astype(np.float64), spec.had_block)
    assert rel_fro(host(z[torch.as_tensor(rows).cuda()]), ref) <= TOL_BF16
